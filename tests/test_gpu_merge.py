"""The split-K merge at every partial count the host distinguishes: one warp
per row (up to 8 and 16 partials), 4, 8 and 16 warps per row (up to 32, 64,
128 and 256), and 32 warps taking batches of 8 (beyond 256, where a warp
merges more than one batch and rescales its running sums to each batch's
max). A single sequence with short partitions keeps the plain grid, so the
count is exactly ceil(length / partition); the last partition is ragged.
Outputs are compared with the float64 oracle."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [2, 9, 17, 33, 65, 129, 257, 600])
@pytest.mark.parametrize("d", [64, 128])
def test_partition_counts(n, d):
    pt = 32
    L = n * pt - 5
    w = W.custom([L], num_q_heads=8, num_kv_heads=2, head_dim=d, dtype="bf16", seed=n + d)
    step = DecodeStep(w, "cuda", partition_tokens=pt)
    step.out.fill_(float("nan"))
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    _, _, want = oracle_step(w)
    got = step.out_f64()
    assert not np.isnan(got).any()
    assert max_abs_err(got, want) <= TOL[w.io_dtype]


def test_sequences_with_fewer_partitions_than_the_launch():
    # the launch is planned for the longest sequence (300 partitions); the
    # others have 1 (no merge), 2, 40 and 299
    lens = [9600, 20, 40, 1270, 9570]
    w = W.custom(lens, num_q_heads=16, num_kv_heads=4, head_dim=128, seed=41)
    step = DecodeStep(w, "cuda", partition_tokens=32)
    step.out.fill_(float("nan"))
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    _, _, want = oracle_step(w)
    got = step.out_f64()
    assert not np.isnan(got).any()
    assert max_abs_err(got, want) <= TOL[w.io_dtype]
