"""GPU parity at the full workload sizes, in the launch configuration the
bench times (automatic split-K plan). Whole caches are compared bit for bit
after copy + append, and the decode output of every sequence of the batch is
compared with the float64 oracle."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep, to_bits

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu

FULL = [
    ("tiny_mha", {}),
    ("llama2_7b", {}),
    ("llama2_70b_prefix", {}),
    ("long_context", {"batch": 1}),
    ("long_context", {"batch": 4}),
    ("fp8_beams", {"block_size": 16}),
    ("fp8_beams", {"block_size": 32}),
    ("fp8_beams", {"block_size": 128}),
]


@pytest.mark.parametrize("name,kw", FULL + [("llama2_70b_prefix", {"cascade": True})],
                         ids=[f"{n}-{k}" for n, k in FULL] + ["llama2_70b_prefix-cascade"])
def test_full_size_step(name, kw):
    kw = dict(kw)
    cascade = kw.pop("cascade", False)
    w = W.make(name, **kw)
    step = DecodeStep(w, "cuda",
                      shared_prefix_blocks=w.meta["shared_prefix_blocks"] if cascade else 0)
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    kc, vc, want = oracle_step(w)
    assert np.array_equal(to_bits(step.k_cache), kc)
    assert np.array_equal(to_bits(step.v_cache), vc)
    got = step.out_f64()
    assert got.shape == want.shape == (w.batch, w.num_q_heads, w.head_dim)
    err = max_abs_err(got, want)
    assert err <= TOL[w.io_dtype], f"{name}{kw}: max abs err {err}"
