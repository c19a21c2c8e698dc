"""GPU parity at the full workload sizes, in the launch configuration the
bench times (automatic split-K plan). Whole caches are compared bit for bit
after copy + append; decode outputs are compared with the oracle on a
sample of sequences (the shortest, the longest, beams and random ones)."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep, to_bits

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu

FULL = [
    ("tiny_mha", {}, 4),
    ("llama2_7b", {}, 6),
    ("llama2_70b_prefix", {}, 8),
    ("long_context", {"batch": 1}, 1),
    ("long_context", {"batch": 4}, 1),
    ("fp8_beams", {"block_size": 16}, 16),
    ("fp8_beams", {"block_size": 32}, 16),
    ("fp8_beams", {"block_size": 128}, 16),
]


def sample(w, n, seed=0):
    if n >= w.batch:
        return np.arange(w.batch)
    rng = np.random.default_rng(seed)
    must = {int(np.argmin(w.context_lens)), int(np.argmax(w.context_lens))}
    if "beam_groups" in w.meta:
        must |= {0, 1, 2, 3}  # one whole beam group (forked blocks)
    rest = [i for i in rng.permutation(w.batch).tolist() if i not in must]
    return np.array(sorted(list(must) + rest[:max(0, n - len(must))]))


@pytest.mark.parametrize("name,kw,n", FULL + [("llama2_70b_prefix", {"cascade": True}, 8)],
                         ids=[f"{n}-{k}" for n, k, _ in FULL] + ["llama2_70b_prefix-cascade"])
def test_full_size_step(name, kw, n):
    kw = dict(kw)
    cascade = kw.pop("cascade", False)
    w = W.make(name, **kw)
    step = DecodeStep(w, "cuda",
                      shared_prefix_blocks=w.meta["shared_prefix_blocks"] if cascade else 0)
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    seqs = sample(w, n)
    kc, vc, want = oracle_step(w, seqs)
    assert np.array_equal(to_bits(step.k_cache), kc)
    assert np.array_equal(to_bits(step.v_cache), vc)
    got = step.out_f64()[seqs]
    err = max_abs_err(got, want)
    assert err <= TOL[w.io_dtype], f"{name}{kw}: max abs err {err}"
