"""pa_decode_static_workspace: decode for callers that cannot allocate device
memory (their engine owns all of it, or the call sits on a path where an
allocation's synchronisation is not acceptable). Its output must match the
float64 oracle within the decode tolerance and be bitwise that of pa_decode
with a caller-supplied workspace, call after call, since both use the same
split-K plan and kernels; only where the partials live differs. (The
comparison asks for reproducible results: a single long sequence would
otherwise be decoded in steal mode, whose last bits vary from call to call.)

This file is collected last on purpose, so a failure here leaves every other
test already run."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw", [
    ("long_context", {"batch": 1, "context_len": 20000}),   # 40 partitions: the array is used
    ("llama2_7b", {"batch": 8}),
    ("fp8_beams", {"batch": 24, "beam_groups": 2, "block_size": 32}),
])
def test_matches_the_oracle_and_pa_decode_twice(name, kw):
    with B.deterministic():
        matches_the_oracle_and_pa_decode_twice(name, kw)


def matches_the_oracle_and_pa_decode_twice(name, kw):
    w = W.make(name, **kw)
    step = DecodeStep(w, "cuda")
    step.run()                      # caches after copy + append; out from pa_decode
    torch.cuda.synchronize()
    _, _, want = oracle_step(w)     # the float64 oracle after the same copy + append
    ref = step.out.clone()
    assert B.pa_decode_workspace_size(w.batch, w.num_q_heads, w.max_context, step.cache) > 0
    for _ in range(2):              # the array keeps the first call's partials
        out = torch.full_like(step.out, float("nan"))
        B.pa_decode_static_workspace(step.q, step.k_cache, step.v_cache, step.block_tables,
                                     step.context_lens, float(w.scale), out, step.cache,
                                     step.max_context)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert max_abs_err(got, want) <= TOL[w.io_dtype]
        # the same plan and kernels as pa_decode: the same bits
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert step.device_errors() == 0


def test_rejects_plans_larger_than_the_array():
    w = W.custom([100, 200, 300, 400, 500, 600, 700, 800], num_q_heads=64, num_kv_heads=8,
                 head_dim=128, dtype="bf16")
    step = DecodeStep(w, "cuda")
    max_context = 131072  # 249 partitions: 8 x 64 heads x 249 x 520 B > 32 MiB
    assert B.pa_decode_workspace_size(w.batch, w.num_q_heads, max_context, step.cache) > 32 << 20
    before = step.out.clone()
    with pytest.raises(B.PagedAttentionError) as e:
        B.pa_decode_static_workspace(step.q, step.k_cache, step.v_cache, step.block_tables,
                                     step.context_lens, float(w.scale), step.out, step.cache,
                                     max_context)
    assert e.value.status == 4  # PA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(step.out, before)  # nothing was enqueued
