"""Steal mode: a single sequence split into partitions of 1024 tokens or
more, over a 16-bit cache with blocks of 16 tokens or more, is decoded by a
grid whose CTAs of one KV head group share the sequence's tiles through a
counter in the workspace (each CTA's share of about half the row, then
chunks of four tiles per warp from a common pool) instead of each taking a
fixed partition; a CTA on a slower SM then takes fewer tiles. Which CTA
takes which tiles changes from call to call, so the output is compared with
the float64 oracle within the decode tolerance, call after call, with the
workspace refilled with garbage before each call (counters of no epoch of
this process). When the whole grid fits on the GPU at once, each row's CTAs
merge the row's partials themselves inside the (cooperative) launch, with
two more counters per row; otherwise the merge kernel runs after the grid.
After each call the counters are back at zero (the merge kernel, or the
row's last CTA, zeroes them), which also shows that steal mode ran; a
launch outside steal mode (shorter
partitions, blocks of 8 tokens, reproducible results asked for) leaves that
section as it was."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


def counters_at(w, span, pt):
    """Byte offset of the work list's section (where the steal counters
    sit) in the split-K workspace: partials, then (max, sum) pairs."""
    n_parts = -(-span // pt)
    rows = w.batch * w.num_q_heads
    return (-(-(rows * n_parts * w.head_dim * 4) // 256) * 256 +
            -(-(rows * n_parts * 8) // 256) * 256)


def run_calls(w, pt, window=0, calls=3, expect_steal=True):
    step = DecodeStep(w, "cuda", partition_tokens=pt, window=window)
    step.copy()
    step.append()
    torch.cuda.synchronize()
    _, _, want = oracle_step(w, window=window)
    span = min(step.max_context, window + 15) if window else step.max_context
    if pt == 0:
        pt = B.pa_decode_partition_tokens(w.batch, span, step.cache)
    at = counters_at(w, span, pt)
    group = w.num_q_heads // w.num_kv_heads
    hb = w.num_kv_heads * -(-group // 16)
    for c in range(calls):
        step.workspace.fill_(0xA5 if c % 2 else 0xFF)
        step.out.fill_(float("nan"))
        step.decode()
        torch.cuda.synchronize()
        assert step.device_errors() == 0
        got = step.out_f64()
        assert not np.isnan(got).any()
        err = max_abs_err(got, want)
        assert err <= TOL[w.io_dtype], f"call {c}: max abs err {err}"
        ctr = step.workspace[at:at + 8 * hb].view(torch.int64).cpu().numpy()
        if expect_steal:
            assert np.all(ctr == 0), "the steal counters were not reset"
        else:
            assert not np.any(ctr == 0)
    return step


@pytest.mark.parametrize("L,pt", [(1025, 1024), (1100, 1024), (3000, 1024), (20000, 1024),
                                  (70001, 2048)])
def test_lengths(L, pt):
    # from a last partition of one token (no share: the whole row is the
    # pool) to 35 CTAs per KV head over 4375 tiles
    w = W.custom([L], num_q_heads=32, num_kv_heads=8, head_dim=128, seed=L)
    run_calls(w, pt)


@pytest.mark.parametrize("hq,hkv,d,dtype", [
    (32, 32, 128, "f16"),   # MHA: 32 counters
    (16, 1, 128, "bf16"),   # group of 16: two column blocks, one counter
    (24, 1, 64, "bf16"),    # a full and a partial head group: two counters
    (40, 8, 64, "f16"),     # group of 5 at head_dim 64
])
def test_head_groupings(hq, hkv, d, dtype):
    w = W.custom([5001], num_q_heads=hq, num_kv_heads=hkv, head_dim=d, dtype=dtype,
                 seed=hq * 7 + d)
    run_calls(w, 1024)


def test_block_size_64_and_automatic_partition():
    # 32 KV heads: one wave of CTAs gives 13 partitions of 1232 tokens
    w = W.custom([16000], num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=64,
                 dtype="bf16", seed=21)
    step = DecodeStep(w, "cuda")
    assert B.pa_decode_partition_tokens(1, step.max_context, step.cache) >= 1024
    run_calls(w, 0)


def test_sliding_window():
    # the first attended tile starts inside a block; the window's span sets
    # the plan
    w = W.custom([9000], num_q_heads=16, num_kv_heads=4, head_dim=128, seed=23)
    run_calls(w, 1024, window=5000)


def test_grid_larger_than_the_gpu_holds():
    # 20 partitions x 32 KV heads: more CTAs than fit at once, so the rows
    # are merged by the merge kernel after the grid (smaller grids merge
    # their rows inside the launch)
    w = W.custom([20000], num_q_heads=32, num_kv_heads=32, head_dim=128, seed=29)
    run_calls(w, 1024)


def test_static_workspace():
    w = W.custom([12000], num_q_heads=32, num_kv_heads=8, head_dim=128, seed=27)
    step = DecodeStep(w, "cuda")
    step.copy()
    step.append()
    _, _, want = oracle_step(w)
    for _ in range(3):
        step.out.fill_(float("nan"))
        B.pa_decode_static_workspace(step.q, step.k_cache, step.v_cache, step.block_tables,
                                     step.context_lens, float(w.scale), step.out, step.cache,
                                     step.max_context, 1024)
        torch.cuda.synchronize()
        assert step.device_errors() == 0
        assert max_abs_err(step.out_f64(), want) <= TOL[w.io_dtype]


@pytest.mark.parametrize("why", ["short partitions", "blocks of 8 tokens", "reproducible"])
def test_not_used(why):
    bs = 8 if why == "blocks of 8 tokens" else 16
    w = W.custom([5000], num_q_heads=16, num_kv_heads=4, head_dim=128, block_size=bs, seed=25)
    pt = 512 if why == "short partitions" else 1024
    if why == "reproducible":
        with B.deterministic():
            step = run_calls(w, pt, expect_steal=False)
            first = step.out.clone()
            step.decode()
            torch.cuda.synchronize()
            assert torch.equal(step.out, first)
        assert not B.pa_set_deterministic(False)  # the previous setting is back
    else:
        run_calls(w, pt, expect_steal=False)


def test_merge_wait_timeout_is_reported_and_recoverable():
    # the in-launch merge's wait for a row's partials is bounded: with one
    # CTA per row not counting its partial, every wait runs out (1 s), the
    # device error word reports PA_DEVERR_TIMEOUT and no row is merged;
    # afterwards the context is usable and a normal call matches the oracle
    w = W.custom([12000], num_q_heads=32, num_kv_heads=8, head_dim=128, seed=31)
    step = DecodeStep(w, "cuda", partition_tokens=1024)
    step.copy()
    step.append()
    torch.cuda.synchronize()
    step.out.fill_(float("nan"))
    B.pa_testing_withhold_steal_counts(1)
    try:
        step.decode()
        torch.cuda.synchronize()
        assert step.device_errors() & B.DEVERR_TIMEOUT
        assert torch.isnan(step.out).all()  # nothing was merged
    finally:
        B.pa_testing_withhold_steal_counts(0)
    for _ in range(2):
        step.decode()
        torch.cuda.synchronize()
        assert step.device_errors() == 0
    _, _, want = oracle_step(w)
    assert max_abs_err(step.out_f64(), want) <= TOL[w.io_dtype]


@pytest.mark.parametrize("L", [0, 3000, 9000])
def test_launch_planned_for_longer_histories(L):
    # max_context (what the launch and its plan are sized for) well above the
    # sequence's length: the CTA columns past the sequence's partitions leave
    # at once, and only its own partitions' CTAs share its tiles and merge
    w = W.custom([max(L, 1)], num_q_heads=32, num_kv_heads=8, head_dim=128, seed=33 + L)
    step = DecodeStep(w, "cuda")
    step.copy()
    step.append()
    step.context_lens.fill_(L)
    w.context_lens[:] = L
    maxc = 40000
    ws_n = B.pa_decode_workspace_size(1, w.num_q_heads, maxc, step.cache, 1024)
    ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
    for fill in (0xFF, 0x00):
        ws.fill_(fill)
        out = torch.full_like(step.out, float("nan"))
        B.pa_decode(step.q, step.k_cache, step.v_cache, step.block_tables, step.context_lens,
                    float(w.scale), out, step.cache, maxc, 1024, ws, step.stream)
        torch.cuda.synchronize()
        assert step.device_errors() == 0
        got = out.double().cpu().numpy()
        if L == 0:
            assert np.all(got == 0)
        else:
            _, _, want = oracle_step(w)
            assert max_abs_err(got, want) <= TOL[w.io_dtype]
