"""The work-list decode (a batch of more than one sequence split into more
than one partition): a plan kernel lists the (sequence, partition) items,
largest first, and a persistent grid takes (item, KV head group) units from
a counter. Every unit must be computed exactly once, and computed as the
full grid would: the output of each sequence is compared with the float64
oracle (outputs start as NaN, so a unit never taken shows), and bit for bit
with the same sequence decoded alone (a batch of one keeps the full grid)
with the partition length the plan kernel chose (read back from the
workspace, where the plan publishes it: 1, 2 or 4 times the host's, or up to
8 times it to hold the longest sequence whole) and a
plan of as many partitions as the batch's launch had, so that the merge
runs the same code. The decodes alone ask for reproducible results, which
keeps each CTA on its own partition (no steal mode)."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep, to_bits

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


def listed_vs_alone(w, pt, window=0, fused=False, repeats=2):
    step = DecodeStep(w, "cuda", partition_tokens=pt, window=window, fused=fused)
    step.copy()
    if fused:
        step.out.fill_(float("nan"))
        step.append_decode()
    else:
        step.append()
        outs = []
        for _ in range(repeats):  # the counter and list are rebuilt by every call
            step.out.fill_(float("nan"))
            step.decode()
            torch.cuda.synchronize()
            outs.append(to_bits(step.out).copy())
        assert all(np.array_equal(outs[0], o) for o in outs[1:])
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    _, _, want = oracle_step(w, window=window)
    got = step.out_f64()
    assert not np.isnan(got).any(), "a unit was never computed"
    err = max_abs_err(got, want)
    assert err <= TOL[w.io_dtype], f"max abs err {err}"
    bits = to_bits(step.out)
    # the launch's plan: the host's partition length and count, and the
    # length the plan kernel chose (workspace: partials, (max, sum) pairs,
    # then the work list's counter section [ticket, items, partition length])
    span = min(step.max_context, window + 15) if window else step.max_context
    if pt == 0:
        pt = B.pa_decode_partition_tokens(w.batch, span, step.cache)
    n_parts = -(-span // pt)
    rows = w.batch * w.num_q_heads
    list_at = (-(-(rows * n_parts * w.head_dim * 4) // 256) * 256 +
               -(-(rows * n_parts * 8) // 256) * 256)
    pt_used = int(step.workspace[list_at + 8:list_at + 12].view(torch.int32).item())
    # the longest attended span (a window's starts at its 16-aligned base)
    lens = step.context_lens.cpu().numpy().astype(int)
    bases = [((L - window) & ~15) if window and L > window else 0 for L in lens]
    longest = max([L - b for L, b in zip(lens, bases)] + [0])
    assert pt_used % 16 == 0 and pt <= pt_used <= 8 * pt, (pt, pt_used)
    assert pt_used in (pt, 2 * pt, 4 * pt) or pt_used >= longest, (pt, pt_used, longest)
    # each sequence alone: the full grid at that length, with a plan of as
    # many partitions (the merge picks its code by the plan's count; a
    # window's plan spans window + 15 tokens whatever max_context is)
    maxc_one = step.max_context if window else n_parts * pt_used
    ws_one = (B.pa_decode_sliding_window_workspace_size(1, w.num_q_heads, maxc_one, window,
                                                        step.cache, pt_used) if window else
              B.pa_decode_workspace_size(1, w.num_q_heads, maxc_one, step.cache, pt_used))
    wsb = torch.empty(max(ws_one, 1), dtype=torch.uint8, device="cuda")
    one = torch.empty_like(step.out[:1])
    det = B.deterministic()
    det.__enter__()
    for b in range(w.batch):
        one.fill_(float("nan"))
        args = (step.q[b:b + 1], step.k_cache, step.v_cache, step.block_tables[b:b + 1],
                step.context_lens[b:b + 1], float(w.scale), one, step.cache, maxc_one)
        if window:
            B.pa_decode_sliding_window(*args, window, pt_used, wsb if ws_one else None,
                                       step.stream)
        else:
            B.pa_decode(*args, pt_used, wsb if ws_one else None, step.stream)
        torch.cuda.synchronize()
        if not np.array_equal(to_bits(one)[0], bits[b]):
            det.__exit__(None, None, None)
            raise AssertionError(f"sequence {b} differs from its decode alone")
    det.__exit__(None, None, None)
    assert step.device_errors() == 0
    return step, pt_used


def test_mixed_lengths_with_empty_and_exact_partitions():
    # empty sequences, lengths on and either side of partition ends, and one
    # sequence many partitions longer than the rest
    lens = [0, 1, 15, 16, 17, 255, 256, 257, 512, 1000, 0, 4000, 3, 768]
    w = W.custom(lens, num_q_heads=8, num_kv_heads=2, head_dim=128, seed=5)
    step, _ = listed_vs_alone(w, pt=256)
    got = step.out_f64()
    assert np.all(got[0] == 0) and np.all(got[10] == 0)


@pytest.mark.parametrize("hq,hkv,d,dtype", [
    (32, 32, 128, "f16"),   # MHA, many units per item
    (16, 1, 128, "bf16"),   # group of 16: two column blocks
    (24, 1, 64, "bf16"),    # a full and a partial head group
    (40, 8, 64, "f16"),     # group of 5 at head_dim 64
])
def test_head_groupings(hq, hkv, d, dtype):
    w = W.custom([5, 300, 1200, 64, 2049, 700], num_q_heads=hq, num_kv_heads=hkv,
                 head_dim=d, dtype=dtype, seed=hq + d)
    listed_vs_alone(w, pt=128)


def test_many_sequences_more_units_than_resident_ctas():
    # enough tokens per slot that the plan lengthens the partitions
    rng = np.random.default_rng(3)
    lens = np.clip(np.exp(rng.normal(np.log(300), 1.0, size=300)), 1, 6000).astype(int)
    w = W.custom(lens.tolist(), num_q_heads=8, num_kv_heads=8, head_dim=128, seed=9)
    _, pt_used = listed_vs_alone(w, pt=256, repeats=3)
    assert pt_used > 256


def test_fp8_beams_automatic_partition():
    w = W.fp8_beams(batch=48, beam_groups=4, block_size=16, max_len=3000)
    listed_vs_alone(w, pt=0)


def test_sliding_window():
    w = W.custom([10, 700, 1500, 3000, 90], num_q_heads=8, num_kv_heads=2, head_dim=128,
                 seed=11)
    listed_vs_alone(w, pt=64, window=500)


@pytest.mark.parametrize("family", ["fp8", "f16"])
def test_fused_append(family):
    if family == "fp8":
        w = W.fp8_beams(batch=40, beam_groups=4, block_size=16, max_len=2500)
    else:
        w = W.custom([1, 40, 600, 1700, 2], num_q_heads=8, num_kv_heads=2, head_dim=128, seed=13)
    step, _ = listed_vs_alone(w, pt=256, fused=True)
    kc, vc, _ = oracle_step(w)
    assert np.array_equal(to_bits(step.k_cache), kc)
    assert np.array_equal(to_bits(step.v_cache), vc)
