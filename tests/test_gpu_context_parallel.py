"""pa_decode_partial and pa_merge_partials on one GPU: the ranks of a
context-parallel step are played in turn by one process (each call decodes
one rank's block-aligned slice of every history, through that rank's view of
the block tables), the pieces are stacked as an all-gather would stack them,
and the merge must give the float64 oracle's decode of the whole histories.
Each piece is checked against the oracle's own partial too: the output, and
the log2 of the softmax denominator that its (max, sum) pair encodes (the
kernel keeps a reference maximum that may trail the true one, so the pair,
not its parts, is what is fixed). Several GPUs exchanging the pieces over
NCCL is the same code with a real all-gather (context_parallel.decode); it
is not run here."""
import math

import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import context_parallel as CP
from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep

import oracle
from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


def ranks_in_turn(w, step, world, pt=0):
    sl = CP.context_slices(w.context_lens, world, w.block_size)
    rows = (w.batch, w.num_q_heads)
    all_o = torch.empty((world, *rows, w.head_dim), dtype=torch.float32, device="cuda")
    all_ml = torch.empty((world, *rows, 2), dtype=torch.float32, device="cuda")
    views = []
    for r in range(world):
        bt, lens = CP.local_view(w.block_tables, w.context_lens, sl, r, w.block_size)
        maxc = max(int(lens.max()), 1)
        ws_n = B.pa_decode_workspace_size(w.batch, w.num_q_heads, maxc, step.cache, pt)
        ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device="cuda")
        all_o[r].fill_(float("nan"))
        B.pa_decode_partial(step.q, step.k_cache, step.v_cache,
                            torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(),
                            float(w.scale), all_o[r], all_ml[r], step.cache, maxc, pt,
                            ws if ws_n else None, step.stream)
        views.append((bt, lens))
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    return all_o, all_ml, views


@pytest.mark.parametrize("make,world,pt", [
    (lambda: W.custom([1, 40, 700, 0, 33, 2500], num_q_heads=8, num_kv_heads=2, head_dim=128,
                      seed=4), 2, 0),
    (lambda: W.custom([1, 40, 700, 0, 33, 2500], num_q_heads=8, num_kv_heads=2, head_dim=128,
                      seed=4), 3, 64),                  # split partitions inside each slice
    (lambda: W.custom([17, 4000], num_q_heads=16, num_kv_heads=16, head_dim=64, dtype="bf16",
                      seed=5), 8, 0),                   # some ranks hold nothing of seq 0
    (lambda: W.long_context(batch=1, context_len=20000), 4, 0),
    (lambda: W.fp8_beams(batch=12, beam_groups=1, block_size=16, max_len=3000), 2, 0),
])
def test_ranks_in_turn_match_the_whole_decode(make, world, pt):
    w = make()
    step = DecodeStep(w, "cuda")
    step.copy()
    step.append()
    torch.cuda.synchronize()
    all_o, all_ml, views = ranks_in_turn(w, step, world, pt)
    kc, vc, want = oracle_step(w)
    # each piece against the oracle's partial of the same slice
    for r, (bt, lens) in enumerate(views):
        o, m, l = oracle.decode_partial(w.q, w.io_dtype, kc, vc, w.cache_dtype, bt, lens,
                                        w.scale, w.k_scale, w.v_scale)
        got_o = all_o[r].double().cpu().numpy()
        got_m = all_ml[r, ..., 0].double().cpu().numpy()
        got_l = all_ml[r, ..., 1].double().cpu().numpy()
        has = l > 0
        assert np.all(got_o[~has] == 0) and np.all(got_l[~has] == 0)
        assert np.all(np.isneginf(got_m[~has]))
        assert max_abs_err(got_o[has], o[has]) <= 2e-3
        # log2 of sum_j 2^(s_j log2 e): the library's max + log2(sum)
        lse_lib = got_m[has] + np.log2(got_l[has])
        lse_or = m[has] * math.log2(math.e) + np.log2(l[has])
        assert np.max(np.abs(lse_lib - lse_or)) <= 1e-2
    out = torch.full_like(step.out, float("nan"))
    B.pa_merge_partials(all_o, all_ml, out, step.stream)
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    assert not np.isnan(got).any()
    assert max_abs_err(got, want) <= TOL[w.io_dtype]


def test_one_rank_through_the_module_equals_pa_decode_closely():
    # world 1 (no process group): partial, then the merge of one piece
    w = W.custom([5, 900, 3000], num_q_heads=8, num_kv_heads=2, head_dim=128, seed=8)
    step = DecodeStep(w, "cuda")
    step.copy()
    step.append()
    ws_n = B.pa_decode_workspace_size(w.batch, w.num_q_heads, step.max_context, step.cache)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device="cuda")
    out = torch.full_like(step.out, float("nan"))
    CP.decode(step.q, step.k_cache, step.v_cache, step.block_tables, step.context_lens,
              float(w.scale), out, step.cache, step.max_context, workspace=ws if ws_n else None,
              stream=step.stream)
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    _, _, want = oracle_step(w)
    assert max_abs_err(out.double().cpu().numpy(), want) <= TOL[w.io_dtype]


def test_merge_rejects_bad_sizes():
    o = torch.zeros((2, 3, 4, 96), dtype=torch.float32, device="cuda")
    ml = torch.zeros((2, 3, 4, 2), dtype=torch.float32, device="cuda")
    out = torch.zeros((3, 4, 96), dtype=torch.float16, device="cuda")
    with pytest.raises(B.PagedAttentionError) as e:
        B.pa_merge_partials(o, ml, out)  # head_dim 96 is not supported
    assert e.value.status == 1
