"""Context parallelism on the host (no GPU): how histories are dealt out to
ranks, each rank's view of its slice, and a full step over a 2- and 3-rank
gloo group with the float64 oracle standing in for the library's partial
decode and merge; the merged result must equal the oracle's decode of the
whole histories. The oracle's split identity (parts merged = the whole) is
pinned against its own C decode here too."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402
from paged_kv_cache_410_b200 import context_parallel as CP  # noqa: E402
from paged_kv_cache_410_b200 import workloads as W  # noqa: E402


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_slices_cover_each_history_once_on_block_boundaries(world):
    lens = np.array([0, 1, 15, 16, 17, 100, 1000, 4097])
    bs = 16
    sl = CP.context_slices(lens, world, bs)
    assert sl.shape == (world, len(lens), 2)
    for b, L in enumerate(lens):
        ends = 0
        sizes = []
        for r in range(world):
            s, e = sl[r, b]
            assert s == ends and s <= e <= L      # contiguous, in order
            assert s % bs == 0 or s == L           # a block boundary (or empty at the end)
            sizes.append(-(-(e - s) // bs))
            ends = e
        assert ends == L
        assert max(sizes) - min(sizes) <= 1        # blocks dealt out evenly


def test_local_view_lists_the_slice_blocks():
    w = W.custom([70, 3, 0], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16, seed=2)
    sl = CP.context_slices(w.context_lens, 2, 16)
    bt0, l0 = CP.local_view(w.block_tables, w.context_lens, sl, 0, 16)
    bt1, l1 = CP.local_view(w.block_tables, w.context_lens, sl, 1, 16)
    assert l0.tolist() == [48, 3, 0] and l1.tolist() == [22, 0, 0]
    assert bt0[0, :3].tolist() == w.block_tables[0, :3].tolist()
    assert bt1[0, :2].tolist() == w.block_tables[0, 3:5].tolist()


def _oracle_parts(w, world):
    sl = CP.context_slices(w.context_lens, world, w.block_size)
    parts = []
    for r in range(world):
        bt, lens = CP.local_view(w.block_tables, w.context_lens, sl, r, w.block_size)
        parts.append(oracle.decode_partial(w.q, w.io_dtype, w.k_pool, w.v_pool, w.cache_dtype,
                                           bt, lens, w.scale))
    return parts


@pytest.mark.parametrize("world", [1, 2, 5])
def test_oracle_split_identity(world):
    # merging the parts of any block-aligned split gives the oracle's C decode
    # of the whole histories; a rank with an empty part contributes nothing
    w = W.custom([1, 40, 700, 0, 33], num_q_heads=8, num_kv_heads=2, head_dim=64, seed=4)
    parts = _oracle_parts(w, world)
    got = oracle.merge_partials(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]),
                                np.stack([p[2] for p in parts]))
    want = oracle.decode(w.q, w.io_dtype, w.k_pool, w.v_pool, w.cache_dtype, w.block_tables,
                         w.context_lens, w.scale)
    assert np.max(np.abs(got - want)) < 1e-12
    assert np.all(got[3] == 0)


def _standin_partial(w):
    def partial(q, k_cache, v_cache, block_tables, context_lens, scale, part_o, part_ml, cache,
                max_context, partition_tokens, workspace, stream):
        o, m, l = oracle.decode_partial(q.numpy(), w.io_dtype, k_cache, v_cache, w.cache_dtype,
                                        block_tables, context_lens, scale)
        part_o.copy_(torch.from_numpy(o))
        part_ml[..., 0] = torch.from_numpy(m)
        part_ml[..., 1] = torch.from_numpy(l)
    return partial


def _standin_merge(all_o, all_ml, out, stream):
    out.copy_(torch.from_numpy(oracle.merge_partials(all_o.double().numpy(),
                                                     all_ml[..., 0].double().numpy(),
                                                     all_ml[..., 1].double().numpy())))


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.custom([5, 300, 1000, 16, 0, 77], num_q_heads=8, num_kv_heads=2, head_dim=64,
                     seed=6)
        sl = CP.context_slices(w.context_lens, world, w.block_size)
        bt, lens = CP.local_view(w.block_tables, w.context_lens, sl, rank, w.block_size)
        out = torch.zeros((w.batch, w.num_q_heads, w.head_dim), dtype=torch.float64)
        CP.decode(torch.from_numpy(w.q.astype(np.int16)), w.k_pool, w.v_pool, bt, lens,
                  w.scale, out, None, int(lens.max()), partial=_standin_partial(w),
                  merge=_standin_merge)
        want = oracle.decode(w.q, w.io_dtype, w.k_pool, w.v_pool, w.cache_dtype,
                             w.block_tables, w.context_lens, w.scale)
        q.put((rank, float(np.max(np.abs(out.numpy() - want)))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_step_over_gloo_ranks_matches_the_whole_decode(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + world * 10 + os.getpid() % 500
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == list(range(world))
    for _, err in res:
        assert err < 1e-6  # (the pieces travel as float32)
