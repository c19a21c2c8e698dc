"""Host block manager (include/pa_block_manager.h) on the CPU.

What the pages fix and these tests check: blocks of a fixed size, taken on
demand -- a sequence gets its second block only when token BS+1 arrives (page
'AI 陪读顶会论文（三）：KV Cache 显存占用计算与 PagedAttention 原理拆解',
section 'PagedAttention 的破局哲学'); a shared prefix is stored once and
reference-counted, and branches copy a block only where they diverge (KV cache
article, section 'PagedAttention：把操作系统的老智慧搬进推理引擎'); a radix tree
of token ids lets later requests reuse a cached prefix (chapter '第2章 KV
Cache：模型内部的显存复用')."""
import ctypes
import functools
import re
import os

import numpy as np
import pytest

from paged_kv_cache_410_b200 import block_manager as BM
from paged_kv_cache_410_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def test_header_symbols_are_exported():
    header = open(os.path.join(ROOT, "include", "pa_block_manager.h")).read()
    text = re.sub(r"/\*.*?\*/", "", header,
                  flags=re.S)
    names = sorted(set(re.findall(r"\b(pa_bm_[a-z_]+)\s*\(", text)))
    assert names == sorted(BM.EXPORTED)
    lib = BM._lib()
    for n in names:
        assert hasattr(lib, n)


def test_blocks_are_taken_on_demand():
    bm = BM.BlockManager(10, 16)
    bm.add_sequence(1, range(16))                    # 16 tokens: one block
    assert bm.num_free_blocks == 9
    slot, cow = bm.append_token(1, 99)               # token 17: the second block
    assert cow is None and bm.num_free_blocks == 8
    tables, lens = bm.block_tables([1], 4)
    assert lens.tolist() == [17]
    assert slot == tables[0, 1] * 16 + 0
    for k in range(15):                              # tokens 18..32 fill it
        bm.append_token(1, k)
    assert bm.num_free_blocks == 8
    bm.append_token(1, 0)                            # token 33: the third block
    assert bm.num_free_blocks == 7


def test_slots_follow_the_block_table():
    bm = BM.BlockManager(50, 8)
    bm.add_sequence(7, range(29))
    tables, lens = bm.block_tables([7], 6)
    slots = bm.slots(7, 0, 29)
    j = np.arange(29)
    assert np.array_equal(slots, tables[0, j // 8].astype(np.int64) * 8 + j % 8)
    assert len(set(tables[0, :4].tolist())) == 4 and tables[0, 4:].tolist() == [0, 0]


def test_fork_shares_blocks_and_copies_only_the_partial_last_block():
    bm = BM.BlockManager(20, 16)
    bm.add_sequence(0, range(40))                    # 2 full blocks + 8 tokens in a third
    for c in (1, 2, 3):
        bm.fork(0, c)
    t, _ = bm.block_tables([0, 1, 2, 3], 4)
    assert (t == t[0]).all()                         # the beams share every block
    assert [bm.refcount(b) for b in t[0, :3]] == [4, 4, 4]
    free0 = bm.num_free_blocks
    copies = []
    for s in (0, 1, 2, 3):
        slot, cow = bm.append_token(s, 1000 + s)
        if cow:
            copies.append(cow)
    # three beams copy the shared partial block; the last one writes in place
    assert len(copies) == 3 and {c[0] for c in copies} == {int(t[0, 2])}
    assert bm.num_free_blocks == free0 - 3
    t2, lens = bm.block_tables([0, 1, 2, 3], 4)
    assert lens.tolist() == [41] * 4
    assert (t2[:, :2] == t[0, :2]).all()             # full blocks still shared
    assert len(set(t2[:, 2].tolist())) == 4          # last blocks now private
    assert [bm.refcount(b) for b in t2[0, :2]] == [4, 4]


def test_fork_at_a_block_boundary_needs_no_copy():
    bm = BM.BlockManager(20, 16)
    bm.add_sequence(0, range(32))
    bm.fork(0, 1)
    for s in (0, 1):
        _, cow = bm.append_token(s, 5)
        assert cow is None


def test_freeing_drops_references_not_shared_blocks():
    bm = BM.BlockManager(12, 4)
    bm.add_sequence(0, range(10))                    # 3 blocks
    bm.fork(0, 1)
    bm.free_sequence(0)
    assert bm.num_free_blocks == 9                   # the child still holds all three
    t, _ = bm.block_tables([1], 3)
    assert [bm.refcount(b) for b in t[0]] == [1, 1, 1]
    bm.free_sequence(1)
    assert bm.num_free_blocks == 12


def test_prefix_cache_reuses_full_prompt_blocks():
    bm = BM.BlockManager(40, 16, prefix_cache=True)
    system = list(range(100, 132))                   # a 32-token system prompt
    assert bm.add_sequence(1, system + [1, 2, 3]) == 0
    assert bm.add_sequence(2, system + [7, 8]) == 32
    assert bm.add_sequence(3, [5] + system) == 0     # different first block: no reuse
    t, _ = bm.block_tables([1, 2, 3], 3)
    assert (t[0, :2] == t[1, :2]).all() and t[0, 2] != t[1, 2]
    assert not set(t[2, :2].tolist()) & set(t[0, :2].tolist())
    # the cached blocks outlive the requests that made them
    bm.free_sequence(1)
    bm.free_sequence(2)
    assert bm.num_cached_blocks >= 2
    assert bm.add_sequence(4, system + [9]) == 32
    t4, _ = bm.block_tables([4], 3)
    assert (t4[0, :2] == t[0, :2]).all()


def test_partial_prefix_match_stops_at_the_first_different_block():
    bm = BM.BlockManager(40, 4, prefix_cache=True)
    bm.add_sequence(1, [1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12])
    assert bm.add_sequence(2, [1, 2, 3, 4, 5, 6, 7, 0, 9, 10, 11, 12]) == 4
    assert bm.add_sequence(3, [1, 2, 3, 4, 5, 6, 7, 8, 9]) == 8


def test_blocks_filled_by_decoding_join_the_cache():
    bm = BM.BlockManager(20, 8, prefix_cache=True)
    bm.add_sequence(1, [3] * 5)
    for k in range(3):
        bm.append_token(1, 3)                        # the first block fills with token 8
    assert bm.add_sequence(2, [3] * 8 + [4]) == 8


def test_lru_eviction_of_cached_blocks():
    bm = BM.BlockManager(4, 2, prefix_cache=True)
    bm.add_sequence(1, [1, 1])                       # cached block A
    bm.free_sequence(1)
    bm.add_sequence(2, [2, 2])                       # cached block B
    bm.free_sequence(2)
    assert bm.num_free_blocks == 2 and bm.num_cached_blocks == 2
    assert bm.add_sequence(3, [1, 1]) == 2           # touches A: B is now least recent
    bm.free_sequence(3)
    bm.add_sequence(4, [9, 9, 9, 9, 9, 9])           # 3 blocks: 2 free + 1 evicted (B)
    assert bm.num_free_blocks == 0
    bm.free_sequence(4)
    assert bm.add_sequence(5, [1, 1]) == 2           # A survived
    assert bm.add_sequence(6, [2, 2]) == 0           # B did not


def test_out_of_blocks_leaves_the_manager_unchanged():
    bm = BM.BlockManager(3, 4)
    bm.add_sequence(1, range(8))
    with pytest.raises(BM.BlockManagerError) as e:
        bm.add_sequence(2, range(8))
    assert e.value.code == BM.ERR_NO_BLOCKS
    assert bm.num_free_blocks == 1
    with pytest.raises(BM.BlockManagerError):
        bm.length(2)


def test_release_before_frees_blocks_outside_a_window():
    bm = BM.BlockManager(10, 4)
    bm.add_sequence(1, range(18))                    # 5 blocks
    bm.release_before(1, 9)                          # blocks 0 and 1 hold only tokens < 8
    assert bm.num_free_blocks == 7
    bm.slots(1, 8, 10)
    with pytest.raises(BM.BlockManagerError):
        bm.slots(1, 7, 2)
    bm.free_sequence(1)
    assert bm.num_free_blocks == 10


def test_invalid_calls():
    bm = BM.BlockManager(5, 4)
    bm.add_sequence(1, range(3))
    for fn in (lambda: bm.add_sequence(1, [1]), lambda: bm.append_token(9),
               lambda: bm.fork(9, 10), lambda: bm.fork(1, 1), lambda: bm.free_sequence(9),
               lambda: bm.slots(1, 2, 5), lambda: bm.block_tables([1, 9], 2)):
        with pytest.raises(BM.BlockManagerError):
            fn()
    with pytest.raises(BM.BlockManagerError) as e:
        bm.block_tables([1], 0)
    bm.add_sequence(2, range(9))
    with pytest.raises(BM.BlockManagerError) as e:
        bm.block_tables([2], 2)
    assert e.value.code == BM.ERR_CAPACITY


def test_incremental_tables_rewrite_only_changed_rows():
    bm = BM.BlockManager(64, 4)
    for sid in (1, 2, 3):
        bm.add_sequence(sid, range(6))              # 2 blocks each, last one half full
    ids = [1, 2, 3]
    tables = np.full((3, 5), -7, dtype=np.int32)     # garbage the first call must overwrite
    lens = np.zeros(3, dtype=np.int32)
    ver = np.zeros(3, dtype=np.uint64)
    assert bm.block_tables_update(ids, tables, lens, ver) == 3
    assert (ver != 0).all() and len(set(ver.tolist())) == 3   # unique, never 0
    full_t, full_l = bm.block_tables(ids, 5)
    assert (tables == full_t).all() and (lens == full_l).all()
    assert bm.block_tables_update(ids, tables, lens, ver) == 0  # nothing changed
    bm.append_token(1)                               # position 6: same block
    bm.append_token(1)                               # position 7: same block
    bm.append_token(2); bm.append_token(2); bm.append_token(2)  # position 8: new block
    assert bm.block_tables_update(ids, tables, lens, ver) == 1
    full_t, full_l = bm.block_tables(ids, 5)
    assert (tables == full_t).all() and (lens == full_l).all()
    # fork 3 into a row that held 1's table; appending to the shared partial block copies it
    bm.fork(3, 4)
    ids = [4, 2, 3]
    assert bm.block_tables_update(ids, tables, lens, ver) == 1
    _, cow = bm.append_token(4)
    assert cow is not None
    assert bm.block_tables_update(ids, tables, lens, ver) == 1
    # two sequences trade rows: both rewritten
    ids = [2, 4, 3]
    assert bm.block_tables_update(ids, tables, lens, ver) == 2
    full_t, full_l = bm.block_tables(ids, 5)
    assert (tables == full_t).all() and (lens == full_l).all()
    # releasing blocks outside a window keeps the table (the full export keeps it too)
    bm.release_before(2, 4)
    assert bm.block_tables_update(ids, tables, lens, ver) == 0
    assert (tables == bm.block_tables(ids, 5)[0]).all()
    # a failing call writes nothing
    bm.add_sequence(9, range(30))                    # 8 blocks > 5
    before = (tables.copy(), lens.copy(), ver.copy())
    with pytest.raises(BM.BlockManagerError) as e:
        bm.block_tables_update([2, 9, 3], tables, lens, ver)
    assert e.value.code == BM.ERR_CAPACITY
    for x, y in zip(before, (tables, lens, ver)):
        assert (x == y).all()


def test_incremental_tables_match_the_full_export_under_churn():
    rng = np.random.default_rng(7)
    bm = BM.BlockManager(4000, 8, prefix_cache=True)
    prompt = list(range(40))
    batch, max_blocks = 24, 64
    ids = []
    for b in range(batch):
        bm.add_sequence(b, prompt + [1000 + b] * int(rng.integers(1, 20)))
        ids.append(b)
    tables = np.zeros((batch, max_blocks), dtype=np.int32)
    lens = np.zeros(batch, dtype=np.int32)
    ver = np.zeros(batch, dtype=np.uint64)
    next_id, total_written = batch, 0
    for step in range(200):
        for sid in ids:
            bm.append_token(sid, int(rng.integers(0, 50)))
        if step % 7 == 3:                            # a beam forks into another's row
            parent, victim = rng.choice(batch, 2, replace=False)
            bm.fork(ids[parent], next_id)
            bm.free_sequence(ids[victim])
            ids[victim] = next_id
            next_id += 1
        if step % 11 == 5:                           # two rows trade places
            i, j = rng.choice(batch, 2, replace=False)
            ids[i], ids[j] = ids[j], ids[i]
        total_written += bm.block_tables_update(ids, tables, lens, ver)
        full_t, full_l = bm.block_tables(ids, max_blocks)
        assert (tables == full_t).all() and (lens == full_l).all(), step
    # a row changes about once per block_size appends, plus the churn
    assert batch * 200 // 16 <= total_written < batch * 200 // 2


def test_host_benchmark_runs():
    # the block manager's host benchmark (serving-step loop) builds and
    # reports sensible numbers on a small case
    import json
    import subprocess
    from paged_kv_cache_410_b200 import build
    exe = build.build_block_manager_bench()
    out = subprocess.run([exe, "16", "100", "256", "16", "16", "10"], check=True,
                         capture_output=True, text=True).stdout
    r = json.loads(out.strip().splitlines()[-1])
    assert r["batch"] == 16 and r["steps"] == 100
    # every request after the first reuses the 256-token system prompt (16 blocks)
    assert r["prompt_tokens_cached"] == 15 * 256
    assert r["forks"] == 40 and r["cow_pairs"] > 0
    assert r["append_ns_per_token"] > 0 and r["step_us"] > 0
    assert 0 < r["block_tables_update_us_per_step"] and 0 < r["rows_rewritten_per_step"] < 16
    assert r["append_batched_ns_per_token"] > 0     # the batched pass gave the same slots


def _check_contents(bm, seqs, released, content, bs):
    """Every live sequence still reads its own tokens through its slots."""
    for sid, toks in seqs.items():
        first = released[sid] // bs * bs
        if first >= len(toks):
            continue
        slots = bm.slots(sid, first, len(toks) - first)
        got = [content.get(int(s)) for s in slots]
        assert got == toks[first:], (sid, first)


@functools.lru_cache(maxsize=None)
def _random_serving(seed):
    """A random mix of admissions (prompts built from a few shared system
    prompts), appends, forks, ends and window releases on a small pool, with
    the caller's K/V writes mirrored in a model of the cache contents: each
    slot holds the token written there last; prompt tokens past the cached
    prefix are written after admission; copy-on-write pairs are applied
    before the append. After every operation each live sequence must read
    exactly its own tokens (so no block it uses was handed to another
    sequence, evicted, or written by a sibling), failed calls must change
    nothing, and the block accounting must add up."""
    rng = np.random.default_rng(seed)
    bs = int(rng.choice([1, 2, 4, 8]))
    nb = int(rng.integers(24, 64))
    bm = BM.BlockManager(nb, bs, prefix_cache=seed % 4 != 3)
    systems = [list(rng.integers(0, 5, size=int(rng.integers(0, 3 * bs + 2))))
               for _ in range(3)]
    content, seqs, released = {}, {}, {}
    next_id, failures, hits, copies = 0, 0, 0, 0

    def write(slot, tok):
        content[int(slot)] = int(tok)

    def snapshot():
        return bm.num_free_blocks, bm.num_cached_blocks

    for step in range(400):
        op = rng.choice(["add", "append", "append", "append", "batch", "fork", "free",
                         "release"])
        live = list(seqs)
        if op == "add" or not live:
            toks = [int(t) for t in systems[int(rng.integers(0, 3))]]
            toks += [int(t) for t in rng.integers(0, 5, size=int(rng.integers(1, 2 * bs + 2)))]
            before = snapshot()
            try:
                cached = bm.add_sequence(next_id, toks)
            except BM.BlockManagerError as e:
                assert e.code == BM.ERR_NO_BLOCKS and snapshot() == before
                failures += 1
                continue
            assert cached % bs == 0 and cached <= len(toks)
            hits += cached > 0
            # the reused prefix already holds these very tokens
            if cached:
                got = [content.get(int(s)) for s in bm.slots(next_id, 0, cached)]
                assert got == toks[:cached]
            for s_, t in zip(bm.slots(next_id, cached, len(toks) - cached), toks[cached:]):
                write(s_, t)
            seqs[next_id], released[next_id] = toks, 0
            next_id += 1
        elif op == "append":
            sid = live[int(rng.integers(0, len(live)))]
            tok = int(rng.integers(0, 5))
            before = snapshot()
            try:
                slot, cow = bm.append_token(sid, tok)
            except BM.BlockManagerError as e:
                assert e.code == BM.ERR_NO_BLOCKS and snapshot() == before
                failures += 1
                continue
            if cow:
                copies += 1
                src, dst = cow
                for r in range(bs):
                    if src * bs + r in content:
                        content[dst * bs + r] = content[src * bs + r]
                    else:
                        content.pop(dst * bs + r, None)
            write(slot, tok)
            seqs[sid] = seqs[sid] + [tok]
        elif op == "batch":
            # one token for several sequences in one call: every copy pair is
            # applied first, then every new token is written
            k = int(rng.integers(1, len(live) + 1))
            sids = [live[i] for i in rng.choice(len(live), size=k, replace=False)]
            toks = [int(t) for t in rng.integers(0, 5, size=k)]
            before = snapshot()
            try:
                slots, pairs = bm.append_tokens(sids, toks)
            except BM.BlockManagerError as e:
                assert e.code == BM.ERR_NO_BLOCKS and snapshot() == before
                failures += 1
                continue
            for src, dst in pairs.tolist():
                copies += 1
                for r in range(bs):
                    if src * bs + r in content:
                        content[dst * bs + r] = content[src * bs + r]
                    else:
                        content.pop(dst * bs + r, None)
            for sid, slot, tok in zip(sids, slots.tolist(), toks):
                write(slot, tok)
                seqs[sid] = seqs[sid] + [tok]
        elif op == "fork":
            parent = live[int(rng.integers(0, len(live)))]
            bm.fork(parent, next_id)
            seqs[next_id], released[next_id] = list(seqs[parent]), released[parent]
            next_id += 1
        elif op == "free":
            sid = live[int(rng.integers(0, len(live)))]
            bm.free_sequence(sid)
            del seqs[sid], released[sid]
        else:
            sid = live[int(rng.integers(0, len(live)))]
            pos = int(rng.integers(0, len(seqs[sid]) + 1))
            bm.release_before(sid, pos)
            released[sid] = max(released[sid], pos)
        _check_contents(bm, seqs, released, content, bs)
        # accounting: every block is free or referenced, never both
        refs = [bm.refcount(b) for b in range(nb)]
        assert bm.num_free_blocks == sum(r == 0 for r in refs)
        held = {}
        for sid, toks in seqs.items():
            t, _ = bm.block_tables([sid], max(1, (len(toks) + bs - 1) // bs))
            for k in range(released[sid] // bs, (len(toks) + bs - 1) // bs):
                held[int(t[0, k])] = held.get(int(t[0, k]), 0) + 1
        for b, n in held.items():
            assert refs[b] - n in (0, 1), (b, refs[b], n)   # plus the cache's own reference
        cache_only = [b for b in range(nb) if refs[b] > 0 and b not in held]
        assert all(refs[b] == 1 for b in cache_only)
        assert bm.num_cached_blocks == len(cache_only)
    return dict(seqs=next_id, hits=hits, copies=copies, failures=failures)


# seeds 190.. once made a batched append fail part-way: a row filling a block
# pinned a released block only the cache held, which the batch had counted
@pytest.mark.parametrize("seed", list(range(8)) + [190, 236, 246, 272, 328])
def test_random_serving_keeps_every_sequence_cache_intact(seed):
    _random_serving(seed)


def test_random_serving_reaches_every_case():
    # across the seeds the loop exercises prefix hits, copy-on-write and a
    # full pool (so the checks above are not vacuous)
    stats = [_random_serving(seed) for seed in range(8)]
    assert sum(s["hits"] for s in stats) > 20
    assert sum(s["copies"] for s in stats) > 20
    assert sum(s["failures"] for s in stats) > 5
    assert all(s["seqs"] > 20 for s in stats)


def test_batched_appends_equal_one_by_one():
    """pa_bm_append_tokens gives the slots and copy pairs that the same
    appends made one call at a time give, including beams that shared a
    partial block (the last beam to append writes in place)."""
    def setup():
        bm = BM.BlockManager(200, 4, prefix_cache=True)
        bm.add_sequence(0, range(10))                # 2 full blocks + 2 tokens
        for c in (1, 2, 3):
            bm.fork(0, c)                            # 4 beams share the partial block
        bm.add_sequence(4, range(100, 108))          # ends on a block boundary
        bm.add_sequence(5, range(100, 103))
        return bm
    one, many = setup(), setup()
    for step in range(9):
        ids = [3, 0, 4, 1, 5, 2] if step % 2 else [0, 1, 2, 3, 4, 5]
        toks = [step * 10 + i for i in ids]
        want_slots, want_pairs = [], []
        for sid, t in zip(ids, toks):
            slot, cow = one.append_token(sid, t)
            want_slots.append(slot)
            if cow:
                want_pairs.append(cow)
        slots, pairs = many.append_tokens(ids, toks)
        assert slots.tolist() == want_slots, step
        assert [tuple(p) for p in pairs.tolist()] == want_pairs, step
        if step == 0:
            assert len(pairs) == 3                   # three beams copy, the fourth writes in place
    t1, l1 = one.block_tables(range(6), 8)
    t2, l2 = many.block_tables(range(6), 8)
    assert (t1 == t2).all() and (l1 == l2).all()
    assert one.num_free_blocks == many.num_free_blocks
    assert one.num_cached_blocks == many.num_cached_blocks


def test_batched_appends_change_nothing_on_error():
    bm = BM.BlockManager(4, 2)
    bm.add_sequence(1, [1, 2])                       # 1 block, full
    bm.add_sequence(2, [3])                          # 1 block, half
    bm.fork(2, 3)                                    # shares the half block
    before = (bm.num_free_blocks, bm.block_tables([1, 2, 3], 3))
    for ids in ([1, 9], [1, 1], [2, 2]):
        with pytest.raises(BM.BlockManagerError) as e:
            bm.append_tokens(ids, [0] * len(ids))
        assert e.value.code == BM.ERR_INVALID
    # 1 needs a new block, 2 copies the shared block, 3 then writes in place: 2 blocks, 2 free
    slots, pairs = bm.append_tokens([1, 2, 3], [7, 8, 9])
    assert len(pairs) == 1 and bm.num_free_blocks == 0
    # now sequences 2 and 3 each need a new block and none is left
    state = (bm.num_free_blocks, bm.block_tables([1, 2, 3], 3))
    with pytest.raises(BM.BlockManagerError) as e:
        bm.append_tokens([1, 2, 3], [0, 0, 0])
    assert e.value.code == BM.ERR_NO_BLOCKS
    after = (bm.num_free_blocks, bm.block_tables([1, 2, 3], 3))
    assert state[0] == after[0] and all((a == b).all() for a, b in zip(state[1], after[1]))
    assert before[0] == 2
    assert bm.append_tokens([], [])[0].shape == (0,)


def test_release_window_equals_release_before_per_sequence():
    a, b = BM.BlockManager(40, 4), BM.BlockManager(40, 4)
    for bm in (a, b):
        bm.add_sequence(1, range(18))                # 5 blocks
        bm.add_sequence(2, range(7))                 # 2 blocks
        bm.fork(1, 3)
    a.release_window([1, 2, 3], 6)
    for sid in (1, 2, 3):
        b.release_before(sid, max(b.length(sid) - 6, 0))
    assert a.num_free_blocks == b.num_free_blocks
    assert [a.refcount(x) for x in range(40)] == [b.refcount(x) for x in range(40)]
    free = a.num_free_blocks
    a.release_window([2], 100)                       # nothing before the window: no change
    assert a.num_free_blocks == free
    with pytest.raises(BM.BlockManagerError):
        a.release_window([1, 9], 6)                  # unknown id: nothing released
    with pytest.raises(BM.BlockManagerError):
        a.release_window([1], 0)
    a.free_sequence(1)
    a.free_sequence(3)                               # released blocks are not dropped twice
    a.free_sequence(2)
    assert a.num_free_blocks == 40


def test_null_arguments_are_rejected_not_dereferenced():
    """Every entry point of the C ABI answers a NULL manager or a NULL array
    (where one is needed) with PA_BM_ERR_INVALID (or -1 / NULL), never a crash."""
    lib = BM._lib()
    bm = BM.BlockManager(8, 4)
    bm.add_sequence(1, [1, 2, 3])
    h = bm._h
    I = BM.ERR_INVALID
    assert lib.pa_bm_create(0, 4, 0) is None and lib.pa_bm_create(8, 0, 0) is None
    assert lib.pa_bm_num_free_blocks(None) == -1 and lib.pa_bm_num_cached_blocks(None) == -1
    assert lib.pa_bm_block_refcount(None, 0) == -1 and lib.pa_bm_block_refcount(h, 8) == -1
    assert lib.pa_bm_add_sequence(None, 2, None, 0, None) == I
    assert lib.pa_bm_add_sequence(h, 2, None, 3, None) == I          # tokens missing
    assert lib.pa_bm_append_token(h, 1, 0, None, None, None) == I    # slot output missing
    n = ctypes.c_int32(0)
    assert lib.pa_bm_append_tokens(h, None, None, 2, None, None, ctypes.byref(n)) == I
    assert lib.pa_bm_append_tokens(h, None, None, 0, None, None, None) == I  # count output missing
    assert lib.pa_bm_release_window(h, None, 1, 4) == I
    assert lib.pa_bm_fork(None, 1, 2) == I and lib.pa_bm_free_sequence(None, 1) == I
    assert lib.pa_bm_release_before(None, 1, 0) == I and lib.pa_bm_sequence_length(None, 1) == I
    assert lib.pa_bm_slots(h, 1, 0, 2, None) == I
    assert lib.pa_bm_block_tables(h, None, 1, 4, None, None) == I
    assert lib.pa_bm_block_tables_update(h, None, 1, 4, None, None, None, None) == I
    lib.pa_bm_destroy(None)                                           # a no-op
    assert bm.length(1) == 3                                          # the manager is intact
