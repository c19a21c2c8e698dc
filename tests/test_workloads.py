"""The seeded input generator (paged_kv_cache_410_b200/workloads.py) on the CPU.

Its structure decides what both the kernels and the oracle are fed, so a
mistake here (two sequences writing one slot, a beam reading a block it does
not own, a pool without headroom) would pass every parity test unnoticed.
These tests check the block placement of every family at its full size (the
value draws, which come after all structural draws, are replaced by zeros so
no gigabytes are generated) and the value draws themselves on small cases.
"""
import math

import numpy as np
import pytest

from paged_kv_cache_410_b200 import workloads as W


@pytest.fixture
def no_values(monkeypatch):
    monkeypatch.setattr(W, "normal_bits", lambda rng, shape, dtype, chunk=0:
                        np.zeros(shape, np.uint16))


def used_blocks(w, b):
    L = int(w.context_lens[b])
    return [int(x) for x in w.block_tables[b, :-(-L // w.block_size)]]


def check_common(w):
    """Checks every family must pass."""
    B, BS = w.batch, w.block_size
    assert w.block_tables.dtype == np.int32 and w.block_tables.shape[0] == B
    assert w.context_lens.dtype == np.int32 and w.context_lens.shape == (B,)
    assert w.slot_mapping.dtype == np.int64 and w.slot_mapping.shape == (B,)
    assert w.q.shape == (B, w.num_q_heads, w.head_dim)
    assert w.k_new.shape == w.v_new.shape == (B, w.num_kv_heads, w.head_dim)
    assert w.num_q_heads % w.num_kv_heads == 0
    new_blocks = []
    for b in range(B):
        L = int(w.context_lens[b])
        blocks = used_blocks(w, b)
        assert all(0 <= x < w.num_blocks for x in blocks)
        if w.slot_mapping[b] >= 0:
            # the new token is position L - 1, found through the table
            assert w.slot_mapping[b] == blocks[(L - 1) // BS] * BS + (L - 1) % BS
            new_blocks.append((b, blocks[(L - 1) // BS]))
    live = w.slot_mapping[w.slot_mapping >= 0]
    assert len(set(live.tolist())) == len(live)          # no slot written twice
    # the block a sequence writes into belongs to that sequence alone
    users = {}
    for o in range(B):
        for x in set(used_blocks(w, o)):
            users[x] = users.get(x, 0) + 1
    for b, blk in new_blocks:
        assert users[blk] == 1, (b, blk)


def assert_private(w, skip=0):
    """Blocks past the first `skip` of each table are used by one sequence only."""
    seen = {}
    for b in range(w.batch):
        for x in used_blocks(w, b)[skip:]:
            assert seen.setdefault(x, b) == b, (x, seen[x], b)
    return seen


def test_tiny_mha(no_values):
    w = W.tiny_mha()
    check_common(w)
    assert (w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.num_blocks) == (4, 8, 8, 64, 64)
    hist = np.asarray(w.meta["history"])
    assert ((1 <= hist) & (hist <= 200)).all()
    assert (w.context_lens == hist + 1).all()                # one token appended
    assert_private(w)


def test_llama2_7b(no_values):
    w = W.llama2_7b()
    check_common(w)
    assert (w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim) == (64, 32, 32, 128)
    assert w.cache_dtype == "f16" and w.block_size == 16
    assert ((512 <= w.context_lens) & (w.context_lens <= 4096)).all()
    seen = assert_private(w)
    assert w.num_blocks == math.ceil(1.1 * len(seen))        # pool = blocks needed + 10%
    assert w.scale == np.float32(1 / math.sqrt(128))


def test_llama2_70b_prefix(no_values):
    w = W.llama2_70b_prefix()
    check_common(w)
    assert (w.batch, w.num_q_heads, w.num_kv_heads, w.cache_dtype) == (128, 64, 8, "bf16")
    npre = w.meta["shared_prefix_blocks"]
    assert npre == 125 and w.meta["prefix_len"] == 2000
    assert (w.block_tables[:, :npre] == w.block_tables[0, :npre]).all()  # one stored prefix
    suffix = w.context_lens - 2001
    assert ((0 <= suffix) & (suffix <= 2048)).all()
    seen = assert_private(w, skip=npre)
    assert not set(seen) & set(w.block_tables[0, :npre].tolist())
    assert w.num_blocks == math.ceil(1.1 * (npre + len(seen)))


@pytest.mark.parametrize("batch", [1, 4])
def test_long_context(no_values, batch):
    w = W.long_context(batch=batch)
    check_common(w)
    assert (w.context_lens == 131072).all() and w.block_tables.shape[1] == 8192
    seen = assert_private(w)
    assert w.num_blocks == math.ceil(1.1 * len(seen))
    # scattered: consecutive logical blocks are rarely neighbours in the pool
    steps = np.diff(w.block_tables[0].astype(np.int64))
    assert np.mean(np.abs(steps) == 1) < 0.01


@pytest.mark.parametrize("bs", [16, 32, 128])
def test_fp8_beams_structure(no_values, bs):
    w = W.fp8_beams(block_size=bs)
    check_common(w)
    assert (w.batch, w.num_q_heads, w.num_kv_heads, w.cache_dtype) == (256, 32, 8, "e4m3")
    assert ((16 <= w.context_lens) & (w.context_lens <= 8192)).all()
    G, Wd = w.meta["beam_groups"], w.meta["beam_width"]
    pairs = [tuple(p) for p in w.copy_pairs.tolist()]
    srcs, dsts = {p[0] for p in pairs}, [p[1] for p in pairs]
    assert len(set(dsts)) == len(dsts) and not srcs & set(dsts)
    expected_pairs = 0
    for g in range(G):
        beams = list(range(g * Wd, (g + 1) * Wd))
        L = int(w.context_lens[beams[0]])
        assert all(int(w.context_lens[b]) == L for b in beams)
        full = (L - 1) // bs
        tabs = [used_blocks(w, b) for b in beams]
        assert all(t[:full] == tabs[0][:full] for t in tabs)  # the prompt's full blocks shared
        lasts = [t[full] for t in tabs]
        assert len(set(lasts)) == Wd                          # each beam writes its own block
        if (L - 1) % bs:
            expected_pairs += Wd - 1
            assert [(lasts[0], d) for d in lasts[1:]] == [p for p in pairs if p[0] == lasts[0]]
        else:
            assert lasts[0] not in srcs
    assert len(pairs) == expected_pairs <= 3 * G
    # pool: shared prompt blocks once, one last block per beam, solo blocks; + 10%
    distinct = {x for b in range(w.batch) for x in used_blocks(w, b)}
    assert w.num_blocks == math.ceil(1.1 * len(distinct))
    users = {}
    for o in range(w.batch):
        for x in set(used_blocks(w, o)):
            users[x] = users.get(x, 0) + 1
    for b in range(G * Wd, w.batch):                          # solo sequences: private
        assert all(users[x] == 1 for x in used_blocks(w, b))


def test_fp8_beams_history_reads_back_after_the_copies():
    """Each history token is written once; after the copy pairs are applied,
    every sequence reads its own history (and the parent's prompt, for
    beams) through its own table, and no history slot is a new-token slot."""
    w = W.fp8_beams(batch=40, beam_groups=4, beam_width=4, median_len=40, max_len=300,
                    block_size=16)
    check_common(w)
    bs = w.block_size
    fill = {int(s): i for i, s in enumerate(w.fill_slots.tolist())}
    assert len(fill) == len(w.fill_slots)                     # each slot once
    assert not set(fill) & set(w.slot_mapping.tolist())
    moved = {}
    for src, dst in w.copy_pairs.tolist():
        for r in range(bs):
            if src * bs + r in fill:
                moved[dst * bs + r] = fill[src * bs + r]
    view = {**fill, **moved}
    for g in range(4):
        beams = range(g * 4, g * 4 + 4)
        L = int(w.context_lens[g * 4])
        rows = [[view.get(int(w.block_tables[b, j // bs]) * bs + j % bs) for j in range(L - 1)]
                for b in beams]
        assert None not in rows[0] and all(r == rows[0] for r in rows)  # same prompt values
    for b in range(16, w.batch):
        L = int(w.context_lens[b])
        got = [view.get(int(w.block_tables[b, j // bs]) * bs + j % bs) for j in range(L - 1)]
        assert None not in got
    assert len(view) == sum(int(w.context_lens[b]) - 1 for b in range(16, w.batch)) + \
        sum(int(w.context_lens[g * 4]) - 1 for g in range(4)) + \
        sum(((int(w.context_lens[g * 4]) - 1) % bs) * 3 for g in range(4))


def test_fp8_scales_are_max_abs_over_what_the_cache_holds():
    w = W.fp8_beams(batch=24, beam_groups=2, median_len=40, max_len=200)
    fk = np.abs(W.bits_to_float32(w.fill_k, "f16"))
    nk = np.abs(W.bits_to_float32(w.k_new, "f16"))
    m = np.maximum(fk.max(axis=0), nk.max(axis=0))
    assert w.k_scale.shape == (w.num_kv_heads, w.head_dim) and w.k_scale.dtype == np.float32
    assert np.array_equal(w.k_scale, np.where(m == 0, 1, m / np.float32(448)).astype(np.float32))
    assert np.array_equal(w.k_inv_scale, (np.float32(1) / w.k_scale).astype(np.float32))


def test_custom_families_and_empty_sequences():
    w = W.custom([0, 1, 16, 17, 300], num_q_heads=8, num_kv_heads=2, head_dim=128)
    check_common(w)
    assert w.slot_mapping[0] == -1                           # nothing to append
    assert_private(w)
    p = W.custom_shared_prefix(64, [0, 1, 30], num_q_heads=8, num_kv_heads=2)
    check_common(p)
    assert p.slot_mapping[0] == -1 and int(p.context_lens[0]) == 64
    assert (p.block_tables[:, :4] == p.block_tables[0, :4]).all()
    assert_private(p, skip=4)
    with pytest.raises(ValueError):
        W.custom_shared_prefix(60, [1, 2])                    # must end on a block boundary


def test_subset_keeps_the_pool_and_the_pairs_it_needs():
    w = W.fp8_beams(batch=40, beam_groups=4, median_len=40, max_len=300)
    s = W.subset(w, [1, 2, 30])
    assert s.batch == 3 and s.num_blocks == w.num_blocks
    assert np.array_equal(s.block_tables, w.block_tables[[1, 2, 30]])
    lasts = {int(w.block_tables[b, (int(w.context_lens[b]) - 1) // w.block_size])
             for b in (1, 2, 30)}
    assert {d for _, d in s.copy_pairs.tolist()} == \
        {d for _, d in w.copy_pairs.tolist() if d in lasts}


def test_values_are_seeded_rounded_normals():
    rng1, rng2 = np.random.default_rng(5), np.random.default_rng(5)
    a = W.normal_bits(rng1, (300, 1000), "f16", chunk=7000)   # 43 chunks, filled by threads
    b = W.normal_bits(rng2, (300, 1000), "f16", chunk=7000)
    assert np.array_equal(a, b)
    x = W.bits_to_float32(a, "f16").astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    # each value is the float32 draw rounded to nearest even in the storage type
    base = int(np.random.default_rng(5).integers(0, 2 ** 63 - 1))
    first = np.random.default_rng([base, 0]).standard_normal(7000, dtype=np.float32)
    assert np.array_equal(a.reshape(-1)[:7000], first.astype(np.float16).view(np.uint16))
    bf = W.normal_bits(np.random.default_rng(5), (64,), "bf16")
    xb = W.bits_to_float32(bf, "bf16")
    assert np.array_equal(W.round_bits(xb, "bf16"), bf)      # exact round trip
    assert W.bits_to_float32(np.array([0x3F80], np.uint16), "bf16")[0] == 1.0


def test_default_seeds_follow_the_documented_rule(no_values):
    assert np.array_equal(W.tiny_mha().block_tables, W.tiny_mha(seed=411).block_tables)
    assert np.array_equal(W.fp8_beams(block_size=32).context_lens,
                          W.fp8_beams(block_size=32, seed=410 + 5 + 32).context_lens)
