"""Pins of the oracle's decode attention.

The method (page 'AI 陪读顶会论文（三）：KV Cache 显存占用计算与 PagedAttention
原理拆解', section '为什么自回归解码必须使用 KV Cache？', attention equation)
computes softmax(q K^T / sqrt(d)) V for one query token over all cached
tokens; the KV cache article's PagedAttention section stores those tokens in
fixed-size blocks found through a block table, shares prefix blocks, and
groups query heads onto shared KV heads (GQA, section '显存账本').

The oracle is pinned here against: torch's scaled_dot_product_attention
(an independent library routine, float64, with its own GQA grouping) on
contiguous K/V that the test lays out itself; closed forms; invariances that
the pages state (physical placement and block size do not matter, a shared
prefix equals private copies, GQA equals MHA with replicated KV heads); and
the block-table diagram of the PagedAttention section."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f16_bits(x):
    return np.asarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def _bits_f64(bits, dtype):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16).double()


def _round(x, dtype):
    t = torch.from_numpy(np.asarray(x, dtype=np.float32))
    t = t.to(torch.float16 if dtype == "f16" else torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def scatter(logical, bs, nb, rng, hkv, d, dtype="f16", garbage=50.0, perm=None,
            shared_prefix_blocks=0):
    """Lay out per-sequence logical K (list of [L, Hkv, D] bit arrays) in a
    paged pool [nb, bs, Hkv, D] following the cache layout; unused slots hold
    large garbage so that any stray read shows up. Returns pool, tables."""
    pool = _round(rng.normal(0, garbage, size=(nb, bs, hkv, d)), dtype)
    perm = rng.permutation(nb) if perm is None else np.asarray(perm)
    nxt = 0
    tables = []
    prefix = []
    for b, kv in enumerate(logical):
        L = kv.shape[0]
        nblk = -(-L // bs)
        blocks = []
        for n in range(nblk):
            if n < shared_prefix_blocks and b > 0:
                blocks.append(prefix[n])
                continue
            blocks.append(int(perm[nxt]))
            nxt += 1
            if n < shared_prefix_blocks:
                prefix.append(blocks[-1])
        for j in range(L):
            pool[blocks[j // bs], j % bs] = kv[j]
        tables.append(blocks)
    mb = max(len(t) for t in tables)
    tab = np.zeros((len(tables), mb + 2), dtype=np.int32)  # extra columns stay unused
    for b, t in enumerate(tables):
        tab[b, :len(t)] = t
    return pool, tab


def sdpa_ref(q_bits, ks, vs, scale, dtype, kscale=None, vscale=None):
    """torch SDPA (float64, enable_gqa) per sequence on contiguous K/V."""
    out = []
    for b in range(q_bits.shape[0]):
        q = _bits_f64(q_bits[b], dtype)[None, :, None, :]          # [1, Hq, 1, D]
        k = ks[b] if isinstance(ks[b], torch.Tensor) else _bits_f64(ks[b], dtype)
        v = vs[b] if isinstance(vs[b], torch.Tensor) else _bits_f64(vs[b], dtype)
        if kscale is not None:
            k = k * kscale
            v = v * vscale
        k = k.permute(1, 0, 2)[None]                               # [1, Hkv, L, D]
        v = v.permute(1, 0, 2)[None]
        o = F.scaled_dot_product_attention(q, k, v, scale=float(scale), enable_gqa=True)
        out.append(o[0, :, 0, :].numpy())
    return np.stack(out)


def _case(rng, B, hq, hkv, d, bs, lens, dtype):
    ks = [_round(rng.standard_normal((L, hkv, d)), dtype) for L in lens]
    vs = [_round(rng.standard_normal((L, hkv, d)), dtype) for L in lens]
    nb = sum(-(-L // bs) for L in lens) + 7
    perm = rng.permutation(nb)
    kpool, tab = scatter(ks, bs, nb, rng, hkv, d, dtype, perm=perm)
    vpool, tab2 = scatter(vs, bs, nb, rng, hkv, d, dtype, perm=perm)
    assert np.array_equal(tab, tab2)
    q = _round(rng.standard_normal((B, hq, d)), dtype)
    return q, ks, vs, kpool, vpool, tab


@pytest.mark.parametrize("hq,hkv,d,bs,dtype", [
    (8, 8, 64, 16, "f16"), (8, 2, 64, 16, "f16"), (8, 1, 32, 4, "bf16"),
    (16, 4, 128, 32, "bf16"), (6, 3, 16, 1, "f16"), (4, 4, 64, 128, "f16"),
])
def test_matches_torch_sdpa(oracle_mod, hq, hkv, d, bs, dtype):
    rng = np.random.default_rng(hq * 1000 + hkv * 100 + d + bs)
    lens = [1, bs, bs + 1, 3 * bs - 1, 37, 130]
    q, ks, vs, kpool, vpool, tab = _case(rng, len(lens), hq, hkv, d, bs, lens, dtype)
    scale = np.float32(0.37)  # not 1/sqrt(d): a dropped or misplaced scale shows up
    got = oracle_mod.decode(q, dtype, kpool, vpool, dtype, tab, np.array(lens, np.int32), scale)
    want = sdpa_ref(q, ks, vs, scale, dtype)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_single_token_returns_its_value_exactly(oracle_mod):
    rng = np.random.default_rng(1)
    q, ks, vs, kpool, vpool, tab = _case(rng, 3, 4, 2, 64, 16, [1, 1, 1], "f16")
    got = oracle_mod.decode(q, "f16", kpool, vpool, "f16", tab, np.ones(3, np.int32), 0.125)
    for b in range(3):
        v = vs[b][0].view(np.float16).astype(np.float64)  # [Hkv, D]
        assert np.array_equal(got[b], np.repeat(v, 2, axis=0))


def test_zero_query_and_equal_keys_give_the_mean_value(oracle_mod):
    rng = np.random.default_rng(2)
    L, hkv, d = 53, 2, 64
    ks = [_f16_bits(rng.standard_normal((L, hkv, d)))]
    vs = [_f16_bits(rng.standard_normal((L, hkv, d)))]
    kpool, tab = scatter(ks, 16, 8, rng, hkv, d, perm=np.arange(8))
    vpool, _ = scatter(vs, 16, 8, rng, hkv, d, perm=np.arange(8))
    mean = vs[0].view(np.float16).astype(np.float64).mean(axis=0)  # [Hkv, D]
    q0 = np.zeros((1, 4, d), np.uint16)  # +0.0 bits
    got = oracle_mod.decode(q0, "f16", kpool, vpool, "f16", tab, np.array([L], np.int32), 1.0)
    np.testing.assert_allclose(got[0], np.repeat(mean, 2, axis=0), rtol=0, atol=1e-14)
    # all keys equal: every score is the same, whatever q is
    keq = [np.broadcast_to(ks[0][:1], ks[0].shape).copy()]
    kpool2, _ = scatter(keq, 16, 8, rng, hkv, d, perm=np.arange(8))
    q = _f16_bits(rng.standard_normal((1, 4, d)))
    got = oracle_mod.decode(q, "f16", kpool2, vpool, "f16", tab, np.array([L], np.int32), 1.0)
    np.testing.assert_allclose(got[0], np.repeat(mean, 2, axis=0), rtol=0, atol=1e-13)


def test_two_keys_closed_form(oracle_mod):
    d = 16
    k = np.zeros((2, 1, d), np.float32)
    k[0, 0, 0] = 1.0
    k[1, 0, 0] = 3.0
    v = np.zeros((2, 1, d), np.float32)
    v[0, 0, :] = 2.0
    v[1, 0, :] = -1.0
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, 0] = 0.5
    scale = np.float32(0.75)
    rng = np.random.default_rng(3)
    kpool, tab = scatter([_f16_bits(k)], 16, 4, rng, 1, d, perm=np.arange(4))
    vpool, _ = scatter([_f16_bits(v)], 16, 4, rng, 1, d, perm=np.arange(4))
    got = oracle_mod.decode(_f16_bits(q), "f16", kpool, vpool, "f16", tab,
                            np.array([2], np.int32), scale)
    s0, s1 = float(scale) * 0.5 * 1.0, float(scale) * 0.5 * 3.0
    p1 = 1.0 / (1.0 + math.exp(s0 - s1))
    want = 2.0 * (1 - p1) + (-1.0) * p1
    np.testing.assert_allclose(got[0, 0], np.full(d, want), rtol=0, atol=1e-15)


def test_block_table_diagram_fixture(oracle_mod):
    """Logical blocks 0, 1, 2 live in physical blocks 42, 105, 12: a key that
    dominates the softmax at logical token j must return token j's value."""
    fx = json.load(open(os.path.join(GOLDEN, "block_table_diagram.json")))
    bs, n, phys = fx["block_size"], fx["num_tokens"], fx["logical_to_physical"]
    d, nb = 16, 128
    rng = np.random.default_rng(4)
    kpool = _f16_bits(rng.normal(0, 1, size=(nb, bs, 1, d)))
    vpool = _f16_bits(rng.normal(0, 1, size=(nb, bs, 1, d)))
    # keys of the 48 tokens are 0 except channel 0 of the probed token;
    # channel 0 of each value holds its logical index
    for j in range(n):
        blk, r = phys[j // bs], j % bs
        kpool[blk, r, 0, :] = _f16_bits(np.zeros(d))
        vpool[blk, r, 0, 0] = _f16_bits(np.array([float(j)]))[0]
    tab = np.array([phys], dtype=np.int32)
    q = _f16_bits(np.r_[1000.0, np.zeros(d - 1)].reshape(1, 1, d))
    for j in [0, 15, 16, 31, 32, 47]:
        blk, r = phys[j // bs], j % bs
        kp = kpool.copy()
        kp[blk, r, 0, 0] = _f16_bits(np.array([1.0]))[0]
        got = oracle_mod.decode(q, "f16", kp, vpool, "f16", tab, np.array([n], np.int32), 1.0)
        assert got[0, 0, 0] == float(j)


def test_physical_placement_and_block_size_do_not_matter(oracle_mod):
    rng = np.random.default_rng(5)
    hq, hkv, d = 8, 4, 64
    lens = [5, 77, 160, 33]
    ks = [_round(rng.standard_normal((L, hkv, d)), "bf16") for L in lens]
    vs = [_round(rng.standard_normal((L, hkv, d)), "bf16") for L in lens]
    q = _round(rng.standard_normal((len(lens), hq, d)), "bf16")
    L = np.array(lens, np.int32)
    outs = []
    for bs, seed in [(16, 10), (16, 11), (1, 12), (32, 13)]:
        r = np.random.default_rng(seed)
        nb = sum(-(-x // bs) for x in lens) + 3
        perm = r.permutation(nb)
        kp, tab = scatter(ks, bs, nb, r, hkv, d, "bf16", perm=perm)
        vp, _ = scatter(vs, bs, nb, r, hkv, d, "bf16", perm=perm)
        outs.append(oracle_mod.decode(q, "bf16", kp, vp, "bf16", tab, L, 0.125))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_shared_prefix_equals_private_copies(oracle_mod):
    rng = np.random.default_rng(6)
    hq, hkv, d, bs = 8, 2, 64, 16
    prefix_k = _f16_bits(rng.standard_normal((48, hkv, d)))
    prefix_v = _f16_bits(rng.standard_normal((48, hkv, d)))
    suf = [3, 0, 21, 16]
    ks = [np.concatenate([prefix_k, _f16_bits(rng.standard_normal((s, hkv, d)))]) for s in suf]
    vs = [np.concatenate([prefix_v, _f16_bits(rng.standard_normal((s, hkv, d)))]) for s in suf]
    q = _f16_bits(rng.standard_normal((len(suf), hq, d)))
    L = np.array([48 + s for s in suf], np.int32)
    nb = 40
    perm = rng.permutation(nb)
    kp_s, tab_s = scatter(ks, bs, nb, rng, hkv, d, perm=perm, shared_prefix_blocks=3)
    vp_s, _ = scatter(vs, bs, nb, rng, hkv, d, perm=perm, shared_prefix_blocks=3)
    assert all(tab_s[b, :3].tolist() == tab_s[0, :3].tolist() for b in range(len(suf)))
    kp_p, tab_p = scatter(ks, bs, nb, rng, hkv, d, perm=perm)
    vp_p, _ = scatter(vs, bs, nb, rng, hkv, d, perm=perm)
    shared = oracle_mod.decode(q, "f16", kp_s, vp_s, "f16", tab_s, L, 0.125)
    private = oracle_mod.decode(q, "f16", kp_p, vp_p, "f16", tab_p, L, 0.125)
    assert np.array_equal(shared, private)


def test_gqa_equals_mha_with_replicated_kv_heads(oracle_mod):
    rng = np.random.default_rng(7)
    hq, hkv, d, bs = 16, 2, 32, 16
    g = hq // hkv
    lens = [9, 40]
    ks = [_f16_bits(rng.standard_normal((L, hkv, d))) for L in lens]
    vs = [_f16_bits(rng.standard_normal((L, hkv, d))) for L in lens]
    q = _f16_bits(rng.standard_normal((2, hq, d)))
    L = np.array(lens, np.int32)
    perm = rng.permutation(8)
    kp, tab = scatter(ks, bs, 8, rng, hkv, d, perm=perm)
    vp, _ = scatter(vs, bs, 8, rng, hkv, d, perm=perm)
    gqa = oracle_mod.decode(q, "f16", kp, vp, "f16", tab, L, 0.2)
    krep = [np.repeat(k, g, axis=1) for k in ks]  # KV head h serves q heads h*g .. h*g+g-1
    vrep = [np.repeat(v, g, axis=1) for v in vs]
    kp2, tab2 = scatter(krep, bs, 8, rng, hq, d, perm=perm)
    vp2, _ = scatter(vrep, bs, 8, rng, hq, d, perm=perm)
    mha = oracle_mod.decode(q, "f16", kp2, vp2, "f16", tab2, L, 0.2)
    assert np.array_equal(gqa, mha)


def test_fp8_cache_matches_sdpa_on_dequantised_values(oracle_mod):
    rng = np.random.default_rng(8)
    hq, hkv, d, bs = 8, 2, 64, 16
    lens = [1, 17, 90]
    kscale = rng.uniform(0.002, 0.02, size=(hkv, d)).astype(np.float32)
    vscale = rng.uniform(0.002, 0.02, size=(hkv, d)).astype(np.float32)

    def codes(L, s):
        x = torch.from_numpy((rng.standard_normal((L, hkv, d)) / s).astype(np.float32))
        return x.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    kc = [codes(L, kscale) for L in lens]
    vc = [codes(L, vscale) for L in lens]
    nb = 12
    perm = rng.permutation(nb)
    # lay out the byte codes (garbage codes in unused slots)
    kp =rng.integers(0, 0x7E, size=(nb, bs, hkv, d), dtype=np.uint8)
    vp = rng.integers(0, 0x7E, size=(nb, bs, hkv, d), dtype=np.uint8)
    tab = np.zeros((len(lens), 8), np.int32)
    nxt = 0
    for b, L in enumerate(lens):
        for n in range(-(-L // bs)):
            tab[b, n] = perm[nxt]
            nxt += 1
        for j in range(L):
            kp[tab[b, j // bs], j % bs] = kc[b][j]
            vp[tab[b, j // bs], j % bs] = vc[b][j]
    q = _f16_bits(rng.standard_normal((len(lens), hq, d)))
    got = oracle_mod.decode(q, "f16", kp, vp, "e4m3", tab, np.array(lens, np.int32), 0.125,
                            k_scale=kscale, v_scale=vscale)
    deq = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).double()
    want = sdpa_ref(q, [deq(c) for c in kc], [deq(c) for c in vc], 0.125, "f16",
                    kscale=torch.from_numpy(kscale).double(),
                    vscale=torch.from_numpy(vscale).double())
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_empty_context_gives_zeros_and_bad_block_ids_are_rejected(oracle_mod):
    rng = np.random.default_rng(9)
    q, ks, vs, kp, vp, tab = _case(rng, 2, 4, 4, 32, 16, [5, 20], "f16")
    got = oracle_mod.decode(q, "f16", kp, vp, "f16", tab, np.array([0, 20], np.int32), 0.5)
    assert np.all(got[0] == 0.0)
    bad = tab.copy()
    bad[1, 1] = kp.shape[0]
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.decode(q, "f16", kp, vp, "f16", bad, np.array([5, 20], np.int32), 0.5)


# ---- sliding window (KV cache article, section '再往后：压 KV 的三条路线':
# each token attends only to the most recent window of tokens) ------------------

def test_window_at_least_the_length_changes_nothing(oracle_mod):
    rng = np.random.default_rng(30)
    lens = [1, 16, 37, 100]
    q, ks, vs, kp, vp, tab = _case(rng, 4, 8, 2, 64, 16, lens, "f16")
    L = np.array(lens, np.int32)
    full = oracle_mod.decode(q, "f16", kp, vp, "f16", tab, L, 0.125)
    for w in (100, 101, 5000):
        assert np.array_equal(oracle_mod.decode(q, "f16", kp, vp, "f16", tab, L, 0.125,
                                                window=w), full)


def test_window_of_one_returns_the_newest_value(oracle_mod):
    rng = np.random.default_rng(31)
    lens = [1, 9, 40]
    q, ks, vs, kp, vp, tab = _case(rng, 3, 4, 4, 32, 16, lens, "f16")
    got = oracle_mod.decode(q, "f16", kp, vp, "f16", tab, np.array(lens, np.int32), 0.3,
                            window=1)
    for b, L in enumerate(lens):
        assert np.array_equal(got[b], vs[b][L - 1].view(np.float16).astype(np.float64))


@pytest.mark.parametrize("window", [2, 15, 16, 17, 33])
def test_window_equals_attention_over_the_last_tokens(oracle_mod, window):
    rng = np.random.default_rng(32 + window)
    hq, hkv, d, bs = 8, 2, 64, 16
    lens = [3, 16, 50, 129]
    q, ks, vs, kp, vp, tab = _case(rng, len(lens), hq, hkv, d, bs, lens, "bf16")
    scale = np.float32(0.2)
    got = oracle_mod.decode(q, "bf16", kp, vp, "bf16", tab, np.array(lens, np.int32), scale,
                            window=window)
    # the same tokens laid out afresh as whole sequences of their own
    ks_t = [k[max(0, L - window):] for k, L in zip(ks, lens)]
    vs_t = [v[max(0, L - window):] for v, L in zip(vs, lens)]
    nb = sum(-(-len(k) // bs) for k in ks_t) + 3
    perm = rng.permutation(nb)
    kp2, tab2 = scatter(ks_t, bs, nb, rng, hkv, d, "bf16", perm=perm)
    vp2, _ = scatter(vs_t, bs, nb, rng, hkv, d, "bf16", perm=perm)
    short = oracle_mod.decode(q, "bf16", kp2, vp2, "bf16", tab2,
                              np.array([len(k) for k in ks_t], np.int32), scale)
    assert np.array_equal(got, short)
    np.testing.assert_allclose(got, sdpa_ref(q, ks_t, vs_t, scale, "bf16"), rtol=0, atol=1e-12)
