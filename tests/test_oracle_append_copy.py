"""Pins of the oracle's append and copy-on-write block copy.

Append (page 'AI 陪读顶会论文（三）：KV Cache 显存占用计算与 PagedAttention
原理拆解', section '为什么自回归解码必须使用 KV Cache？': each step stores only
the new token's k_t, v_t) writes token t into block slot // BS, row
slot % BS of the [NB, BS, Hkv, D] cache; block copy (KV cache article,
section 'PagedAttention：把操作系统的老智慧搬进推理引擎': copy-on-write at the
fork point) duplicates whole blocks. The pins read the caches back by plain
indexing and check the FP8 codes against torch's float8_e4m3fn conversion."""
import numpy as np
import pytest
import torch


def _bits(rng, shape, dtype="f16"):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32))
    x = x.to(torch.float16 if dtype == "f16" else torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("dtype,bs", [("f16", 16), ("bf16", 1), ("f16", 128)])
def test_append_writes_exactly_the_mapped_slots(oracle_mod, dtype, bs):
    rng = np.random.default_rng(20)
    nb, hkv, d, T = 12, 3, 32, 9
    kc = _bits(rng, (nb, bs, hkv, d), dtype)
    vc = _bits(rng, (nb, bs, hkv, d), dtype)
    k0, v0 = kc.copy(), vc.copy()
    k = _bits(rng, (T, hkv, d), dtype)
    v = _bits(rng, (T, hkv, d), dtype)
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    slots[2] = -1  # padding token: skipped
    oracle_mod.append_kv(k, v, dtype, slots, kc, vc, dtype, bs)
    touched = np.zeros((nb, bs), bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        assert np.array_equal(kc[s // bs, s % bs], k[t])
        assert np.array_equal(vc[s // bs, s % bs], v[t])
        touched[s // bs, s % bs] = True
    assert np.array_equal(kc[~touched], k0[~touched])
    assert np.array_equal(vc[~touched], v0[~touched])


def test_append_fp8_codes_match_torch_conversion(oracle_mod):
    rng = np.random.default_rng(21)
    nb, bs, hkv, d, T = 4, 16, 2, 64, 40
    k = _bits(rng, (T, hkv, d))
    v = _bits(rng, (T, hkv, d))
    kinv = rng.uniform(50, 90, size=(hkv, d)).astype(np.float32)
    vinv = rng.uniform(50, 90, size=(hkv, d)).astype(np.float32)
    kc = np.zeros((nb, bs, hkv, d), np.uint8)
    vc = np.zeros((nb, bs, hkv, d), np.uint8)
    slots = np.arange(T, dtype=np.int64) + 7
    oracle_mod.append_kv(k, v, "f16", slots, kc, vc, "e4m3", bs, kinv, vinv)

    def want(x):
        xf = torch.from_numpy(x.view(np.int16)).view(torch.float16).float()
        y = xf * torch.from_numpy(kinv if x is k else vinv)  # fp32 product, RN
        assert y.abs().max() <= 448  # in range: torch's conversion is then the reference
        return y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    wk, wv = want(k), want(v)
    for t, s in enumerate(slots):
        assert np.array_equal(kc[s // bs, s % bs], wk[t])
        assert np.array_equal(vc[s // bs, s % bs], wv[t])


def test_append_fp8_saturates(oracle_mod):
    k = np.array([[[0x7BFF, 0xFBFF, 0x3C00, 0x7C00]]], np.uint16)  # 65504, -65504, 1, +inf
    kc = np.zeros((1, 1, 1, 4), np.uint8)
    vc = np.zeros((1, 1, 1, 4), np.uint8)
    inv = np.ones((1, 4), np.float32)
    oracle_mod.append_kv(k, k, "f16", np.array([0], np.int64), kc, vc, "e4m3", 1, inv, inv)
    assert kc.ravel().tolist() == [0x7E, 0xFE, 0x38, 0x7E]


def test_append_rejects_out_of_range_slot(oracle_mod):
    kc = np.zeros((2, 4, 1, 8), np.uint16)
    k = np.zeros((1, 1, 8), np.uint16)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.append_kv(k, k, "f16", np.array([8], np.int64), kc, kc.copy(), "f16", 4)


@pytest.mark.parametrize("dtype", ["f16", "e4m3"])
def test_copy_blocks_duplicates_whole_blocks(oracle_mod, dtype):
    rng = np.random.default_rng(22)
    nb, bs, hkv, d = 10, 16, 2, 32
    if dtype == "e4m3":
        kc = rng.integers(0, 256, (nb, bs, hkv, d), dtype=np.uint8)
        vc = rng.integers(0, 256, (nb, bs, hkv, d), dtype=np.uint8)
    else:
        kc = _bits(rng, (nb, bs, hkv, d))
        vc = _bits(rng, (nb, bs, hkv, d))
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[3, 7], [3, 8], [1, 0]], np.int32)
    oracle_mod.copy_blocks(pairs, kc, vc, dtype)
    for s, dst in pairs:
        assert np.array_equal(kc[dst], k0[s]) and np.array_equal(vc[dst], v0[s])
    rest = [b for b in range(nb) if b not in pairs[:, 1]]
    assert np.array_equal(kc[rest], k0[rest]) and np.array_equal(vc[rest], v0[rest])
