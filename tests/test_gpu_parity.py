"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle,
at sizes the oracle finishes in seconds. Append and block copy are compared
bit for bit over the whole caches; decode outputs within the tolerances of
tests/helpers.py."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep, to_bits

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


def run_and_compare(w, partition_tokens=0, check_caches=True):
    step = DecodeStep(w, "cuda", partition_tokens=partition_tokens)
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    kc, vc, want = oracle_step(w)
    if check_caches:
        assert np.array_equal(to_bits(step.k_cache), kc), "K cache differs from the oracle"
        assert np.array_equal(to_bits(step.v_cache), vc), "V cache differs from the oracle"
    got = step.out_f64()
    err = max_abs_err(got, want)
    assert err <= TOL[w.io_dtype], f"{w.name}: max abs err {err}"
    return step, got, want


REDUCED = [
    ("tiny_mha", {}),
    ("llama2_7b", {"batch": 3}),
    ("llama2_70b_prefix", {"batch": 6}),
    ("long_context", {"batch": 1, "context_len": 20000}),
    ("fp8_beams", {"batch": 24, "beam_groups": 2, "block_size": 16}),
    ("fp8_beams", {"batch": 24, "beam_groups": 2, "block_size": 32}),
    ("fp8_beams", {"batch": 24, "beam_groups": 2, "block_size": 128}),
]


@pytest.mark.parametrize("name,kw", REDUCED, ids=[f"{n}-{k}" for n, k in REDUCED])
def test_step_matches_oracle(name, kw):
    run_and_compare(W.make(name, **kw))


@pytest.mark.parametrize("pt", [16, 48, 256, 4096, 1 << 20, 0])
def test_split_k_partition_count_does_not_change_the_result(pt):
    w = W.llama2_70b_prefix(batch=4, max_suffix=700)
    run_and_compare(w, partition_tokens=pt, check_caches=False)


@pytest.mark.parametrize("bs", [1, 2, 4, 8, 32, 64, 128, 256])
def test_block_sizes(bs):
    w = W.custom([1, 15, 16, 17, 100, 333], num_q_heads=8, num_kv_heads=2, head_dim=128,
                 block_size=bs, seed=bs)
    run_and_compare(w)


@pytest.mark.parametrize("hq,hkv,d,dtype", [
    (32, 1, 128, "f16"),   # MQA: 32 query heads on one KV head (two head groups)
    (6, 2, 64, "bf16"),    # group of 3
    (40, 8, 64, "f16"),    # group of 5
    (16, 1, 64, "bf16"),   # group of 16: both MMA row halves
    (24, 1, 128, "bf16"),  # group of 24: a full and a partial head group
    (4, 4, 128, "bf16"),
])
def test_head_groupings(hq, hkv, d, dtype):
    w = W.custom([3, 64, 250, 1000], num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                 dtype=dtype, seed=hq + hkv + d)
    run_and_compare(w)


def test_zero_length_and_single_token_sequences():
    w = W.custom([0, 1, 2, 0, 17], num_q_heads=8, num_kv_heads=4, head_dim=64)
    step, got, _ = run_and_compare(w)
    assert np.all(got[0] == 0) and np.all(got[3] == 0)


def test_single_token_returns_its_value():
    w = W.custom([1, 1], num_q_heads=4, num_kv_heads=2, head_dim=128)
    step, got, _ = run_and_compare(w)
    v = w.v_new.view(np.float16).astype(np.float64)  # the appended token is the only one
    assert np.array_equal(got, np.repeat(v, 2, axis=1))


def test_empty_calls_are_no_ops():
    w = W.custom([5], head_dim=64)
    step = DecodeStep(w, "cuda")
    before = to_bits(step.k_cache).copy()
    B.pa_copy_blocks(np.zeros((0, 2), np.int32), step.k_cache, step.v_cache, step.cache)
    B.pa_append_kv(step.k_new[:0], step.v_new[:0], step.slot_mapping[:0], step.k_cache,
                   step.v_cache, step.cache)
    B.pa_decode(step.q[:0], step.k_cache, step.v_cache, step.block_tables[:0],
                step.context_lens[:0], 0.1, step.out[:0], step.cache, 0)
    torch.cuda.synchronize()
    assert np.array_equal(to_bits(step.k_cache), before)
    assert step.device_errors() == 0


def test_copy_blocks_many_pairs_bit_exact():
    # more pairs than one launch carries
    w = W.custom([16] * 700, num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
                 headroom=1.0)
    step = DecodeStep(w, "cuda")
    rng = np.random.default_rng(0)
    ids = rng.permutation(w.num_blocks)
    pairs = np.stack([ids[:600], ids[600:1200]], axis=1).astype(np.int32)
    B.pa_copy_blocks(pairs, step.k_cache, step.v_cache, step.cache)
    torch.cuda.synchronize()
    k, v = w.k_pool.copy(), w.v_pool.copy()
    import oracle
    oracle.copy_blocks(pairs, k, v, "f16")
    assert np.array_equal(to_bits(step.k_cache), k)
    assert np.array_equal(to_bits(step.v_cache), v)


@pytest.mark.parametrize("in_dtype", ["f16", "bf16"])
def test_fp8_quantiser_every_input_pattern(in_dtype):
    """Every 16-bit input pattern through the E4M3 append, against the
    oracle's encoder, for several per-channel inverse scales."""
    import oracle
    T, hkv, d = 64, 8, 128
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(T, hkv, d)
    rng = np.random.default_rng(1)
    for inv in [np.ones((hkv, d), np.float32),
                rng.uniform(0.01, 300.0, size=(hkv, d)).astype(np.float32),
                np.full((hkv, d), 1.0 / 0.0123, np.float32)]:
        kc = np.zeros((T, 1, hkv, d), np.uint8)
        vc = np.zeros((T, 1, hkv, d), np.uint8)
        slots = np.arange(T, dtype=np.int64)
        vbits = allbits[::-1].copy()
        oracle.append_kv(allbits, vbits, in_dtype, slots, kc, vc, "e4m3", 1, inv, inv)
        dev = "cuda"
        tdt = torch.float16 if in_dtype == "f16" else torch.bfloat16
        k = torch.from_numpy(allbits.view(np.int16)).to(dev).view(tdt)
        v = torch.from_numpy(vbits.view(np.int16)).to(dev).view(tdt)
        gk = torch.zeros((T, 1, hkv, d), dtype=torch.uint8, device=dev)
        gv = torch.zeros_like(gk)
        ti = torch.from_numpy(inv).to(dev)
        cache = B.PagedCache(T, 1, hkv, d, torch.uint8, ti, ti, ti, ti)
        B.pa_append_kv(k, v, torch.from_numpy(slots).to(dev), gk, gv, cache)
        got_k, got_v = gk.cpu().numpy(), gv.cpu().numpy()
        # NaN inputs must give a NaN code; every other input the oracle's code
        for got, src, want in ((got_k, allbits, kc), (got_v, vbits, vc)):
            x = torch.from_numpy(src.view(np.int16)).view(tdt).float().numpy().reshape(got.shape)
            nan = np.isnan(x)
            assert np.all((got[nan] & 0x7F) == 0x7F)
            assert np.array_equal(got[~nan], want[~nan])


def test_device_bounds_are_reported_not_faulted():
    w = W.custom([40, 40], num_q_heads=4, num_kv_heads=4, head_dim=64)
    step = DecodeStep(w, "cuda")
    assert step.device_errors() == 0
    bad_tables = step.block_tables.clone()
    bad_tables[1, 1] = w.num_blocks + 5
    B.pa_decode(step.q, step.k_cache, step.v_cache, bad_tables, step.context_lens, 0.1,
                step.out, step.cache, step.max_context)
    assert step.device_errors() & B.DEVERR_BLOCK_ID
    bad_lens = step.context_lens.clone()
    bad_lens[0] = step.max_context + 1
    B.pa_decode(step.q, step.k_cache, step.v_cache, step.block_tables, bad_lens, 0.1,
                step.out, step.cache, step.max_context)
    assert step.device_errors() & B.DEVERR_CONTEXT_LEN
    bad_slots = step.slot_mapping.clone()
    bad_slots[0] = w.num_blocks * w.block_size
    before = to_bits(step.k_cache).copy()
    B.pa_append_kv(step.k_new, step.v_new, bad_slots, step.k_cache, step.v_cache, step.cache)
    assert step.device_errors() & B.DEVERR_SLOT
    after = to_bits(step.k_cache)
    s1 = int(w.slot_mapping[1])
    after_other = after.reshape(-1, 4, 64).copy()
    after_other[s1] = before.reshape(-1, 4, 64)[s1]
    assert np.array_equal(after_other, before.reshape(-1, 4, 64))  # only the valid token landed
    assert step.device_errors() == 0  # the word was cleared


def test_split_k_merge_with_a_dirty_workspace():
    # the split-K partials live in the caller's workspace: a reused workspace
    # full of garbage must give the same result as a fresh one
    w = W.llama2_7b(batch=3, min_len=2000, max_len=3000)
    step = DecodeStep(w, "cuda", partition_tokens=64)
    assert step.workspace is not None
    step.workspace.fill_(0xA5)
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    first = step.out.clone()
    step.workspace.fill_(0xFF)
    step.decode()
    torch.cuda.synchronize()
    assert torch.equal(step.out, first)
    _, _, want = oracle_step(w)
    assert max_abs_err(step.out_f64(), want) <= TOL["f16"]
