"""The KV-bytes formula of the KV cache article (section
'生成一个字，为什么要背一整本账': 2 x layers x KV heads x head_dim x sequence
length x batch x bytes per element) against every worked size the pages
print (tests/golden/kv_bytes_examples.json, each entry with its citation),
and the bench's byte accounting against the same formula."""
import json
import os

import pytest

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "kv_bytes_examples.json")))
UNITS = {"B": 1, "KiB": 2 ** 10, "MiB": 2 ** 20, "GiB": 2 ** 30, "GB": 10 ** 9}


def _args(e):
    return (e["layers"], e["kv_heads"], e["head_dim"], e["seq_len"], e["batch"],
            e["elem_bytes"])


@pytest.mark.parametrize("e", GOLDEN["entries"], ids=lambda e: e["id"])
def test_printed_sizes(oracle_mod, e):
    got = oracle_mod.kv_cache_bytes(*_args(e))
    want = e["printed"] * UNITS[e["unit"]]
    if e["rel_tol"] == 0:
        assert got == want
    else:
        assert abs(got - want) <= e["rel_tol"] * want, (got, want)


@pytest.mark.parametrize("r", GOLDEN["ratios"], ids=lambda r: r["id"])
def test_cache_to_weights_ratios(oracle_mod, r):
    ratio = oracle_mod.kv_cache_bytes(*_args(r)) / r["weights_bytes"]
    lo, hi = r["ratio_range"]
    assert lo <= ratio <= hi, ratio


def test_gqa_shrinks_the_cache_by_the_group_factor(oracle_mod):
    # KV cache article, section '显存账本': Llama-2-70B keeps 8 KV heads for 64
    # query heads, an eighth of the MHA cache
    mha = oracle_mod.kv_cache_bytes(80, 64, 128, 4096, 1, 2)
    gqa = oracle_mod.kv_cache_bytes(80, 8, 128, 4096, 1, 2)
    assert mha == 8 * gqa


def test_bench_byte_accounting_uses_the_formula(oracle_mod):
    from paged_kv_cache_410_b200 import accounting, workloads
    w = workloads.llama2_7b(batch=6, min_len=20, max_len=300)
    acc = accounting.decode_bytes(w)
    want_kv = sum(oracle_mod.kv_cache_bytes(1, w.num_kv_heads, w.head_dim, int(L), 1, 2)
                  for L in w.context_lens)
    assert acc["kv_unique"] == want_kv == acc["kv_logical"]
    # a shared prefix is counted once in the unique bytes, once per sequence in the logical
    p = workloads.llama2_70b_prefix(batch=5, max_suffix=40)
    acc = accounting.decode_bytes(p)
    per_tok = oracle_mod.kv_cache_bytes(1, p.num_kv_heads, p.head_dim, 1, 1, 2)
    assert acc["kv_logical"] == per_tok * int(p.context_lens.sum())
    assert acc["kv_unique"] == per_tok * (2000 + int((p.context_lens - 2000).sum()))


def test_accounting_of_window_fused_and_fp8(oracle_mod):
    from paged_kv_cache_410_b200 import accounting, workloads
    w = workloads.custom([5, 40, 77, 300], num_q_heads=8, num_kv_heads=2, head_dim=128)
    per_tok = oracle_mod.kv_cache_bytes(1, 2, 128, 1, 1, 2)
    # a window of 32 reads min(L, 32) tokens per sequence, and the table entries of
    # the blocks those tokens lie in
    acc = accounting.decode_bytes(w, window=32)
    lens = [5, 40, 77, 300]
    assert acc["kv_unique"] == acc["kv_logical"] == per_tok * sum(min(L, 32) for L in lens)
    blocks = sum((L - 1) // 16 - max(L - 32, 0) // 16 + 1 for L in lens)
    qo = 2 * 4 * 8 * 128 * 2
    assert acc["other"] == qo + 4 * blocks + 4 * 4
    # append + decode in one pass: the new rows are not read back from the cache
    a = accounting.append_bytes(w)
    assert a == 2 * 4 * 2 * 128 * (2 + 2) + 8 * 4
    new_rows = 4 * per_tok
    assert accounting.fused_bytes(w) == accounting.decode_bytes(w)["total_unique"] + a - new_rows
    st = accounting.step_bytes(w, fused=True)
    assert st["total"] == st["append_decode"] + st["copy"]
    # E4M3: one byte per element, plus both scale arrays (fp32 [Hkv][D]) read once
    f = workloads.fp8_beams(batch=24, beam_groups=2, median_len=40, max_len=200)
    acc8 = accounting.decode_bytes(f)
    slots = set()
    for b in range(f.batch):
        for j in range(int(f.context_lens[b])):
            slots.add(int(f.block_tables[b, j // 16]) * 16 + j % 16)
    assert acc8["kv_unique"] == len(slots) * 2 * 8 * 128
    assert acc8["kv_logical"] == int(f.context_lens.sum()) * 2 * 8 * 128
    assert acc8["kv_unique"] < acc8["kv_logical"]                 # beams share prompt blocks
    assert accounting.copy_bytes(f) == len(f.copy_pairs) * 16 * 8 * 128 * 2 * 2
