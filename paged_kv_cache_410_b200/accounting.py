"""Algorithmic byte counts of one pass of the hot path (host side, numpy).

These are the bytes the method must move, not what a kernel happens to
move: every KV element a decode reads (once per physical slot for the
``unique`` count, once per sequence for the ``logical`` count), the query,
the output, the block-table entries and lengths it reads, the tokens an
append writes and the blocks a copy duplicates. The KV part follows the
KV cache article's formula (section '生成一个字，为什么要背一整本账': 2 x KV
heads x head_dim x tokens x bytes per element, one layer).
"""
from __future__ import annotations

import numpy as np

ELEM_BYTES = {"f16": 2, "bf16": 2, "e4m3": 1}


def _attended(w, window: int):
    """Per sequence, the first attended token and the count."""
    lens = w.context_lens.astype(np.int64)
    lo = np.maximum(lens - window, 0) if window > 0 else np.zeros_like(lens)
    return lo, lens - lo


def _unique_slots(w, window: int = 0) -> int:
    """Distinct physical (block, row) slots read by all sequences."""
    bs = w.block_size
    lo, n = _attended(w, window)
    seen = np.zeros(w.num_blocks * bs, dtype=bool)
    for b in range(w.batch):
        if n[b] <= 0:
            continue
        j = np.arange(lo[b], lo[b] + n[b], dtype=np.int64)
        seen[w.block_tables[b, j // bs].astype(np.int64) * bs + j % bs] = True
    return int(seen.sum())


def decode_bytes(w, window: int = 0) -> dict:
    """`window` > 0: each sequence reads only its last `window` tokens."""
    eb = ELEM_BYTES[w.cache_dtype]
    io = ELEM_BYTES[w.io_dtype]
    per_token = 2 * w.num_kv_heads * w.head_dim * eb  # K and V of one token, one layer
    lo, n = _attended(w, window)
    kv_logical = int(per_token * n.sum())
    kv_unique = int(per_token * _unique_slots(w, window))
    qo = 2 * w.batch * w.num_q_heads * w.head_dim * io
    bs = w.block_size
    tables = int(4 * np.sum(np.where(n > 0, (lo + n - 1) // bs - lo // bs + 1, 0)))
    other = qo + tables + 4 * w.batch
    if w.cache_dtype == "e4m3":
        other += 2 * w.num_kv_heads * w.head_dim * 4
    return {"kv_unique": kv_unique, "kv_logical": kv_logical, "other": other,
            "total_unique": kv_unique + other, "total_logical": kv_logical + other}


def append_bytes(w) -> int:
    io = ELEM_BYTES[w.io_dtype]
    eb = ELEM_BYTES[w.cache_dtype]
    T = int(np.sum(w.slot_mapping >= 0))
    n = 2 * T * w.num_kv_heads * w.head_dim * (io + eb) + 8 * w.batch
    if w.cache_dtype == "e4m3":
        n += 2 * w.num_kv_heads * w.head_dim * 4
    return int(n)


def copy_bytes(w) -> int:
    block = w.block_size * w.num_kv_heads * w.head_dim * ELEM_BYTES[w.cache_dtype]
    return int(len(w.copy_pairs) * block * 2 * 2)


def fused_bytes(w) -> int:
    """Append and decode as one pass: the decode's bytes and the append's,
    less the cache read of each new token's row (the pass takes that row from
    the appended input instead; it lies in a block no other sequence reads)."""
    eb = ELEM_BYTES[w.cache_dtype]
    T = int(np.sum(w.slot_mapping >= 0))
    new_rows = 2 * T * w.num_kv_heads * w.head_dim * eb
    return decode_bytes(w)["total_unique"] + append_bytes(w) - new_rows


def step_bytes(w, window: int = 0, fused: bool = False) -> dict:
    """`fused`: append and decode counted as one pass (fused_bytes)."""
    d = decode_bytes(w, window)
    a = append_bytes(w)
    c = copy_bytes(w)
    out = {"decode": d["total_unique"], "decode_logical": d["total_logical"],
           "kv_unique": d["kv_unique"], "append": a, "copy": c,
           "total": d["total_unique"] + a + c}
    if fused:
        out["append_decode"] = fused_bytes(w)
        out["total"] = out["append_decode"] + c
    return out
