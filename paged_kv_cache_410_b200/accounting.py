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


def _unique_slots(w) -> int:
    """Distinct physical (block, row) slots read by all sequences: rows of a
    block are filled from row 0, so a block contributes the largest row count
    any sequence uses in it."""
    rows = np.zeros(w.num_blocks, dtype=np.int64)
    bs = w.block_size
    for b in range(w.batch):
        L = int(w.context_lens[b])
        if L <= 0:
            continue
        n = -(-L // bs)
        blocks = w.block_tables[b, :n].astype(np.int64)
        used = np.full(n, bs, dtype=np.int64)
        used[-1] = L - (n - 1) * bs
        np.maximum.at(rows, blocks, used)
    return int(rows.sum())


def decode_bytes(w) -> dict:
    eb = ELEM_BYTES[w.cache_dtype]
    io = ELEM_BYTES[w.io_dtype]
    per_token = 2 * w.num_kv_heads * w.head_dim * eb  # K and V of one token, one layer
    lens = w.context_lens.astype(np.int64)
    kv_logical = int(per_token * lens.sum())
    kv_unique = int(per_token * _unique_slots(w))
    qo = 2 * w.batch * w.num_q_heads * w.head_dim * io
    tables = int(4 * np.sum(-(-lens // w.block_size)))
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


def step_bytes(w) -> dict:
    d = decode_bytes(w)
    a = append_bytes(w)
    c = copy_bytes(w)
    return {"decode": d["total_unique"], "decode_logical": d["total_logical"],
            "kv_unique": d["kv_unique"], "append": a, "copy": c,
            "total": d["total_unique"] + a + c}
