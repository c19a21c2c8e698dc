"""Test-side helpers: run one step of a workload through the oracle, and the
tolerances the parity tests use.

Tolerances (max absolute error of the decode output against the float64
oracle): 2e-3 when the output is fp16 (fp16 caches and E4M3 caches with fp16
queries, the oracle fed the same dequantised values), 1e-2 when it is bf16.
Append and block copy must be bit-exact."""
import numpy as np

import oracle

TOL = {"f16": 2e-3, "bf16": 1e-2}


def oracle_caches(w):
    """The pool before the step: drawn bits for 16-bit caches, the history
    quantised by the oracle's own encoder for E4M3 caches."""
    if w.cache_dtype == "e4m3":
        shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
        kc = np.zeros(shape, np.uint8)
        vc = np.zeros(shape, np.uint8)
        if w.fill_slots is not None and len(w.fill_slots):
            oracle.append_kv(w.fill_k, w.fill_v, w.io_dtype, w.fill_slots, kc, vc, "e4m3",
                             w.block_size, w.k_inv_scale, w.v_inv_scale)
        return kc, vc
    return w.k_pool.copy(), w.v_pool.copy()


def oracle_step(w, seqs=None, window=0):
    """copy_blocks -> append -> decode on the CPU; returns (k_cache, v_cache,
    out) with out float64 [len(seqs), Hq, D]."""
    kc, vc = oracle_caches(w)
    if len(w.copy_pairs):
        oracle.copy_blocks(w.copy_pairs, kc, vc, w.cache_dtype)
    oracle.append_kv(w.k_new, w.v_new, w.io_dtype, w.slot_mapping, kc, vc, w.cache_dtype,
                     w.block_size, w.k_inv_scale, w.v_inv_scale)
    sel = np.arange(w.batch) if seqs is None else np.asarray(seqs)
    out = oracle.decode(w.q[sel], w.io_dtype, kc, vc, w.cache_dtype, w.block_tables[sel],
                        w.context_lens[sel], w.scale, w.k_scale, w.v_scale, window=window)
    return kc, vc, out


def max_abs_err(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))
