"""Float64 CPU oracle for paged-attention decode (TEST INFRASTRUCTURE ONLY).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its binding in ``paged_kv_cache_410_b200``) never imports, links or calls it,
and this package imports nothing from the product.

The arithmetic lives in ``pa_oracle.c`` (plain C, float64, parallel only over
independent (sequence, query head) outputs); this module compiles it with gcc
and marshals numpy arrays through ctypes. Every function states the passage it
follows in the C source. Storage arrays are passed as raw bit patterns:
fp16/bf16 as ``uint16``, E4M3 as ``uint8``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPES = {"f16": 0, "bf16": 1, "e4m3": 2}

_lib = None


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into liboracle.so next to it (gcc, OpenMP, -O2,
    no fast-math so float64 operations keep their written order)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", "-Wall", "-Wextra", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        lib.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        lib.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_from_float.restype = ctypes.c_uint8
        lib.oracle_kv_cache_bytes.argtypes = [i64] * 6
        lib.oracle_kv_cache_bytes.restype = i64
        lib.oracle_append_kv.argtypes = [P, P, ctypes.c_int, i64, P, P, P, ctypes.c_int, i64,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        lib.oracle_append_kv.restype = ctypes.c_int
        lib.oracle_copy_blocks.argtypes = [P, i32, P, P, ctypes.c_int, i64, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int]
        lib.oracle_copy_blocks.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [P, ctypes.c_int, i32, i32, P, P, ctypes.c_int, i64,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, i32, P,
                                      f32, i32, P]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what} returned status {rc}")


# ---- codecs (format definitions) -------------------------------------------

def f16_to_double(bits: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.oracle_f16_to_double(int(b)) for b in flat]).reshape(np.shape(bits))


def bf16_to_double(bits: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.oracle_bf16_to_double(int(b)) for b in flat]).reshape(np.shape(bits))


def e4m3_to_double(codes: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([lib.oracle_e4m3_to_double(int(c)) for c in flat]).reshape(np.shape(codes))


def e4m3_from_float(x: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(x, dtype=np.float32).ravel()
    return np.array([lib.oracle_e4m3_from_float(float(v)) for v in flat],
                    dtype=np.uint8).reshape(np.shape(x))


def kv_cache_bytes(layers, kv_heads, head_dim, seq_len, batch, elem_bytes) -> int:
    return int(_load().oracle_kv_cache_bytes(layers, kv_heads, head_dim, seq_len, batch,
                                              elem_bytes))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# ---- the three operations --------------------------------------------------

def append_kv(k, v, in_dtype, slot_mapping, k_cache, v_cache, cache_dtype, block_size,
              k_inv_scale=None, v_inv_scale=None):
    """In place: write tokens k, v ([T, Hkv, D] bit patterns) into the caches
    ([NB, BS, Hkv, D]) at slot_mapping; E4M3 caches get the quantised codes."""
    lib = _load()
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    slot_mapping = _c(slot_mapping, np.int64)
    cdt = np.uint8 if cache_dtype == "e4m3" else np.uint16
    for c in (k_cache, v_cache):
        if not (c.flags["C_CONTIGUOUS"] and c.dtype == cdt):
            raise TypeError("cache must be a C-contiguous array of the storage type")
    nb, bs, hkv, d = k_cache.shape
    assert bs == block_size and k.shape[1:] == (hkv, d)
    ks = None if k_inv_scale is None else _c(k_inv_scale, np.float32)
    vs = None if v_inv_scale is None else _c(v_inv_scale, np.float32)
    rc = lib.oracle_append_kv(_ptr(k), _ptr(v), DTYPES[in_dtype], k.shape[0], _ptr(slot_mapping),
                              _ptr(k_cache), _ptr(v_cache), DTYPES[cache_dtype], nb, bs, hkv, d,
                              _ptr(ks), _ptr(vs))
    _check(rc, "oracle_append_kv")


def copy_blocks(pairs, k_cache, v_cache, cache_dtype):
    """In place: for each (src, dst) row of pairs copy block src to dst."""
    lib = _load()
    pairs = _c(np.asarray(pairs, dtype=np.int32).reshape(-1, 2), np.int32)
    nb, bs, hkv, d = k_cache.shape
    rc = lib.oracle_copy_blocks(_ptr(pairs), pairs.shape[0], _ptr(k_cache), _ptr(v_cache),
                                DTYPES[cache_dtype], nb, bs, hkv, d)
    _check(rc, "oracle_copy_blocks")


def decode(q, q_dtype, k_cache, v_cache, cache_dtype, block_tables, context_lens, scale,
           k_scale=None, v_scale=None, window=0) -> np.ndarray:
    """Float64 attention output [B, Hq, D] of one query per sequence over its
    paged history (its last `window` tokens when window > 0)."""
    lib = _load()
    q = _c(q, np.uint16)
    block_tables = _c(block_tables, np.int32)
    context_lens = _c(context_lens, np.int32)
    b, hq, d = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    assert d == d2
    ks = None if k_scale is None else _c(k_scale, np.float32)
    vs = None if v_scale is None else _c(v_scale, np.float32)
    kc = np.ascontiguousarray(k_cache)
    vc = np.ascontiguousarray(v_cache)
    out = np.empty((b, hq, d), dtype=np.float64)
    rc = lib.oracle_decode(_ptr(q), DTYPES[q_dtype], b, hq, _ptr(kc), _ptr(vc),
                           DTYPES[cache_dtype], nb, bs, hkv, d, _ptr(ks), _ptr(vs),
                           _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                           float(np.float32(scale)), int(window), _ptr(out))
    _check(rc, "oracle_decode")
    return out


def _values(a: np.ndarray, dtype: str) -> np.ndarray:
    """Stored bit patterns as float64 values."""
    if dtype == "f16":
        return f16_to_double(a)
    if dtype == "bf16":
        return bf16_to_double(a)
    return e4m3_to_double(a)


def decode_partial(q, q_dtype, k_cache, v_cache, cache_dtype, block_tables, context_lens, scale,
                   k_scale=None, v_scale=None):
    """The pieces of the decode over the tokens each table lists, for merging
    with other parts of the same histories (numpy, float64; small cases).
    Returns (o [B, Hq, D], m [B, Hq], l [B, Hq]) with s_j = scale * q . k_j
    over the row's tokens, m = max_j s_j, l = sum_j exp(s_j - m) and
    o = sum_j exp(s_j - m) v_j / l: the softmax of the decode's attention
    equation split at its normaliser. A row with no tokens gives o = 0,
    m = -inf, l = 0. (The attention equation of "AI 陪读顶会论文（三）：KV
    Cache 显存占用计算与 PagedAttention 原理拆解", section "为什么自回归解码
    必须使用 KV Cache？", as ``decode`` computes it, with the softmax's sum
    left unnormalised across parts.)"""
    qv = _values(np.asarray(q), q_dtype)
    kc = _values(np.asarray(k_cache), cache_dtype)
    vc = _values(np.asarray(v_cache), cache_dtype)
    if cache_dtype == "e4m3":
        kc = kc * np.asarray(k_scale, np.float64)[None, None]
        vc = vc * np.asarray(v_scale, np.float64)[None, None]
    b_n, hq, d = qv.shape
    _, bs, hkv, _ = kc.shape
    group = hq // hkv
    o = np.zeros((b_n, hq, d))
    m = np.full((b_n, hq), -np.inf)
    l = np.zeros((b_n, hq))
    for b in range(b_n):
        L = int(context_lens[b])
        if L == 0:
            continue
        j = np.arange(L)
        blk = np.asarray(block_tables[b])[j // bs]
        K = kc[blk, j % bs]  # [L, Hkv, D]
        V = vc[blk, j % bs]
        for i in range(hq):
            h = i // group
            s = float(np.float32(scale)) * (K[:, h] @ qv[b, i])
            m[b, i] = s.max()
            e = np.exp(s - m[b, i])
            l[b, i] = e.sum()
            o[b, i] = (e @ V[:, h]) / l[b, i]
    return o, m, l


def merge_partials(o, m, l):
    """Merge parts stacked part-major (o [N, ..., D], m and l [N, ...]) of the
    same rows into the decode output: sum_n w_n o_n / sum_n w_n with
    w_n = l_n exp(m_n - max_n m_n); parts with l = 0 weigh nothing and rows
    without any token give 0."""
    o = np.asarray(o, np.float64)
    m = np.asarray(m, np.float64)
    l = np.asarray(l, np.float64)
    M = np.max(np.where(l > 0, m, -np.inf), axis=0)
    M = np.where(np.isfinite(M), M, 0.0)  # (rows without tokens: every weight is 0)
    w = np.where(l > 0, l * np.exp(np.where(l > 0, m, 0.0) - M[None]), 0.0)
    den = w.sum(axis=0)
    num = (w[..., None] * o).sum(axis=0)
    return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)
