"""Python binding of libpagedattn.so (ctypes, argument marshalling only).

Each function forwards torch tensors' device pointers and sizes to the C
entry point of the same name (include/pa_api.h); every step of the hot path
runs in the library's CUDA kernels. Torch provides device memory and
streams. If the library is not built the first call raises: there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpagedattn.so")

PA_F16, PA_BF16, PA_E4M3 = 0, 1, 2
PA_OK = 0
STATUS = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_CUDA",
          4: "PA_ERR_WORKSPACE", 5: "PA_ERR_DEVICE_BOUNDS"}
DEVERR_BLOCK_ID, DEVERR_CONTEXT_LEN, DEVERR_SLOT, DEVERR_PREFIX = 0x1, 0x2, 0x4, 0x8
DEVERR_TIMEOUT = 0x10

# names of every symbol include/pa_api.h declares
EXPORTED = ["pa_append_kv", "pa_decode_workspace_size", "pa_decode_partition_tokens",
            "pa_decode", "pa_copy_blocks", "pa_get_device_error", "pa_status_string",
            "pa_version", "pa_decode_static_workspace",
            "pa_decode_shared_prefix_workspace_size", "pa_decode_shared_prefix",
            "pa_decode_sliding_window_workspace_size", "pa_decode_sliding_window",
            "pa_append_decode", "pa_copy_blocks_layers",
            "pa_decode_shared_prefix_partition_tokens", "pa_testing_withhold_prefix_scores",
            "pa_set_deterministic", "pa_testing_withhold_steal_counts",
            "pa_decode_partial", "pa_merge_partials"]


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class _CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int64), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("cache_dtype", ctypes.c_int32), ("k_scale", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("k_inv_scale", ctypes.c_void_p),
                ("v_inv_scale", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libpagedattn.so and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built (run paged_kv_cache_410_b200.build.build());"
                           " the paged-attention path has no fallback")
    lib = ctypes.CDLL(path)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    D = ctypes.POINTER(_CacheDesc)
    lib.pa_append_kv.argtypes = [P, P, i32, i64, P, P, P, D, P]
    lib.pa_append_kv.restype = ctypes.c_int
    lib.pa_decode_workspace_size.argtypes = [i32, i32, i32, i32, D]
    lib.pa_decode_workspace_size.restype = ctypes.c_size_t
    lib.pa_decode_partition_tokens.argtypes = [i32, i32, D]
    lib.pa_decode_partition_tokens.restype = i32
    lib.pa_decode.argtypes = [P, i32, i32, i32, P, P, D, P, i32, P, i32, ctypes.c_float, P, i32,
                              P, ctypes.c_size_t, P]
    lib.pa_decode.restype = ctypes.c_int
    lib.pa_copy_blocks.argtypes = [P, i32, P, P, D, P]
    lib.pa_copy_blocks.restype = ctypes.c_int
    lib.pa_get_device_error.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.pa_get_device_error.restype = ctypes.c_int
    lib.pa_status_string.argtypes = [i32]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_version.argtypes = []
    lib.pa_version.restype = i32
    lib.pa_set_deterministic.argtypes = [i32]
    lib.pa_set_deterministic.restype = i32
    lib.pa_testing_withhold_steal_counts.argtypes = [i32]
    lib.pa_testing_withhold_steal_counts.restype = None
    lib.pa_decode_partial.argtypes = [P, i32, i32, i32, P, P, D, P, i32, P, i32, ctypes.c_float,
                                      P, P, i32, P, ctypes.c_size_t, P]
    lib.pa_decode_partial.restype = ctypes.c_int
    lib.pa_merge_partials.argtypes = [P, P, i32, ctypes.c_int64, i32, P, i32, P]
    lib.pa_merge_partials.restype = ctypes.c_int
    lib.pa_decode_static_workspace.argtypes = [P, i32, i32, i32, P, P, D, P, i32, P, i32,
                                               ctypes.c_float, P, i32, P]
    lib.pa_decode_static_workspace.restype = ctypes.c_int
    lib.pa_decode_shared_prefix_workspace_size.argtypes = [i32, i32, i32, i32, i32, D]
    lib.pa_decode_shared_prefix_workspace_size.restype = ctypes.c_size_t
    lib.pa_decode_shared_prefix.argtypes = [P, i32, i32, i32, P, P, D, P, i32, P, i32, i32,
                                            ctypes.c_float, P, i32, P, ctypes.c_size_t, P]
    lib.pa_decode_shared_prefix.restype = ctypes.c_int
    lib.pa_decode_sliding_window_workspace_size.argtypes = [i32, i32, i32, i32, i32, D]
    lib.pa_decode_sliding_window_workspace_size.restype = ctypes.c_size_t
    lib.pa_decode_sliding_window.argtypes = [P, i32, i32, i32, P, P, D, P, i32, P, i32, i32,
                                             ctypes.c_float, P, i32, P, ctypes.c_size_t, P]
    lib.pa_decode_sliding_window.restype = ctypes.c_int
    lib.pa_append_decode.argtypes = [P, P, P, i32, i32, i32, P, P, P, D, P, i32, P, i32,
                                     ctypes.c_float, P, i32, P, ctypes.c_size_t, P]
    lib.pa_append_decode.restype = ctypes.c_int
    lib.pa_copy_blocks_layers.argtypes = [P, i32, ctypes.POINTER(P), ctypes.POINTER(P), i32, D,
                                          P]
    lib.pa_copy_blocks_layers.restype = ctypes.c_int
    lib.pa_decode_shared_prefix_partition_tokens.argtypes = [i32, i32, i32, i32, D]
    lib.pa_decode_shared_prefix_partition_tokens.restype = i32
    lib.pa_testing_withhold_prefix_scores.argtypes = [i32]
    lib.pa_testing_withhold_prefix_scores.restype = None
    _lib = lib
    return lib


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float16:
        return PA_F16
    if t == torch.bfloat16:
        return PA_BF16
    if t in (torch.uint8, torch.float8_e4m3fn):
        return PA_E4M3
    raise TypeError(f"unsupported dtype {t}")


_IO = (torch.float16, torch.bfloat16)
_E4M3 = (torch.uint8, torch.float8_e4m3fn)


def _on_device(t: torch.Tensor) -> bool:
    return t.is_cuda


def _dev(t, name: str, dtypes=None, shape=None) -> int | None:
    """Device address of a contiguous CUDA tensor, after checking its dtype and
    shape (None, where the C call allows NULL, passes through)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not _on_device(t) or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA tensor")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")
    if shape is not None and t.shape != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


@dataclass
class PagedCache:
    """Shape and (for E4M3) scales of one layer's paged K and V caches,
    laid out [num_blocks, block_size, num_kv_heads, head_dim]."""
    num_blocks: int
    block_size: int
    num_kv_heads: int
    head_dim: int
    dtype: torch.dtype
    k_scale: torch.Tensor | None = None      # fp32 [num_kv_heads, head_dim], device
    v_scale: torch.Tensor | None = None
    k_inv_scale: torch.Tensor | None = None
    v_inv_scale: torch.Tensor | None = None

    def desc(self) -> _CacheDesc:
        sc = (self.num_kv_heads, self.head_dim)
        f32 = (torch.float32,)
        return _CacheDesc(self.num_blocks, self.block_size, self.num_kv_heads, self.head_dim,
                          _dtype_code(self.dtype), _dev(self.k_scale, "k_scale", f32, sc),
                          _dev(self.v_scale, "v_scale", f32, sc),
                          _dev(self.k_inv_scale, "k_inv_scale", f32, sc),
                          _dev(self.v_inv_scale, "v_inv_scale", f32, sc))

    @property
    def shape(self):
        return (self.num_blocks, self.block_size, self.num_kv_heads, self.head_dim)

    def cache_ptrs(self, k_cache, v_cache):
        """Device addresses of this layer's K and V caches (checked against the
        shape and dtype described here)."""
        dt = _E4M3 if self.dtype in _E4M3 else (self.dtype,)
        return _dev(k_cache, "k_cache", dt, self.shape), _dev(v_cache, "v_cache", dt, self.shape)

    @staticmethod
    def for_tensor(cache: torch.Tensor, **scales) -> "PagedCache":
        nb, bs, hkv, d = cache.shape
        return PagedCache(nb, bs, hkv, d, cache.dtype, **scales)


def _check(rc: int, what: str):
    if rc != PA_OK:
        raise PagedAttentionError(rc, what)


def _new_tokens(k, v, slot_mapping, cache: PagedCache, rows=None):
    """Checked addresses of new tokens' k, v ([T, Hkv, D], one 16-bit dtype)
    and slot_mapping ([T] int64)."""
    t = k.shape[0] if rows is None else rows
    shape = (t, cache.num_kv_heads, cache.head_dim)
    pk = _dev(k, "k", _IO, shape)
    pv = _dev(v, "v", (k.dtype,), shape)
    return pk, pv, _dev(slot_mapping, "slot_mapping", (torch.int64,), (t,))


def _decode_io(q, block_tables, context_lens, out, cache: PagedCache):
    """Checked addresses of q [B, Hq, D], block_tables [B, MB] int32,
    context_lens [B] int32 and out (q's shape and dtype)."""
    if q.dim() != 3:
        raise ValueError("q: expected [batch, num_q_heads, head_dim]")
    batch, hq = q.shape[0], q.shape[1]
    pq = _dev(q, "q", _IO, (batch, hq, cache.head_dim))
    if block_tables.dim() != 2:
        raise ValueError("block_tables: expected [batch, max_blocks_per_seq]")
    pt = _dev(block_tables, "block_tables", (torch.int32,), (batch, block_tables.shape[1]))
    pl = _dev(context_lens, "context_lens", (torch.int32,), (batch,))
    po = _dev(out, "out", (q.dtype,), tuple(q.shape))
    return pq, pt, pl, po


def pa_append_kv(k, v, slot_mapping, k_cache, v_cache, cache: PagedCache, stream=None):
    """Store k, v ([T, Hkv, D], fp16/bf16) at slot_mapping ([T] int64)."""
    lib = load_library()
    d = cache.desc()
    pk, pv, ps = _new_tokens(k, v, slot_mapping, cache)
    kc, vc = cache.cache_ptrs(k_cache, v_cache)
    rc = lib.pa_append_kv(pk, pv, _dtype_code(k.dtype), k.shape[0], ps, kc, vc, ctypes.byref(d),
                          _stream(stream))
    _check(rc, "pa_append_kv")


def pa_decode_workspace_size(batch, num_q_heads, max_context, cache: PagedCache,
                             partition_tokens=0) -> int:
    lib = load_library()
    d = cache.desc()
    return int(lib.pa_decode_workspace_size(batch, num_q_heads, max_context, partition_tokens,
                                            ctypes.byref(d)))


def pa_decode_partition_tokens(batch, max_context, cache: PagedCache) -> int:
    lib = load_library()
    d = cache.desc()
    return int(lib.pa_decode_partition_tokens(batch, max_context, ctypes.byref(d)))


def pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, cache: PagedCache,
              max_context: int, partition_tokens: int = 0, workspace=None, stream=None):
    """out[b, i] = softmax(scale * q[b, i] . K^T) V over sequence b's paged
    history. `workspace` is a uint8 device tensor of at least
    pa_decode_workspace_size(...) bytes (or None when that is 0)."""
    lib = load_library()
    d = cache.desc()
    pq, pt, pl, po = _decode_io(q, block_tables, context_lens, out, cache)
    kc, vc = cache.cache_ptrs(k_cache, v_cache)
    rc = lib.pa_decode(pq, _dtype_code(q.dtype), q.shape[0], q.shape[1], kc, vc,
                       ctypes.byref(d), pt, block_tables.shape[1], pl, int(max_context),
                       float(scale), po, int(partition_tokens), _dev(workspace, "workspace"),
                       _nbytes(workspace), _stream(stream))
    _check(rc, "pa_decode")


def pa_decode_partial(q, k_cache, v_cache, block_tables, context_lens, scale, part_o, part_ml,
                      cache: PagedCache, max_context: int, partition_tokens: int = 0,
                      workspace=None, stream=None):
    """pa_decode over the tokens each table lists, left as the pieces a merge
    of several such calls needs: part_o [B, Hq, D] float32 (each row's
    normalised output) and part_ml [B, Hq, 2] float32 (max score in log2
    units, sum of 2^(score - max)). Workspace as for pa_decode."""
    lib = load_library()
    d = cache.desc()
    batch, hq = q.shape[0], q.shape[1]
    pq, pt, pl, _ = _decode_io(q, block_tables, context_lens, q, cache)
    po = _dev(part_o, "part_o", (torch.float32,), (batch, hq, cache.head_dim))
    pm = _dev(part_ml, "part_ml", (torch.float32,), (batch, hq, 2))
    kc, vc = cache.cache_ptrs(k_cache, v_cache)
    rc = lib.pa_decode_partial(pq, _dtype_code(q.dtype), batch, hq, kc, vc, ctypes.byref(d), pt,
                               block_tables.shape[1], pl, int(max_context), float(scale), po, pm,
                               int(partition_tokens), _dev(workspace, "workspace"),
                               _nbytes(workspace), _stream(stream))
    _check(rc, "pa_decode_partial")


def pa_merge_partials(part_o, part_ml, out, stream=None):
    """out [rows..., D] (fp16 / bf16) from pa_decode_partial results stacked
    part-major: part_o [N, rows..., D] float32, part_ml [N, rows..., 2]
    float32 (an all-gather's layout)."""
    lib = load_library()
    if part_o.dim() < 2 or part_o.shape[1:] != out.shape:
        raise ValueError("part_o: expected [num_parts, *out.shape]")
    n, hd = part_o.shape[0], out.shape[-1]
    rows = out.numel() // hd if hd else 0
    po = _dev(part_o, "part_o", (torch.float32,))
    pm = _dev(part_ml, "part_ml", (torch.float32,), tuple(part_o.shape[:-1]) + (2,))
    pout = _dev(out, "out", _IO)
    rc = lib.pa_merge_partials(po, pm, int(n), int(rows), int(hd), pout, _dtype_code(out.dtype),
                               _stream(stream))
    _check(rc, "pa_merge_partials")


def pa_append_decode(q, k, v, slot_mapping, k_cache, v_cache, block_tables, context_lens,
                     scale, out, cache: PagedCache, max_context: int, partition_tokens: int = 0,
                     workspace=None, stream=None):
    """pa_append_kv of one new token per sequence (k, v: [batch, Hkv, D];
    slot_mapping: [batch] int64, the slot of position context_lens[b] - 1,
    or -1 for none) and pa_decode over the updated history, in one launch.
    The workspace is sized by pa_decode_workspace_size."""
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("pa_append_decode: q, k and v share one dtype")
    lib = load_library()
    d = cache.desc()
    pq, pt, pl, po = _decode_io(q, block_tables, context_lens, out, cache)
    pk, pv, ps = _new_tokens(k, v, slot_mapping, cache, rows=q.shape[0])
    kc, vc = cache.cache_ptrs(k_cache, v_cache)
    rc = lib.pa_append_decode(pq, pk, pv, _dtype_code(q.dtype), q.shape[0], q.shape[1], ps, kc,
                              vc, ctypes.byref(d), pt, block_tables.shape[1], pl,
                              int(max_context), float(scale), po, int(partition_tokens),
                              _dev(workspace, "workspace"), _nbytes(workspace), _stream(stream))
    _check(rc, "pa_append_decode")


def pa_decode_shared_prefix_workspace_size(batch, num_q_heads, max_context, prefix_blocks,
                                           cache: PagedCache, partition_tokens=0) -> int:
    lib = load_library()
    d = cache.desc()
    return int(lib.pa_decode_shared_prefix_workspace_size(batch, num_q_heads, max_context,
                                                          prefix_blocks, partition_tokens,
                                                          ctypes.byref(d)))


def pa_decode_shared_prefix_partition_tokens(batch, num_q_heads, max_context, prefix_blocks,
                                             cache: PagedCache) -> int:
    lib = load_library()
    d = cache.desc()
    return int(lib.pa_decode_shared_prefix_partition_tokens(batch, num_q_heads, max_context,
                                                            prefix_blocks, ctypes.byref(d)))


def pa_decode_shared_prefix(q, k_cache, v_cache, block_tables, context_lens, scale, out,
                            cache: PagedCache, max_context: int, prefix_blocks: int,
                            partition_tokens: int = 0, workspace=None, stream=None):
    """pa_decode for a batch whose block tables all start with the same
    `prefix_blocks` physical blocks: the shared prefix is attended once per
    KV head for all sequences, then merged with each sequence's suffix."""
    lib = load_library()
    d = cache.desc()
    pq, pt, pl, po = _decode_io(q, block_tables, context_lens, out, cache)
    kc, vc = cache.cache_ptrs(k_cache, v_cache)
    rc = lib.pa_decode_shared_prefix(pq, _dtype_code(q.dtype), q.shape[0], q.shape[1], kc, vc,
                                     ctypes.byref(d), pt, block_tables.shape[1], pl,
                                     int(max_context), int(prefix_blocks), float(scale), po,
                                     int(partition_tokens), _dev(workspace, "workspace"),
                                     _nbytes(workspace), _stream(stream))
    _check(rc, "pa_decode_shared_prefix")


def pa_decode_sliding_window_workspace_size(batch, num_q_heads, max_context, window,
                                            cache: PagedCache, partition_tokens=0) -> int:
    lib = load_library()
    d = cache.desc()
    return int(lib.pa_decode_sliding_window_workspace_size(batch, num_q_heads, max_context,
                                                           window, partition_tokens,
                                                           ctypes.byref(d)))


def pa_decode_sliding_window(q, k_cache, v_cache, block_tables, context_lens, scale, out,
                             cache: PagedCache, max_context: int, window: int,
                             partition_tokens: int = 0, workspace=None, stream=None):
    """pa_decode attending only to each sequence's last `window` tokens."""
    lib = load_library()
    d = cache.desc()
    pq, pt, pl, po = _decode_io(q, block_tables, context_lens, out, cache)
    kc, vc = cache.cache_ptrs(k_cache, v_cache)
    rc = lib.pa_decode_sliding_window(pq, _dtype_code(q.dtype), q.shape[0], q.shape[1], kc, vc,
                                      ctypes.byref(d), pt, block_tables.shape[1], pl,
                                      int(max_context), int(window), float(scale), po,
                                      int(partition_tokens), _dev(workspace, "workspace"),
                                      _nbytes(workspace), _stream(stream))
    _check(rc, "pa_decode_sliding_window")


def pa_decode_static_workspace(q, k_cache, v_cache, block_tables, context_lens, scale, out,
                               cache: PagedCache, max_context: int, partition_tokens: int = 0,
                               stream=None):
    """pa_decode for callers that cannot allocate device memory: the split-K
    workspace is the library's own fixed 32 MiB array (see include/pa_api.h
    for the limit, the first-call set-up and the rule that overlapping calls
    race on the shared array)."""
    lib = load_library()
    d = cache.desc()
    pq, pt, pl, po = _decode_io(q, block_tables, context_lens, out, cache)
    kc, vc = cache.cache_ptrs(k_cache, v_cache)
    rc = lib.pa_decode_static_workspace(pq, _dtype_code(q.dtype), q.shape[0], q.shape[1], kc, vc,
                                        ctypes.byref(d), pt, block_tables.shape[1], pl,
                                        int(max_context), float(scale), po,
                                        int(partition_tokens), _stream(stream))
    _check(rc, "pa_decode_static_workspace")


def pa_copy_blocks(pairs, k_cache, v_cache, cache: PagedCache, stream=None):
    """Copy K and V block pairs[p][0] -> pairs[p][1]; `pairs` is host data."""
    lib = load_library()
    d = cache.desc()
    arr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    kc, vc = cache.cache_ptrs(k_cache, v_cache)
    rc = lib.pa_copy_blocks(arr.ctypes.data_as(ctypes.c_void_p), arr.shape[0], kc, vc,
                            ctypes.byref(d), _stream(stream))
    _check(rc, "pa_copy_blocks")


def pa_copy_blocks_layers(pairs, k_caches, v_caches, cache: PagedCache, stream=None):
    """pa_copy_blocks on every layer's K and V cache (sequences of device
    tensors, one per layer, all of `cache`'s shape) in one call."""
    if len(k_caches) != len(v_caches):
        raise ValueError("one K and one V cache per layer")
    lib = load_library()
    d = cache.desc()
    arr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    n = len(k_caches)
    ptrs = [cache.cache_ptrs(k, v) for k, v in zip(k_caches, v_caches)]
    kp = (ctypes.c_void_p * max(n, 1))(*[a for a, _ in ptrs])
    vp = (ctypes.c_void_p * max(n, 1))(*[b for _, b in ptrs])
    rc = lib.pa_copy_blocks_layers(arr.ctypes.data_as(ctypes.c_void_p), arr.shape[0], kp, vp, n,
                                   ctypes.byref(d), _stream(stream))
    _check(rc, "pa_copy_blocks_layers")


def pa_testing_withhold_steal_counts(on: bool):
    """Test hook (process-wide): in a steal-mode decode that merges its rows
    in the launch, each row's first CTA does not count its partial, so the
    rows' bounded waits run out (PA_DEVERR_TIMEOUT)."""
    load_library().pa_testing_withhold_steal_counts(1 if on else 0)


def pa_testing_withhold_prefix_scores(on: bool):
    """Test hook (process-wide): the shared-prefix tensor-core kernel's MMA
    warp issues nothing, so its bounded waits run out (PA_DEVERR_TIMEOUT)."""
    load_library().pa_testing_withhold_prefix_scores(1 if on else 0)


def pa_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error bits."""
    lib = load_library()
    flags = ctypes.c_uint32(0)
    rc = lib.pa_get_device_error(_stream(stream), ctypes.byref(flags))
    if rc not in (PA_OK, 5):
        raise PagedAttentionError(rc, "pa_get_device_error")
    return int(flags.value)


def pa_status_string(status: int) -> str:
    return load_library().pa_status_string(status).decode()


def pa_version() -> int:
    return int(load_library().pa_version())


def pa_set_deterministic(on: bool) -> bool:
    """Reproducible results on (no steal mode for single-sequence split
    decodes) or off (the default); returns the previous setting."""
    return bool(load_library().pa_set_deterministic(1 if on else 0))


class deterministic:
    """``with deterministic():`` runs its body with reproducible results on
    and puts the previous setting back after."""

    def __enter__(self):
        self.prev = pa_set_deterministic(True)
        return self

    def __exit__(self, *exc):
        pa_set_deterministic(self.prev)
        return False
