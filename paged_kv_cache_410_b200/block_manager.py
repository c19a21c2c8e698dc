"""Python binding of the host block manager (include/pa_block_manager.h),
ctypes over libpagedattn.so: argument marshalling only."""
from __future__ import annotations

import ctypes

import numpy as np

from .binding import load_library

OK, ERR_INVALID, ERR_NO_BLOCKS, ERR_CAPACITY = 0, -1, -2, -3

EXPORTED = ["pa_bm_create", "pa_bm_destroy", "pa_bm_num_free_blocks", "pa_bm_num_cached_blocks",
            "pa_bm_block_refcount", "pa_bm_add_sequence", "pa_bm_append_token", "pa_bm_fork",
            "pa_bm_free_sequence", "pa_bm_release_before", "pa_bm_sequence_length",
            "pa_bm_slots", "pa_bm_block_tables", "pa_bm_block_tables_update",
            "pa_bm_append_tokens", "pa_bm_release_window"]

_declared = False


def _lib():
    global _declared
    lib = load_library()
    if not _declared:
        P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        lib.pa_bm_create.argtypes = [i64, i32, i32]
        lib.pa_bm_create.restype = P
        lib.pa_bm_destroy.argtypes = [P]
        lib.pa_bm_destroy.restype = None
        lib.pa_bm_num_free_blocks.argtypes = [P]
        lib.pa_bm_num_free_blocks.restype = i64
        lib.pa_bm_num_cached_blocks.argtypes = [P]
        lib.pa_bm_num_cached_blocks.restype = i64
        lib.pa_bm_block_refcount.argtypes = [P, i64]
        lib.pa_bm_block_refcount.restype = i32
        lib.pa_bm_add_sequence.argtypes = [P, i64, P, i32, ctypes.POINTER(i32)]
        lib.pa_bm_add_sequence.restype = i32
        lib.pa_bm_append_token.argtypes = [P, i64, i32, ctypes.POINTER(i64), ctypes.POINTER(i32),
                                           ctypes.POINTER(i32)]
        lib.pa_bm_append_token.restype = i32
        lib.pa_bm_append_tokens.argtypes = [P, P, P, i32, P, P, ctypes.POINTER(i32)]
        lib.pa_bm_append_tokens.restype = i32
        lib.pa_bm_release_window.argtypes = [P, P, i32, i32]
        lib.pa_bm_release_window.restype = i32
        lib.pa_bm_fork.argtypes = [P, i64, i64]
        lib.pa_bm_fork.restype = i32
        lib.pa_bm_free_sequence.argtypes = [P, i64]
        lib.pa_bm_free_sequence.restype = i32
        lib.pa_bm_release_before.argtypes = [P, i64, i32]
        lib.pa_bm_release_before.restype = i32
        lib.pa_bm_sequence_length.argtypes = [P, i64]
        lib.pa_bm_sequence_length.restype = i32
        lib.pa_bm_slots.argtypes = [P, i64, i32, i32, P]
        lib.pa_bm_slots.restype = i32
        lib.pa_bm_block_tables.argtypes = [P, P, i32, i32, P, P]
        lib.pa_bm_block_tables.restype = i32
        lib.pa_bm_block_tables_update.argtypes = [P, P, i32, i32, P, P, P, ctypes.POINTER(i32)]
        lib.pa_bm_block_tables_update.restype = i32
        _declared = True
    return lib


class BlockManagerError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: status {code}")


def _ok(rc, what):
    if rc != OK:
        raise BlockManagerError(rc, what)


class BlockManager:
    """Pool of `num_blocks` blocks of `block_size` tokens (see
    include/pa_block_manager.h for the semantics of every call)."""

    def __init__(self, num_blocks: int, block_size: int, prefix_cache: bool = False):
        self._lib = _lib()
        self._h = self._lib.pa_bm_create(num_blocks, block_size, int(prefix_cache))
        if not self._h:
            raise BlockManagerError(ERR_INVALID, "pa_bm_create")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if self._h:
            self._lib.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    @property
    def num_free_blocks(self) -> int:
        return int(self._lib.pa_bm_num_free_blocks(self._h))

    @property
    def num_cached_blocks(self) -> int:
        return int(self._lib.pa_bm_num_cached_blocks(self._h))

    def refcount(self, block: int) -> int:
        return int(self._lib.pa_bm_block_refcount(self._h, block))

    def add_sequence(self, seq_id: int, tokens) -> int:
        """Returns how many leading prompt tokens are already cached."""
        arr = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        cached = ctypes.c_int32(0)
        rc = self._lib.pa_bm_add_sequence(self._h, seq_id, arr.ctypes.data_as(ctypes.c_void_p),
                                          len(arr), ctypes.byref(cached))
        _ok(rc, "pa_bm_add_sequence")
        return int(cached.value)

    def append_token(self, seq_id: int, token: int = 0):
        """Returns (slot, (cow_src, cow_dst) or None)."""
        slot, src, dst = ctypes.c_int64(0), ctypes.c_int32(0), ctypes.c_int32(0)
        rc = self._lib.pa_bm_append_token(self._h, seq_id, token, ctypes.byref(slot),
                                          ctypes.byref(src), ctypes.byref(dst))
        _ok(rc, "pa_bm_append_token")
        return int(slot.value), (None if src.value < 0 else (int(src.value), int(dst.value)))

    def append_tokens(self, seq_ids, tokens):
        """One token for each listed sequence in one call. Returns (slots int64 [n],
        copy-on-write pairs int32 [k, 2] to apply before the append)."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        if toks.shape != ids.shape or ids.ndim != 1:
            raise BlockManagerError(ERR_INVALID, "pa_bm_append_tokens")
        n = len(ids)
        slots = np.empty(n, dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int32)
        k = ctypes.c_int32(0)
        rc = self._lib.pa_bm_append_tokens(self._h, ids.ctypes.data, toks.ctypes.data, n,
                                           slots.ctypes.data, pairs.ctypes.data, ctypes.byref(k))
        _ok(rc, "pa_bm_append_tokens")
        return slots, pairs[:k.value].copy()

    def fork(self, parent_id: int, child_id: int):
        _ok(self._lib.pa_bm_fork(self._h, parent_id, child_id), "pa_bm_fork")

    def free_sequence(self, seq_id: int):
        _ok(self._lib.pa_bm_free_sequence(self._h, seq_id), "pa_bm_free_sequence")

    def release_before(self, seq_id: int, position: int):
        _ok(self._lib.pa_bm_release_before(self._h, seq_id, position), "pa_bm_release_before")

    def release_window(self, seq_ids, window: int):
        """release_before(seq, length - window) for every listed sequence."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        _ok(self._lib.pa_bm_release_window(self._h, ids.ctypes.data, len(ids), window),
            "pa_bm_release_window")

    def length(self, seq_id: int) -> int:
        n = self._lib.pa_bm_sequence_length(self._h, seq_id)
        if n < 0:
            raise BlockManagerError(n, "pa_bm_sequence_length")
        return int(n)

    def slots(self, seq_id: int, first: int, count: int) -> np.ndarray:
        out = np.zeros(count, dtype=np.int64)
        _ok(self._lib.pa_bm_slots(self._h, seq_id, first, count,
                                  out.ctypes.data_as(ctypes.c_void_p)), "pa_bm_slots")
        return out

    def block_tables(self, seq_ids, max_blocks_per_seq: int):
        """Returns (block_tables int32 [n, max_blocks], context_lens int32 [n])."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        tables = np.zeros((len(ids), max_blocks_per_seq), dtype=np.int32)
        lens = np.zeros(len(ids), dtype=np.int32)
        rc = self._lib.pa_bm_block_tables(self._h, ids.ctypes.data_as(ctypes.c_void_p), len(ids),
                                          max_blocks_per_seq,
                                          tables.ctypes.data_as(ctypes.c_void_p),
                                          lens.ctypes.data_as(ctypes.c_void_p))
        _ok(rc, "pa_bm_block_tables")
        return tables, lens

    def block_tables_update(self, seq_ids, tables: np.ndarray, lens: np.ndarray,
                            row_versions: np.ndarray) -> int:
        """Rewrites, in place, the rows of `tables` (int32 [n, max_blocks]) whose block list
        changed since they were last written; writes every entry of `lens` (int32 [n]);
        `row_versions` (uint64 [n], zeros at first) tracks what each row holds. Returns the
        number of rows rewritten."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        n = len(ids)
        for a, dt, shape in ((tables, np.int32, None), (lens, np.int32, (n,)),
                             (row_versions, np.uint64, (n,))):
            if a.dtype != dt or not a.flags.c_contiguous or (shape and a.shape != shape):
                raise BlockManagerError(ERR_INVALID, "pa_bm_block_tables_update")
        if tables.ndim != 2 or tables.shape[0] != n:
            raise BlockManagerError(ERR_INVALID, "pa_bm_block_tables_update")
        written = ctypes.c_int32(0)
        rc = self._lib.pa_bm_block_tables_update(
            self._h, ids.ctypes.data_as(ctypes.c_void_p), n, tables.shape[1],
            tables.ctypes.data_as(ctypes.c_void_p), lens.ctypes.data_as(ctypes.c_void_p),
            row_versions.ctypes.data_as(ctypes.c_void_p), ctypes.byref(written))
        _ok(rc, "pa_bm_block_tables_update")
        return int(written.value)
