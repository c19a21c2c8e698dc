"""CPU checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad host-side arguments before touching the
GPU (every call below returns from its argument checks, so no device is
needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa_api.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return B.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names == sorted(B.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.pa_version() >= 100
    for s in range(6):
        assert lib.pa_status_string(s)
    assert B.pa_status_string(1) == "invalid argument"


def _desc(**kw):
    d = dict(num_blocks=8, block_size=16, num_kv_heads=2, head_dim=64, cache_dtype=B.PA_F16,
             k_scale=None, v_scale=None, k_inv_scale=None, v_inv_scale=None)
    d.update(kw)
    return B._CacheDesc(**d)


FAKE = 1 << 20  # a 16-byte-aligned non-null address; never dereferenced here


def test_copy_blocks_rejects_conflicting_pairs(lib):
    d = _desc()
    for pairs in ([[1, 2], [3, 2]],      # duplicate destination
                  [[1, 2], [2, 3]],      # destination is also a source
                  [[1, 8]],              # out of range
                  [[-1, 2]]):
        arr = np.asarray(pairs, np.int32)
        rc = lib.pa_copy_blocks(arr.ctypes.data_as(ctypes.c_void_p), len(arr), FAKE, FAKE,
                                ctypes.byref(d), None)
        assert rc == 1, pairs
    assert lib.pa_copy_blocks(None, 0, FAKE, FAKE, ctypes.byref(d), None) == 0


@pytest.mark.parametrize("field,value,status", [
    ("block_size", 24, 1), ("block_size", 512, 1), ("head_dim", 96, 2), ("cache_dtype", 7, 1),
    ("num_blocks", 0, 1), ("num_kv_heads", 0, 1),
])
def test_bad_cache_descriptors(lib, field, value, status):
    d = _desc(**{field: value})
    rc = lib.pa_decode(FAKE, 0, 1, 2, FAKE, FAKE, ctypes.byref(d), FAKE, 4, FAKE, 64, 0.1, FAKE,
                       0, None, 0, None)
    assert rc == status


def test_decode_argument_checks(lib):
    d = _desc()
    call = lambda **kw: lib.pa_decode(*[kw.get(k, v) for k, v in [
        ("q", FAKE), ("q_dtype", 0), ("batch", 2), ("hq", 4), ("k", FAKE), ("v", FAKE),
        ("desc", ctypes.byref(d)), ("bt", FAKE), ("mb", 4), ("lens", FAKE), ("maxc", 64),
        ("scale", 0.1), ("out", FAKE), ("pt", 0), ("ws", None), ("wsb", 0), ("s", None)]])
    assert call(hq=3) == 1                    # not a multiple of num_kv_heads
    assert call(q_dtype=1) == 2               # bf16 query on an fp16 cache
    assert call(pt=24) == 1                   # partition not a multiple of 16
    assert call(q=FAKE + 4) == 1              # misaligned
    assert call(scale=float("nan")) == 1
    assert call(batch=0) == 0                 # nothing to do
    assert call(out=None) == 1
    # a split plan needs a workspace
    need = lib.pa_decode_workspace_size(2, 4, 5000, 64, ctypes.byref(d))
    assert need > 0
    assert call(maxc=5000, pt=64) == 4
    assert call(maxc=5000, pt=64, ws=FAKE + 16, wsb=need) == 4  # not 256-byte aligned
    assert call(maxc=5000, pt=64, ws=FAKE, wsb=need - 1) == 4
    # sizes whose split-K workspace would wrap around size_t are refused, not
    # sized modulo 2^64 (65535 sequences x 1048544 query heads x 2^27 partitions)
    big = dict(batch=65535, hq=2 * 524272, maxc=(1 << 31) - 1, pt=16)
    assert lib.pa_decode_workspace_size(big["batch"], big["hq"], big["maxc"], 16,
                                        ctypes.byref(d)) == 0
    assert call(**big, ws=FAKE, wsb=(1 << 64) - 1) == 2
    assert lib.pa_decode_shared_prefix_workspace_size(big["batch"], big["hq"], big["maxc"], 2,
                                                      16, ctypes.byref(d)) == 0
    # E4M3 caches need scales
    d8 = _desc(cache_dtype=B.PA_E4M3)
    assert lib.pa_decode(FAKE, 0, 1, 2, FAKE, FAKE, ctypes.byref(d8), FAKE, 4, FAKE, 64, 0.1,
                         FAKE, 0, None, 0, None) == 1


def test_shared_prefix_argument_checks(lib):
    d = _desc()
    call = lambda **kw: lib.pa_decode_shared_prefix(*[kw.get(k, v) for k, v in [
        ("q", FAKE), ("q_dtype", 0), ("batch", 2), ("hq", 4), ("k", FAKE), ("v", FAKE),
        ("desc", ctypes.byref(d)), ("bt", FAKE), ("mb", 4), ("lens", FAKE), ("maxc", 64),
        ("pb", 2), ("scale", 0.1), ("out", FAKE), ("pt", 0), ("ws", None), ("wsb", 0),
        ("s", None)]])
    assert call(pb=5) == 1               # more shared blocks than table columns
    assert call(pb=-1) == 1
    assert call(pb=4, maxc=60) == 1      # prefix longer than max_context
    assert call() == 4                   # a cascade always needs a workspace
    need = lib.pa_decode_shared_prefix_workspace_size(2, 4, 64, 2, 0, ctypes.byref(d))
    assert need > 0
    assert call(ws=FAKE, wsb=need - 1) == 4
    assert call(batch=0) == 0
    # no shared blocks: the plain decode's workspace
    assert (lib.pa_decode_shared_prefix_workspace_size(2, 4, 5000, 0, 64, ctypes.byref(d)) ==
            lib.pa_decode_workspace_size(2, 4, 5000, 64, ctypes.byref(d)))
    # partials: prefix chunks + suffix partitions. 16-bit caches (tcgen05
    # prefix kernel): 64-token steps split into chunks so that 128-row tiles
    # x KV heads x chunks is about 2 CTAs per SM (296), at most 64 chunks.
    wsz = lambda parts: (-(-(3 * 4 * parts * 64 * 4) // 256) * 256 +
                         -(-(3 * 4 * parts * 8) // 256) * 256)
    ws = lib.pa_decode_shared_prefix_workspace_size(3, 4, 2048 + 256, 128, 64, ctypes.byref(d))
    assert ws == wsz(32 + 4)    # 2 tiles -> 148 wanted, 32 steps -> 32 chunks of 64 tokens
    ws = lib.pa_decode_shared_prefix_workspace_size(3, 4, 8192 + 64, 512, 64, ctypes.byref(d))
    assert ws == wsz(64 + 1)    # 128 steps, capped at 64 chunks of 128 tokens
    # E4M3 caches (mma.sync prefix CTAs): chunks of up to 512 tokens
    d8 = _desc(cache_dtype=B.PA_E4M3, k_scale=FAKE, v_scale=FAKE)
    ws = lib.pa_decode_shared_prefix_workspace_size(3, 4, 2048 + 256, 128, 64, ctypes.byref(d8))
    assert ws == wsz(4 + 4)
    ws = lib.pa_decode_shared_prefix_workspace_size(3, 4, 8192 + 64, 512, 64, ctypes.byref(d8))
    assert ws == wsz(16 + 1)


def test_append_argument_checks(lib):
    d = _desc()
    assert lib.pa_append_kv(FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, ctypes.byref(d), None) == 2
    assert lib.pa_append_kv(FAKE, FAKE, 2, 4, FAKE, FAKE, FAKE, ctypes.byref(d), None) == 1
    assert lib.pa_append_kv(FAKE, FAKE, 0, -1, FAKE, FAKE, FAKE, ctypes.byref(d), None) == 1
    assert lib.pa_append_kv(None, None, 0, 0, None, None, None, ctypes.byref(d), None) == 0
    d8 = _desc(cache_dtype=B.PA_E4M3)
    assert lib.pa_append_kv(FAKE, FAKE, 0, 4, FAKE, FAKE, FAKE, ctypes.byref(d8), None) == 1


def test_workspace_plan(lib):
    d = _desc(num_kv_heads=8, head_dim=128)
    # one partition covers the context: no workspace
    assert lib.pa_decode_workspace_size(4, 64, 100, 512, ctypes.byref(d)) == 0
    # split: partial outputs (fp32, head_dim) + (max, sum) per partition, then
    # the work list (a 256-byte counter section and one 8-byte item per
    # partition a sequence can have), 256-byte sections
    ws = lib.pa_decode_workspace_size(4, 64, 131072, 512, ctypes.byref(d))
    parts = 131072 // 512
    o = 4 * 64 * parts * 128 * 4
    ml = 4 * 64 * parts * 8
    items = 4 * parts * 8
    assert ws == -(-o // 256) * 256 + -(-ml // 256) * 256 + 256 + -(-items // 256) * 256
    # automatic partition: 128 KB of K rows per KV head (512 tokens at fp16 and
    # head_dim 128, 1024 at head_dim 64 or E4M3), halved while the grid is
    # under two CTAs per SM
    d32 = _desc(num_kv_heads=32, head_dim=128)
    assert lib.pa_decode_partition_tokens(64, 4096, ctypes.byref(d32)) == 512
    assert lib.pa_decode_partition_tokens(64, 4096, ctypes.byref(_desc(num_kv_heads=32))) == 1024
    d8 = _desc(num_kv_heads=8, head_dim=128, cache_dtype=B.PA_E4M3)
    assert lib.pa_decode_partition_tokens(256, 8192, ctypes.byref(d8)) == 1024
    # (8 rows: halved to 64 tokens = 512 CTAs, then one whole wave of 444:
    # 80-token partitions, 416 CTAs)
    assert lib.pa_decode_partition_tokens(1, 4096, ctypes.byref(d)) == 80
    assert lib.pa_decode_partition_tokens(1, 100, ctypes.byref(d)) == 64


def test_small_batches_split_into_whole_waves(lib):
    """With fewer (sequence, KV head) pairs than one wave of decode CTAs (3 per
    SM on 148 SMs), the automatic partition is lengthened so that the CTAs
    fill whole waves: for several sequences the shortest multiple of 16
    tokens that keeps the 512-token plan's whole waves, for a single sequence
    the fewest waves whose partitions stay within 8192 tokens."""
    waves_of = 3 * 148
    d = _desc(num_kv_heads=8, head_dim=128, cache_dtype=B.PA_BF16)
    for batch, ctx, want in ((4, 131072, 528), (2, 20000, 752)):
        pt = lib.pa_decode_partition_tokens(batch, ctx, ctypes.byref(d))
        assert pt == want, (batch, ctx, pt)
        ctas = batch * 8 * -(-ctx // pt)
        full = batch * 8 * -(-ctx // 512) // waves_of  # whole waves of the 512-token plan
        assert ctas <= full * waves_of and pt % 16 == 0
        # 16 tokens shorter would need one more (partial) wave
        assert batch * 8 * -(-ctx // (pt - 16)) > full * waves_of
    # one sequence: a single wave of 440 CTAs (55 partitions of 2384 tokens)...
    pt = lib.pa_decode_partition_tokens(1, 131072, ctypes.byref(d))
    assert pt == 2384 and 8 * -(-131072 // pt) <= waves_of
    assert 8 * -(-131072 // (pt - 16)) > waves_of
    # ... or, when one wave would need partitions over 8192 tokens, the fewest
    # whole waves that do not (2^20 tokens: 3 waves of 166 partitions)
    ctx = 1 << 20
    pt = lib.pa_decode_partition_tokens(1, ctx, ctypes.byref(d))
    def within(w):  # the partition that fills w whole waves, rounded up to 16 tokens
        per = -(-ctx // (w * waves_of // 8))
        return (per + 15) // 16 * 16
    assert within(1) > 8192 and within(2) > 8192 and pt == within(3) <= 8192
    assert 8 * -(-ctx // pt) <= 3 * waves_of
    # a batch that fills the GPU by itself keeps the byte rule
    d32 = _desc(num_kv_heads=32, head_dim=128)
    assert lib.pa_decode_partition_tokens(64, 4096, ctypes.byref(d32)) == 512
    assert lib.pa_decode_partition_tokens(14, 8192, ctypes.byref(d32)) == 512  # 448 rows


def test_static_workspace_checks_arguments_before_its_size_rule(lib):
    """The no-allocation decode reports an invalid call exactly as pa_decode
    does, even when the plan of the call would also exceed its fixed array;
    only a valid call whose plan needs more than the array gets
    PA_ERR_WORKSPACE."""
    d = _desc(num_kv_heads=8, head_dim=128)
    order = [("q", FAKE), ("q_dtype", 0), ("batch", 8), ("hq", 64), ("k", FAKE), ("v", FAKE),
             ("desc", ctypes.byref(d)), ("bt", FAKE), ("mb", 8192), ("lens", FAKE),
             ("maxc", 131072), ("scale", 0.1), ("out", FAKE), ("pt", 0)]
    static = lambda **kw: lib.pa_decode_static_workspace(
        *[kw.get(k, v) for k, v in order], None)
    plain = lambda **kw: lib.pa_decode(*[kw.get(k, v) for k, v in order], None, 0, None)
    # 8 sequences x 64 heads x 249 partitions of 528 tokens: 66 MB of partials
    assert lib.pa_decode_workspace_size(8, 64, 131072, 0, ctypes.byref(d)) > 32 << 20
    for bad, status in ((dict(pt=17), 1), (dict(hq=60), 1), (dict(q=None), 1),
                        (dict(out=FAKE + 8), 1), (dict(scale=float("inf")), 1),
                        (dict(q_dtype=1), 2), (dict(mb=0), 1), (dict(batch=0), 0)):
        assert static(**bad) == status, bad
        assert plain(**bad) == status, bad
    assert static() == 4                      # valid, but the plan needs more than 32 MiB


def test_append_decode_argument_checks(lib):
    d = _desc()
    call = lambda desc=d, **kw: lib.pa_append_decode(*[kw.get(k, v) for k, v in [
        ("q", FAKE), ("k", FAKE), ("v", FAKE), ("dtype", 0), ("batch", 2), ("hq", 4),
        ("slots", FAKE), ("kc", FAKE), ("vc", FAKE), ("desc", ctypes.byref(desc)), ("bt", FAKE),
        ("mb", 4), ("lens", FAKE), ("maxc", 64), ("scale", 0.1), ("out", FAKE), ("pt", 0),
        ("ws", None), ("wsb", 0), ("s", None)]])
    assert call(k=None) == 1                  # the new token's K is required
    assert call(slots=None) == 1
    assert call(v=FAKE + 8) == 1              # misaligned
    assert call(dtype=1) == 2                 # bf16 input on an fp16 cache
    assert call(hq=3) == 1
    assert call(batch=0) == 0                 # nothing to do
    need = lib.pa_decode_workspace_size(2, 4, 5000, 64, ctypes.byref(d))
    assert call(maxc=5000, pt=64) == 4        # same workspace rule as pa_decode
    assert call(maxc=5000, pt=64, ws=FAKE, wsb=need - 1) == 4
    # an E4M3 cache needs the inverse scales to quantise the new token
    d8 = _desc(cache_dtype=B.PA_E4M3, k_scale=FAKE, v_scale=FAKE)
    assert call(desc=d8) == 1
    d8 = _desc(cache_dtype=B.PA_E4M3, k_scale=FAKE, v_scale=FAKE, k_inv_scale=FAKE,
               v_inv_scale=FAKE + 4)
    assert call(desc=d8) == 1


def test_copy_blocks_layers_argument_checks(lib):
    d = _desc()
    arr = np.asarray([[1, 2], [3, 4]], np.int32)
    ptrs = lambda *xs: (ctypes.c_void_p * len(xs))(*xs)
    call = lambda ks, vs, n, pairs=arr: lib.pa_copy_blocks_layers(
        pairs.ctypes.data_as(ctypes.c_void_p), len(pairs), ks, vs, n, ctypes.byref(d), None)
    assert call(ptrs(FAKE, None), ptrs(FAKE, FAKE), 2) == 1        # a null layer
    assert call(ptrs(FAKE, FAKE + 8), ptrs(FAKE, FAKE), 2) == 1    # misaligned layer
    assert call(ptrs(FAKE), ptrs(FAKE), -1) == 1
    assert call(ptrs(FAKE), ptrs(FAKE), 0) == 0                    # no layers: no-op
    assert call(None, None, 2) == 1
    bad = np.asarray([[1, 2], [2, 5]], np.int32)                   # destination is a source
    assert call(ptrs(FAKE, FAKE), ptrs(FAKE, FAKE), 2, bad) == 1


def test_shared_prefix_partition_rule(lib):
    # 70B-shaped cascade (batch 128, 64 / 8 heads, 2000-token prefix, suffixes
    # up to 2049): four times the plain rule's 512 tokens; E4M3 keeps the plain rule
    d = _desc(num_blocks=20000, num_kv_heads=8, head_dim=128, cache_dtype=B.PA_BF16)
    assert lib.pa_decode_partition_tokens(128, 2049, ctypes.byref(d)) == 512
    assert lib.pa_decode_shared_prefix_partition_tokens(128, 64, 4049, 125, ctypes.byref(d)) == 2048
    # 16 sequences (128 rows, under one wave): one whole wave of 688-token
    # partitions (384 CTAs); doubling that would leave < 2 CTAs per SM
    assert lib.pa_decode_partition_tokens(16, 2049, ctypes.byref(d)) == 688
    assert lib.pa_decode_shared_prefix_partition_tokens(16, 64, 4049, 125, ctypes.byref(d)) == 688
    assert (lib.pa_decode_shared_prefix_partition_tokens(128, 64, 4049, 0, ctypes.byref(d)) ==
            lib.pa_decode_partition_tokens(128, 4049, ctypes.byref(d)))
    # a small batch keeps the plain rule (doubling would leave < 2 CTAs per SM)
    small = lib.pa_decode_partition_tokens(2, 2049, ctypes.byref(d))
    assert lib.pa_decode_shared_prefix_partition_tokens(2, 64, 4049, 125, ctypes.byref(d)) == small
    d8 = _desc(num_blocks=20000, num_kv_heads=8, head_dim=128, cache_dtype=B.PA_E4M3,
               k_scale=FAKE, v_scale=FAKE)
    assert (lib.pa_decode_shared_prefix_partition_tokens(128, 64, 4049, 125, ctypes.byref(d8)) ==
            lib.pa_decode_partition_tokens(128, 2049, ctypes.byref(d8)))
    assert lib.pa_decode_shared_prefix_partition_tokens(0, 64, 4049, 125, ctypes.byref(d)) == 0


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "pa_api.h"
#include "pa_block_manager.h"

int main(void) {
  pa_cache_desc cd;
  memset(&cd, 0, sizeof cd);
  cd.num_blocks = 1024; cd.block_size = 16; cd.num_kv_heads = 8; cd.head_dim = 128;
  cd.cache_dtype = PA_BF16;
  size_t ws = pa_decode_workspace_size(4, 64, 131072, 0, &cd);
  int32_t pt = pa_decode_partition_tokens(4, 131072, &cd);
  /* a host-side check fails before anything reaches a GPU */
  pa_status bad = pa_decode(NULL, PA_BF16, 1, 64, NULL, NULL, &cd, NULL, 4, NULL, 64, 0.1f,
                            NULL, 0, NULL, 0, NULL);
  pa_block_manager* bm = pa_bm_create(64, 16, 1);
  int32_t toks[40], cached = -1, src = 0, dst = 0, tables[8], lens[2];
  int64_t slot = -1, ids[2] = {1, 2};
  int i, rc = 0;
  for (i = 0; i < 40; ++i) toks[i] = 1000 + i;
  rc |= pa_bm_add_sequence(bm, 1, toks, 40, &cached);
  rc |= pa_bm_add_sequence(bm, 2, toks, 40, &cached);
  rc |= pa_bm_append_token(bm, 2, 7, &slot, &src, &dst);
  rc |= pa_bm_block_tables(bm, ids, 2, 4, tables, lens);
  /* one token for both sequences in one call, then the incremental export */
  int64_t bslots[2];
  int32_t btoks[2] = {8, 9}, bpairs[4], npairs = -1, kept[8], klens[2], written = -1;
  uint64_t versions[2] = {0, 0};
  rc |= pa_bm_append_tokens(bm, ids, btoks, 2, bslots, bpairs, &npairs);
  rc |= pa_bm_block_tables_update(bm, ids, 2, 4, kept, klens, versions, &written);
  int64_t free_before = pa_bm_num_free_blocks(bm);
  rc |= pa_bm_release_window(bm, ids, 2, 8); /* 41 and 42 tokens: blocks 0 and 1 go */
  printf("%d|%s|%zu|%d|%d|%d|%d|%d|%d|%d|%d|%d|%d|%d|%d|%d\n", (int)pa_version(),
         pa_status_string(PA_ERR_WORKSPACE), ws, (int)pt, (int)bad, rc, (int)cached, (int)src,
         (int)lens[0], (int)lens[1], tables[0] == tables[4] && tables[1] == tables[5],
         (int)npairs, (int)written, (int)klens[0], (int)klens[1],
         (int)(pa_bm_num_free_blocks(bm) - free_before));
  pa_bm_destroy(bm);
  return 0;
}
"""


def test_headers_are_plain_c_and_the_library_links_from_c(lib, tmp_path):
    """Both headers compile as strict C99 with warnings as errors, and a C
    program linked against libpagedattn.so calls its host-side entry points
    (no GPU involved)."""
    import subprocess
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(B.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lpagedattn", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.strip()
    f = out.split("|")
    d = _desc(num_blocks=1024, block_size=16, num_kv_heads=8, head_dim=128,
              cache_dtype=B.PA_BF16)
    assert int(f[0]) == lib.pa_version()
    assert f[1] == "workspace missing or too small"
    assert int(f[2]) == lib.pa_decode_workspace_size(4, 64, 131072, 0, ctypes.byref(d)) > 0
    assert int(f[3]) == lib.pa_decode_partition_tokens(4, 131072, ctypes.byref(d)) == 528
    assert int(f[4]) == 1                         # PA_ERR_INVALID_ARG
    assert int(f[5]) == 0                         # every block-manager call succeeded
    assert int(f[6]) == 32                        # two full 16-token blocks reused
    assert int(f[7]) == -1                        # the partial block was private: no copy
    assert (int(f[8]), int(f[9])) == (40, 41)
    assert int(f[10]) == 1                        # both tables start with the same blocks
    assert int(f[11]) == 0                        # no shared partial block: no copies
    assert int(f[12]) == 2                        # first incremental export writes both rows
    assert (int(f[13]), int(f[14])) == (41, 42)
    # the two shared prompt blocks stay held by the prefix cache: nothing freed
    assert int(f[15]) == 0


def test_workspace_sizes_cover_every_partition_plan(lib):
    """The partition-length queries and the workspace-size queries come from
    one planner: over random shapes, the workspace each size query asks for
    holds exactly (plain, window) or at least (shared prefix: one or more
    prefix chunks besides) the partials the partition queries imply."""
    rng = np.random.default_rng(11)

    def need(batch, hq, parts, d):
        o, ml = batch * hq * parts * d * 4, batch * hq * parts * 8
        return -(-o // 256) * 256 + -(-ml // 256) * 256

    def need_list(batch, hq, parts, d):  # plain and window decodes: + the work list
        return need(batch, hq, parts, d) + 256 + -(-(batch * parts * 8) // 256) * 256

    for _ in range(400):
        hkv = int(rng.choice([1, 2, 8, 32]))
        hq = hkv * int(rng.choice([1, 2, 4, 8, 16]))
        d = int(rng.choice([64, 128]))
        bs = int(rng.choice([1, 8, 16, 64, 256]))
        dt = int(rng.choice([B.PA_F16, B.PA_BF16, B.PA_E4M3]))
        batch = int(rng.integers(1, 300))
        maxc = int(rng.integers(0, 200000))
        desc = ctypes.byref(_desc(num_kv_heads=hkv, head_dim=d, block_size=bs, cache_dtype=dt,
                                  num_blocks=1 << 20))
        pt = lib.pa_decode_partition_tokens(batch, maxc, desc)
        assert pt >= 64 and pt % 16 == 0
        parts = max(1, -(-maxc // pt))
        ws = lib.pa_decode_workspace_size(batch, hq, maxc, 0, desc)
        assert ws == (need_list(batch, hq, parts, d) if parts > 1 else 0)
        # sliding window: the plan spans at most window + 15 tokens
        window = int(rng.integers(1, 10000))
        span = min(maxc, window + 15)
        ptw = lib.pa_decode_partition_tokens(batch, span, desc)
        partsw = max(1, -(-span // ptw))
        wsw = lib.pa_decode_sliding_window_workspace_size(batch, hq, maxc, window, 0, desc)
        assert wsw == (need_list(batch, hq, partsw, d) if partsw > 1 else 0)
        # shared prefix: prefix chunks plus the suffix partitions
        pb = int(rng.integers(1, maxc // bs + 2))
        if pb * bs > maxc:
            continue
        pts = lib.pa_decode_shared_prefix_partition_tokens(batch, hq, maxc, pb, desc)
        assert pts >= 16 and pts % 16 == 0
        sparts = -(-(maxc - pb * bs) // pts)
        wss = lib.pa_decode_shared_prefix_workspace_size(batch, hq, maxc, pb, 0, desc)
        assert wss >= need(batch, hq, 1 + sparts, d)


def test_reproducible_results_switch(lib):
    # a process-wide host setting, read by each decode call; off at load
    prev = B.pa_set_deterministic(True)
    assert prev is False
    assert B.pa_set_deterministic(True) is True
    assert B.pa_set_deterministic(False) is True
    with B.deterministic():
        assert lib.pa_set_deterministic(1) == 1
    assert B.pa_set_deterministic(False) is False
