"""Seeded synthetic inputs for the paged-decode hot path.

This module draws inputs only: lengths, physical block placement, block
tables, slot mappings, copy pairs and N(0,1) tensor values rounded to their
storage type. It computes none of the method's arithmetic (no attention, no
quantisation, no copies) and imports neither the CUDA library nor the oracle,
so both sides can be fed from it.

Five workload families follow the shapes the KV-cache pages discuss (a tiny
MHA layer, a Llama-2-7B-shaped layer, a Llama-2-70B-shaped GQA layer with a
2000-token shared system prompt, a 128K-token long context, and an FP8 cache
with beam-search forks); every size can be overridden for small parity cases.

Conventions:
  * 16-bit tensors are returned as ``uint16`` bit patterns, E4M3 as ``uint8``.
  * ``context_lens[b]`` is the decode length of sequence b and includes the
    token appended in the same step (it sits at position ``L - 1``).
  * Cache layout is ``[num_blocks, block_size, num_kv_heads, head_dim]``; the
    token at logical position j of sequence b lives in physical block
    ``block_tables[b, j // block_size]`` at row ``j % block_size``.
  * For 16-bit caches the whole pool (used and unused slots) is drawn up
    front. For an E4M3 cache the history tokens are drawn in fp16 and listed
    with their slots (``fill_*``), so that each side quantises them itself.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 410


@dataclass
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    io_dtype: str       # dtype of q, new k/v and the output: "f16" | "bf16"
    cache_dtype: str    # "f16" | "bf16" | "e4m3"
    scale: np.float32
    q: np.ndarray            # uint16 [B, Hq, D]
    k_new: np.ndarray        # uint16 [B, Hkv, D]
    v_new: np.ndarray        # uint16 [B, Hkv, D]
    slot_mapping: np.ndarray  # int64 [B]
    block_tables: np.ndarray  # int32 [B, MB]
    context_lens: np.ndarray  # int32 [B]
    copy_pairs: np.ndarray    # int32 [n, 2] (src, dst), applied before the append
    k_pool: np.ndarray | None = None   # uint16 [NB, BS, Hkv, D] (16-bit caches)
    v_pool: np.ndarray | None = None
    fill_k: np.ndarray | None = None   # uint16 [F, Hkv, D] history (E4M3 caches)
    fill_v: np.ndarray | None = None
    fill_slots: np.ndarray | None = None  # int64 [F]
    k_scale: np.ndarray | None = None  # float32 [Hkv, D] (E4M3 caches)
    v_scale: np.ndarray | None = None
    k_inv_scale: np.ndarray | None = None
    v_inv_scale: np.ndarray | None = None
    meta: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context(self) -> int:
        return int(self.context_lens.max()) if self.batch else 0


# ---- value drawing -----------------------------------------------------------

def round_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 -> storage bit pattern, rounding to nearest even."""
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        import torch
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16)
    raise ValueError(dtype)


def normal_bits(rng: np.random.Generator, shape, dtype: str, chunk: int = 1 << 22) -> np.ndarray:
    """N(0,1) drawn in float32, rounded to ``dtype``. One 64-bit draw from
    ``rng`` seeds the whole array; chunk i comes from
    ``default_rng([that seed, i])``, so the values do not depend on how many
    host threads fill the chunks."""
    n = int(np.prod(shape))
    base = int(rng.integers(0, 2 ** 63 - 1))
    out = np.empty(n, dtype=np.uint16)

    def fill(i):
        s = i * chunk
        m = min(chunk, n - s)
        r = np.random.default_rng([base, i])
        out[s:s + m] = round_bits(r.standard_normal(m, dtype=np.float32), dtype)

    nchunks = -(-n // chunk)
    if nchunks <= 1:
        for i in range(nchunks):
            fill(i)
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(min(32, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


def bits_to_float32(bits: np.ndarray, dtype: str) -> np.ndarray:
    """storage bit pattern -> float32 (exact for f16 and bf16)."""
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float32)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << 16).view(np.float32)
    raise ValueError(dtype)


# ---- block placement --------------------------------------------------------

class _Placer:
    """Hands out physical block ids in the order of a seeded permutation."""

    def __init__(self, rng, num_blocks):
        self.perm = rng.permutation(num_blocks).astype(np.int32)
        self.next = 0

    def take(self, n: int) -> list[int]:
        if self.next + n > len(self.perm):
            raise ValueError("pool too small")
        ids = self.perm[self.next:self.next + n].tolist()
        self.next += n
        return ids


def _pool_size(blocks_needed: int, headroom: float) -> int:
    return int(math.ceil(blocks_needed * (1.0 + headroom)))


def _tables(block_lists, min_width=1) -> np.ndarray:
    mb = max([len(b) for b in block_lists] + [min_width])
    t = np.zeros((len(block_lists), mb), dtype=np.int32)
    for i, b in enumerate(block_lists):
        t[i, :len(b)] = b
    return t


def _slot(blocks, pos, bs) -> int:
    return int(blocks[pos // bs]) * bs + pos % bs


def _finish_16bit(name, rng, *, B, Hq, Hkv, D, BS, NB, dtype, lens, block_lists, meta,
                  draw_pool=True):
    k_pool = normal_bits(rng, (NB, BS, Hkv, D), dtype) if draw_pool else None
    v_pool = normal_bits(rng, (NB, BS, Hkv, D), dtype) if draw_pool else None
    q = normal_bits(rng, (B, Hq, D), dtype)
    k_new = normal_bits(rng, (B, Hkv, D), dtype)
    v_new = normal_bits(rng, (B, Hkv, D), dtype)
    slots = np.array([_slot(block_lists[b], lens[b] - 1, BS) if lens[b] > 0 else -1
                      for b in range(B)], dtype=np.int64)
    return Workload(
        name=name, batch=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=BS,
        num_blocks=NB, io_dtype=dtype, cache_dtype=dtype,
        scale=np.float32(1.0 / math.sqrt(D)), q=q, k_new=k_new, v_new=v_new,
        slot_mapping=slots, block_tables=_tables(block_lists),
        context_lens=np.asarray(lens, dtype=np.int32), copy_pairs=np.zeros((0, 2), np.int32),
        k_pool=k_pool, v_pool=v_pool, meta=meta)


# ---- the five families ----------------------------------------------------------

def tiny_mha(batch=4, num_heads=8, head_dim=64, block_size=16, pool_blocks=64,
             max_history=200, seed=SEED_BASE + 1) -> Workload:
    """Tiny MHA layer: history length drawn uniformly from 1..max_history, one
    token appended per sequence, blocks from a seeded permutation of a
    ``pool_blocks`` pool."""
    rng = np.random.default_rng(seed)
    hist = rng.integers(1, max_history + 1, size=batch)
    lens = (hist + 1).astype(np.int64)
    placer = _Placer(rng, pool_blocks)
    block_lists = [placer.take(-(-int(L) // block_size)) for L in lens]
    return _finish_16bit("tiny_mha", rng, B=batch, Hq=num_heads, Hkv=num_heads, D=head_dim,
                         BS=block_size, NB=pool_blocks, dtype="f16", lens=lens,
                         block_lists=block_lists, meta={"history": hist.tolist()})


def llama2_7b(batch=64, min_len=512, max_len=4096, block_size=16, headroom=0.10,
              seed=SEED_BASE + 2, dtype="f16") -> Workload:
    """Llama-2-7B-shaped layer: 32 q heads = 32 KV heads, head_dim 128,
    decode lengths uniform in [min_len, max_len], pool = blocks needed + 10%,
    random block assignment."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(min_len, max_len + 1, size=batch).astype(np.int64)
    need = int(sum(-(-int(L) // block_size) for L in lens))
    NB = _pool_size(need, headroom)
    placer = _Placer(rng, NB)
    block_lists = [placer.take(-(-int(L) // block_size)) for L in lens]
    return _finish_16bit("llama2_7b", rng, B=batch, Hq=32, Hkv=32, D=128, BS=block_size,
                         NB=NB, dtype=dtype, lens=lens, block_lists=block_lists, meta={})


def llama2_70b_prefix(batch=128, prefix_len=2000, max_suffix=2048, block_size=16,
                      headroom=0.10, seed=SEED_BASE + 3) -> Workload:
    """Llama-2-70B-shaped GQA layer (64 q heads / 8 KV heads, head_dim 128,
    bf16) whose sequences all reference the same physical blocks for a shared
    ``prefix_len``-token prompt, followed by a private suffix of s ~ U{0..
    max_suffix} tokens and the token appended this step (decode length
    prefix_len + s + 1). The prefix must fill whole blocks so that no
    sequence ever writes into a shared block."""
    if prefix_len % block_size:
        raise ValueError("the shared prefix must end on a block boundary")
    rng = np.random.default_rng(seed)
    suffix = rng.integers(0, max_suffix + 1, size=batch).astype(np.int64)
    lens = prefix_len + suffix + 1
    npre = prefix_len // block_size
    private = [-(-int(L) // block_size) - npre for L in lens]
    NB = _pool_size(npre + sum(private), headroom)
    placer = _Placer(rng, NB)
    prefix_blocks = placer.take(npre)
    block_lists = [prefix_blocks + placer.take(p) for p in private]
    return _finish_16bit("llama2_70b_prefix", rng, B=batch, Hq=64, Hkv=8, D=128,
                         BS=block_size, NB=NB, dtype="bf16", lens=lens,
                         block_lists=block_lists,
                         meta={"prefix_len": prefix_len, "prefix_blocks": prefix_blocks,
                               "shared_prefix_blocks": npre, "refcount": batch})


def long_context(batch=1, context_len=131072, block_size=16, headroom=0.10,
                 seed=SEED_BASE + 4) -> Workload:
    """Long-context GQA layer (64 q heads / 8 KV heads, head_dim 128, bf16):
    every sequence has ``context_len`` tokens in randomly scattered blocks."""
    rng = np.random.default_rng(seed)
    lens = np.full(batch, context_len, dtype=np.int64)
    per = -(-context_len // block_size)
    NB = _pool_size(per * batch, headroom)
    placer = _Placer(rng, NB)
    block_lists = [placer.take(per) for _ in range(batch)]
    return _finish_16bit("long_context", rng, B=batch, Hq=64, Hkv=8, D=128, BS=block_size,
                         NB=NB, dtype="bf16", lens=lens, block_lists=block_lists, meta={})


def fp8_beams(batch=256, block_size=16, beam_groups=16, beam_width=4, median_len=600,
              sigma=1.0, min_len=16, max_len=8192, headroom=0.10, num_q_heads=32,
              num_kv_heads=8, head_dim=128, seed=None) -> Workload:
    """GQA layer (32 q / 8 KV heads, head_dim 128) with an FP8-E4M3 cache and
    per-(kv_head, channel) fp32 scales from max-abs calibration; q, new k/v
    and the output are fp16. Decode lengths are lognormal (median
    ``median_len``, log-sigma ``sigma``) clipped to [min_len, max_len]. The
    first ``beam_groups * beam_width`` sequences form beam groups: the beams
    of a group share the prompt's blocks; when the prompt ends inside a
    block, beam 0 keeps that block and every other beam gets a fresh block
    plus a (src, dst) copy pair, to be applied before the append."""
    if seed is None:
        seed = SEED_BASE + 5 + block_size
    rng = np.random.default_rng(seed)
    BS = block_size
    n_beam = beam_groups * beam_width
    if n_beam > batch:
        raise ValueError("more beams than sequences")

    def draw(n):
        x = np.exp(rng.normal(math.log(median_len), sigma, size=n))
        return np.clip(np.rint(x), min_len, max_len).astype(np.int64)

    group_lens = draw(beam_groups)
    solo_lens = draw(batch - n_beam)
    lens = np.concatenate([np.repeat(group_lens, beam_width), solo_lens])

    # blocks needed: shared full prompt blocks once per group, one last block
    # per beam (when the prompt ends inside a block the parent's counts as
    # beam 0's), private blocks for the independent sequences
    need = 0
    for L in group_lens:
        need += (L - 1) // BS + beam_width
    for L in solo_lens:
        need += -(-int(L) // BS)
    NB = _pool_size(int(need), headroom)
    placer = _Placer(rng, NB)

    block_lists, pairs = [], []
    hist_slots = []  # slots of history tokens (position < L - 1), one entry per token
    for g, L in enumerate(group_lens):
        L = int(L)
        prompt = L - 1
        full = placer.take(prompt // BS)
        partial = prompt % BS
        if partial:
            parent_last = placer.take(1)[0]
            lasts = [parent_last] + placer.take(beam_width - 1)
            pairs += [(parent_last, d) for d in lasts[1:]]
            prompt_blocks = full + [parent_last]
        else:
            lasts = placer.take(beam_width)
            prompt_blocks = full
        for j in range(prompt):
            hist_slots.append(_slot(prompt_blocks, j, BS))
        for w in range(beam_width):
            block_lists.append(full + [lasts[w]])
    for L in solo_lens:
        L = int(L)
        blocks = placer.take(-(-L // BS))
        for j in range(L - 1):
            hist_slots.append(_slot(blocks, j, BS))
        block_lists.append(blocks)

    Hq, Hkv, D = num_q_heads, num_kv_heads, head_dim
    F = len(hist_slots)
    fill_k = normal_bits(rng, (F, Hkv, D), "f16")
    fill_v = normal_bits(rng, (F, Hkv, D), "f16")
    q = normal_bits(rng, (batch, Hq, D), "f16")
    k_new = normal_bits(rng, (batch, Hkv, D), "f16")
    v_new = normal_bits(rng, (batch, Hkv, D), "f16")
    slots = np.array([_slot(block_lists[b], int(lens[b]) - 1, BS) for b in range(batch)],
                     dtype=np.int64)

    # max-abs calibration over every token the cache will hold
    def calib(fill, new):
        m = np.maximum(np.abs(bits_to_float32(fill, "f16")).max(axis=0, initial=0.0),
                       np.abs(bits_to_float32(new, "f16")).max(axis=0, initial=0.0))
        s = (m / np.float32(448.0)).astype(np.float32)
        s[s == 0] = np.float32(1.0)
        return s, (np.float32(1.0) / s).astype(np.float32)

    k_scale, k_inv = calib(fill_k, k_new)
    v_scale, v_inv = calib(fill_v, v_new)
    return Workload(
        name=f"fp8_beams_bs{BS}", batch=batch, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
        block_size=BS, num_blocks=NB, io_dtype="f16", cache_dtype="e4m3",
        scale=np.float32(1.0 / math.sqrt(D)), q=q, k_new=k_new, v_new=v_new,
        slot_mapping=slots, block_tables=_tables(block_lists),
        context_lens=lens.astype(np.int32),
        copy_pairs=np.asarray(pairs, dtype=np.int32).reshape(-1, 2),
        fill_k=fill_k, fill_v=fill_v, fill_slots=np.asarray(hist_slots, dtype=np.int64),
        k_scale=k_scale, v_scale=v_scale, k_inv_scale=k_inv, v_inv_scale=v_inv,
        meta={"beam_groups": beam_groups, "beam_width": beam_width,
              "group_lens": group_lens.tolist()})


def custom(lens, num_q_heads=8, num_kv_heads=8, head_dim=64, block_size=16, dtype="f16",
           headroom=0.25, seed=SEED_BASE) -> Workload:
    """Any shape, for edge cases: decode lengths ``lens`` (0 allowed: such a
    sequence appends nothing), private blocks from a seeded permutation of a
    pool with ``headroom`` spare blocks, 16-bit cache."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int64)
    need = int(sum(-(-int(L) // block_size) for L in lens))
    NB = max(_pool_size(need, headroom), 1)
    placer = _Placer(rng, NB)
    block_lists = [placer.take(-(-int(L) // block_size)) for L in lens]
    return _finish_16bit("custom", rng, B=len(lens), Hq=num_q_heads, Hkv=num_kv_heads,
                         D=head_dim, BS=block_size, NB=NB, dtype=dtype, lens=lens,
                         block_lists=block_lists, meta={})


def custom_shared_prefix(prefix_len, suffix_lens, num_q_heads=8, num_kv_heads=2, head_dim=64,
                         block_size=16, dtype="f16", headroom=0.25, seed=SEED_BASE + 7):
    """Sequences that all reference the same physical blocks for their first
    ``prefix_len`` tokens (a multiple of the block size), followed by
    ``suffix_lens[b]`` private tokens; the last suffix token is the one
    appended this step. A suffix of 0 appends nothing (slot -1): such a
    sequence ends exactly at the prefix."""
    if prefix_len % block_size:
        raise ValueError("the shared prefix must end on a block boundary")
    rng = np.random.default_rng(seed)
    suffix = np.asarray(suffix_lens, dtype=np.int64)
    lens = prefix_len + suffix
    npre = prefix_len // block_size
    private = [-(-int(L) // block_size) - npre for L in lens]
    NB = max(_pool_size(npre + sum(private), headroom), 1)
    placer = _Placer(rng, NB)
    prefix_blocks = placer.take(npre)
    block_lists = [prefix_blocks + placer.take(p) for p in private]
    w = _finish_16bit("custom_shared_prefix", rng, B=len(lens), Hq=num_q_heads,
                      Hkv=num_kv_heads, D=head_dim, BS=block_size, NB=NB, dtype=dtype, lens=lens,
                      block_lists=block_lists,
                      meta={"prefix_len": prefix_len, "prefix_blocks": prefix_blocks,
                            "shared_prefix_blocks": npre})
    w.slot_mapping[suffix == 0] = -1
    return w


FAMILIES = {
    "custom": custom,
    "custom_shared_prefix": custom_shared_prefix,
    "tiny_mha": tiny_mha,
    "llama2_7b": llama2_7b,
    "llama2_70b_prefix": llama2_70b_prefix,
    "long_context": long_context,
    "fp8_beams": fp8_beams,
}


def make(name: str, **overrides) -> Workload:
    return FAMILIES[name](**overrides)


def subset(w: Workload, seqs) -> Workload:
    """The same pool, restricted to the listed sequences (for sampled checks
    of large workloads and for sharding a batch across ranks)."""
    seqs = np.asarray(seqs, dtype=np.int64)
    import copy
    s = copy.copy(w)
    s.batch = len(seqs)
    s.q = w.q[seqs]
    s.k_new = w.k_new[seqs]
    s.v_new = w.v_new[seqs]
    s.slot_mapping = w.slot_mapping[seqs]
    s.block_tables = w.block_tables[seqs]
    s.context_lens = w.context_lens[seqs]
    keep = np.zeros(0, np.int32).reshape(0, 2)
    if len(w.copy_pairs):
        dsts = set(int(w.block_tables[b, (int(w.context_lens[b]) - 1) // w.block_size])
                   for b in seqs)
        keep = np.asarray([p for p in w.copy_pairs.tolist() if p[1] in dsts],
                          dtype=np.int32).reshape(-1, 2)
    s.copy_pairs = keep
    s.meta = dict(w.meta, subset=seqs.tolist())
    return s
