"""Context parallelism: the decode of sequences whose histories are split
across several GPUs, one process per GPU.

Each rank holds a block-aligned, contiguous slice of every sequence's
history in its own cache pool and block tables. A decode step is then
  1. pa_decode_partial on the rank's slice: per (sequence, query head) row
     the attention output over the slice's tokens, normalised, with the
     slice's score maximum and exponential sum (fp32, D + 2 floats a row);
  2. one all-gather of those pieces over the ranks (NCCL over NVLink on
     GPUs; any torch.distributed backend works);
  3. pa_merge_partials of the gathered pieces into the full output, on
     every rank.
The merge is the decode's own split-K merge applied across ranks, so the
result equals a single-GPU decode of the whole history up to rounding.
Attention at decode time does not depend on where a token sits, so each
slice is decoded as a history of its own.

`partial`, `merge` and `all_gather` default to the library and
torch.distributed; the host-side tests pass stand-ins so the slicing and
exchange run on CPU ranks.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import binding as B


def context_slices(context_lens, world: int, block_size: int) -> np.ndarray:
    """Token ranges of each rank: an int64 array [world, batch, 2] of
    (start, end), each sequence's blocks dealt out in contiguous runs as
    evenly as possible (the first ranks take one block more when the count
    does not divide), every start a multiple of block_size. A rank whose run
    is empty gets (L, L)."""
    lens = np.asarray(context_lens, dtype=np.int64)
    if world < 1 or block_size < 1:
        raise ValueError("world and block_size must be positive")
    out = np.zeros((world, lens.shape[0], 2), dtype=np.int64)
    for b, L in enumerate(lens):
        nblk = -(-int(L) // block_size)
        base, extra = divmod(nblk, world)
        blk = 0
        for r in range(world):
            n = base + (1 if r < extra else 0)
            start = min(blk * block_size, int(L))
            end = min((blk + n) * block_size, int(L))
            out[r, b] = (start, end)
            blk += n
    return out


def local_view(block_tables, context_lens, slices, rank: int, block_size: int):
    """The rank's block tables and lengths for its slices, cut from the full
    tables (host arrays; for callers that hold the whole tables, such as one
    process standing in for several ranks): row b lists the blocks of
    tokens [start, end) and has length end - start."""
    bt = np.asarray(block_tables)
    sl = np.asarray(slices)[rank]
    local = np.zeros_like(bt)
    lens = np.zeros(bt.shape[0], dtype=np.int32)
    for b, (s, e) in enumerate(sl):
        if e <= s:
            continue
        b0, b1 = int(s) // block_size, -(-int(e) // block_size)
        local[b, :b1 - b0] = bt[b, b0:b1]
        lens[b] = int(e - s)
    return local, lens


def _all_gather(dst, src, group):
    """dst[r] = rank r's src: one all-gather into the stacked tensor on NCCL,
    a list of views on backends without that form."""
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(dst, src, group=group)
    else:
        dist.all_gather(list(dst.unbind(0)), src, group=group)


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, cache: B.PagedCache,
           max_context: int, group=None, partition_tokens: int = 0, workspace=None, stream=None,
           partial=None, merge=None, all_gather=None):
    """One decode step of this rank's slice, exchanged and merged: `out`
    ([B, Hq, D], q's dtype) receives the attention over the sequences' whole
    histories. block_tables / context_lens describe this rank's slice
    (local_view), max_context bounds its lengths; every rank of `group`
    calls this with the same q and the same shapes."""
    partial = partial or B.pa_decode_partial
    merge = merge or B.pa_merge_partials
    all_gather = all_gather or (lambda dst, src: _all_gather(dst, src, group))
    batch, hq, d = q.shape
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    part_o = torch.empty((batch, hq, d), dtype=torch.float32, device=q.device)
    part_ml = torch.empty((batch, hq, 2), dtype=torch.float32, device=q.device)
    partial(q, k_cache, v_cache, block_tables, context_lens, scale, part_o, part_ml, cache,
            max_context, partition_tokens, workspace, stream)
    all_o = torch.empty((world, batch, hq, d), dtype=torch.float32, device=q.device)
    all_ml = torch.empty((world, batch, hq, 2), dtype=torch.float32, device=q.device)
    if world == 1:
        all_o[0].copy_(part_o)
        all_ml[0].copy_(part_ml)
    else:
        all_gather(all_o, part_o)
        all_gather(all_ml, part_ml)
    merge(all_o, all_ml, out, stream)
    return out
