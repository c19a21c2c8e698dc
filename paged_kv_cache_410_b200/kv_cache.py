"""Paged K/V caches of a model's attention layers on one GPU, placed by the
host block manager.

``PagedKVCache`` joins the library's two halves: the host block manager
(``block_manager.py``, C++) decides where each token's K/V lives, and the
kernels (``binding.py``, CUDA) store into and attend through those places.
A decode step of a batch:

    plan = cache.begin_step(seq_ids, token_ids)   # slots, copy-on-write copies for
                                                  # every layer, tables and lengths
    for layer in range(num_layers):
        out = cache.attend(plan, layer, q, k, v)  # this layer's append + decode

``begin_step`` runs once per step on the host: one batched append in the
block manager, one multi-layer block copy for the beams that diverge, the
block-table rows that changed since the last step, and one upload of slots,
tables and lengths from pinned memory. ``attend`` is one
``pa_append_decode`` launch per layer (the new token's K/V is stored and
attended in the same kernel), or, when every sequence of the step starts
with the same run of at least ``shared_prefix_min_blocks`` physical blocks
(a system prompt served from the prefix cache), an append and
``pa_decode_shared_prefix``, which attends that prefix once for the whole
batch. With ``window`` > 0 every layer attends only each sequence's last
``window`` tokens (``pa_decode_sliding_window``), and ``begin_step`` hands
the blocks the window has left behind back to the pool.

Prompts: ``add_sequence`` places a prompt, reusing cached prefix blocks, and
returns the slots of the tokens whose K/V the caller still has to store
(``store_prompt``).

Several GPUs (tensor parallelism over KV heads): every rank builds a cache
for its own heads and drives its own block manager with the same calls, so
all ranks place every token in the same slots and no exchange is needed.
Given a process group (``lockstep_group``), ``begin_step`` checks that: it
all-gathers a 64-bit digest of the step's slots, copy pairs and lengths and
raises on every rank if any rank's differs.
"""
from __future__ import annotations

import contextlib
import hashlib
import math
from dataclasses import dataclass

import numpy as np
import torch

from . import binding as B
from .block_manager import BlockManager

_E4M3 = (torch.uint8, torch.float8_e4m3fn)


@dataclass
class StepPlan:
    """Device-side inputs of one decode step (shared by all layers); views of
    buffers the next begin_step overwrites."""
    n: int
    slot_mapping: torch.Tensor   # int64 [n]: slot of each sequence's new token
    block_tables: torch.Tensor   # int32 [n, max_blocks_per_seq]
    context_lens: torch.Tensor   # int32 [n], the new token included
    max_context: int
    copy_pairs: np.ndarray       # int32 [k, 2] copied (every layer) before the step
    shared_prefix_blocks: int    # leading blocks every sequence's table shares


class PagedKVCache:
    """`num_layers` K and V caches of [num_blocks, block_size, num_kv_heads,
    head_dim] in `dtype` (fp16, bf16, or E4M3 stored as uint8 with per-layer
    fp32 scales [num_kv_heads, head_dim] in `k_scales` / `v_scales`; the
    queries and new K/V are then `io_dtype`), and the block manager that
    places tokens in them. Batches hold at most `max_batch` sequences of at
    most `max_blocks_per_seq` blocks. Every upload, copy and kernel goes on
    `stream` (a torch.cuda.Stream; None: torch's current stream)."""

    def __init__(self, num_blocks: int, block_size: int, num_kv_heads: int, head_dim: int,
                 num_layers: int = 1, dtype=torch.float16, io_dtype=None, device="cuda",
                 prefix_cache: bool = True, max_batch: int = 256, max_blocks_per_seq: int = 512,
                 k_scales=None, v_scales=None, stream=None, shared_prefix_min_blocks: int = 32,
                 window: int = 0, lockstep_group=None):
        if window < 0:
            raise ValueError("window must be >= 0 (0: whole history)")
        self.window = window
        self.lockstep_group = lockstep_group
        self.device = torch.device(device)
        self.stream = stream
        self.shared_prefix_min_blocks = shared_prefix_min_blocks
        self.block_size = block_size
        self.num_kv_heads = num_kv_heads
        self.head_dim = head_dim
        self.num_layers = num_layers
        self.e4m3 = dtype in _E4M3
        if self.e4m3:
            if io_dtype not in (torch.float16, torch.bfloat16):
                raise ValueError("an E4M3 cache needs io_dtype float16 or bfloat16")
            if k_scales is None or v_scales is None or \
                    len(k_scales) != num_layers or len(v_scales) != num_layers:
                raise ValueError("an E4M3 cache needs one K and one V scale array per layer")
        self.io_dtype = io_dtype if self.e4m3 else dtype
        shape = (num_blocks, block_size, num_kv_heads, head_dim)
        self.k = [torch.zeros(shape, dtype=dtype, device=self.device) for _ in range(num_layers)]
        self.v = [torch.zeros(shape, dtype=dtype, device=self.device) for _ in range(num_layers)]
        self.layers = []
        for layer in range(num_layers):
            sc = {}
            if self.e4m3:
                ks = k_scales[layer].to(self.device, torch.float32).contiguous()
                vs = v_scales[layer].to(self.device, torch.float32).contiguous()
                sc = dict(k_scale=ks, v_scale=vs, k_inv_scale=(1.0 / ks).contiguous(),
                          v_inv_scale=(1.0 / vs).contiguous())
            self.layers.append(B.PagedCache(num_blocks, block_size, num_kv_heads, head_dim,
                                            dtype, **sc))
        self.bm = BlockManager(num_blocks, block_size, prefix_cache)
        # host staging (pinned on a GPU) and device copies of slots, tables and
        # lengths; table rows are rewritten only when their block list changed
        self.max_batch, self.max_blocks = max_batch, max_blocks_per_seq
        pin = self.device.type == "cuda"
        self._h_slots = torch.zeros(max_batch, dtype=torch.int64, pin_memory=pin)
        self._h_tables = torch.zeros((max_batch, max_blocks_per_seq), dtype=torch.int32,
                                     pin_memory=pin)
        self._h_lens = torch.zeros(max_batch, dtype=torch.int32, pin_memory=pin)
        self._versions = np.zeros(max_batch, dtype=np.uint64)
        self._d_slots = torch.zeros(max_batch, dtype=torch.int64, device=self.device)
        self._d_tables = torch.zeros((max_batch, max_blocks_per_seq), dtype=torch.int32,
                                     device=self.device)
        self._d_lens = torch.zeros(max_batch, dtype=torch.int32, device=self.device)
        self._uploaded = None      # event after the last upload (the staging is reused)
        self._workspace = None

    # ---- sequences -------------------------------------------------------------
    def add_sequence(self, seq_id: int, token_ids):
        """Place a prompt. Returns (tokens whose K/V is already cached, int64
        device slots of the others, in order). Store the others' K/V for every
        layer (store_prompt) before the next add_sequence or step: the prompt's
        full blocks are offered to later prompts as soon as they exist."""
        cached = self.bm.add_sequence(seq_id, token_ids)
        rest = self.bm.slots(seq_id, cached, len(token_ids) - cached)
        return cached, torch.from_numpy(rest).to(self.device)

    def store_prompt(self, layer: int, slots, k, v):
        """Store prompt K/V ([T, Hkv, D] in io_dtype) of one layer at `slots`."""
        B.pa_append_kv(k, v, slots, self.k[layer], self.v[layer], self.layers[layer],
                       self.stream)

    def fork(self, parent_id: int, child_id: int):
        self.bm.fork(parent_id, child_id)

    def free_sequence(self, seq_id: int):
        self.bm.free_sequence(seq_id)

    # ---- decode steps -----------------------------------------------------------
    def begin_step(self, seq_ids, token_ids) -> StepPlan:
        """Reserve one new token per sequence (token_ids: the ids just sampled),
        copy the blocks forked beams diverge on (every layer), and upload the
        step's slots, tables and lengths. An unknown or repeated id, or a pool
        that cannot supply the step, raises with nothing reserved; a sequence
        that outgrows max_blocks_per_seq raises after its token was reserved."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = len(ids)
        if n > self.max_batch:
            raise ValueError(f"{n} sequences > max_batch {self.max_batch}")
        if self._uploaded is not None:
            self._uploaded.synchronize()  # the staging buffers are about to change
        slots, pairs = self.bm.append_tokens(ids, token_ids)
        if len(pairs):
            B.pa_copy_blocks_layers(pairs, self.k, self.v, self.layers[0], self.stream)
        h_slots, h_lens = self._h_slots.numpy(), self._h_lens.numpy()
        h_slots[:n] = slots
        self.bm.block_tables_update(ids, self._h_tables.numpy()[:n], h_lens[:n],
                                    self._versions[:n])
        with self._on_stream():
            self._d_slots[:n].copy_(self._h_slots[:n], non_blocking=True)
            self._d_tables[:n].copy_(self._h_tables[:n], non_blocking=True)
            self._d_lens[:n].copy_(self._h_lens[:n], non_blocking=True)
            if self.device.type == "cuda":
                self._uploaded = torch.cuda.Event()
                self._uploaded.record()
        if self.window:
            # blocks holding only tokens before this step's window; their table
            # entries stay (the window decode never reads them), and they are
            # reused only by later steps, behind this step's kernels on the stream
            self.bm.release_window(ids, self.window)
        if self.lockstep_group is not None:
            self._check_lockstep(slots, pairs, h_lens[:n])
        shared = 0
        if self.shared_prefix_min_blocks > 0 and not self.window:
            shared = common_prefix_blocks(self._h_tables.numpy()[:n], h_lens[:n],
                                          self.block_size)
        return StepPlan(n=n, slot_mapping=self._d_slots[:n], block_tables=self._d_tables[:n],
                        context_lens=self._d_lens[:n],
                        max_context=int(h_lens[:n].max()) if n else 0, copy_pairs=pairs,
                        shared_prefix_blocks=shared)

    def attend(self, plan: StepPlan, layer: int, q, k, v, scale: float | None = None, out=None):
        """Store this layer's new K/V (k, v [n, Hkv, D]) at the plan's slots and
        return the decode output [n, Hq, D] for queries q [n, Hq, D]: one
        pa_append_decode launch, or pa_append_kv + pa_decode_shared_prefix
        when the plan's shared prefix is long enough, or pa_append_kv +
        pa_decode_sliding_window with a window."""
        if out is None:
            out = torch.empty_like(q)
        if scale is None:
            scale = 1.0 / math.sqrt(self.head_dim)
        cache = self.layers[layer]
        spb = plan.shared_prefix_blocks
        cascade = self.shared_prefix_min_blocks > 0 and spb >= self.shared_prefix_min_blocks
        if self.window:
            need = B.pa_decode_sliding_window_workspace_size(plan.n, q.shape[1],
                                                             plan.max_context, self.window, cache)
        elif cascade:
            need = B.pa_decode_shared_prefix_workspace_size(plan.n, q.shape[1], plan.max_context,
                                                            spb, cache)
        else:
            need = B.pa_decode_workspace_size(plan.n, q.shape[1], plan.max_context, cache)
        if need and (self._workspace is None or self._workspace.numel() < need):
            with self._on_stream():
                self._workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
        ws = self._workspace if need else None
        if self.window:
            B.pa_append_kv(k, v, plan.slot_mapping, self.k[layer], self.v[layer], cache,
                           self.stream)
            B.pa_decode_sliding_window(q, self.k[layer], self.v[layer], plan.block_tables,
                                       plan.context_lens, scale, out, cache, plan.max_context,
                                       self.window, workspace=ws, stream=self.stream)
        elif cascade:
            B.pa_append_kv(k, v, plan.slot_mapping, self.k[layer], self.v[layer], cache,
                           self.stream)
            B.pa_decode_shared_prefix(q, self.k[layer], self.v[layer], plan.block_tables,
                                      plan.context_lens, scale, out, cache, plan.max_context,
                                      spb, workspace=ws, stream=self.stream)
        else:
            B.pa_append_decode(q, k, v, plan.slot_mapping, self.k[layer], self.v[layer],
                               plan.block_tables, plan.context_lens, scale, out, cache,
                               plan.max_context, workspace=ws, stream=self.stream)
        return out

    def _check_lockstep(self, slots, pairs, lens):
        import torch.distributed as dist
        h = hashlib.blake2b(digest_size=8)
        for a in (slots, pairs, lens):
            h.update(np.ascontiguousarray(a).tobytes())
        mine = int.from_bytes(h.digest(), "little", signed=True)
        dev = self.device if dist.get_backend(self.lockstep_group) == "nccl" else "cpu"
        t = torch.tensor([mine], dtype=torch.int64, device=dev)
        every = [torch.empty_like(t) for _ in range(dist.get_world_size(self.lockstep_group))]
        dist.all_gather(every, t, group=self.lockstep_group)
        if any(int(x.item()) != mine for x in every):
            raise RuntimeError("block managers out of lockstep: the ranks placed this step's "
                               "tokens differently")

    def _on_stream(self):
        if self.device.type == "cuda" and isinstance(self.stream, torch.cuda.Stream):
            return torch.cuda.stream(self.stream)
        return contextlib.nullcontext()


def common_prefix_blocks(tables: np.ndarray, lens: np.ndarray, block_size: int) -> int:
    """Leading block-table entries that every row shares, counting only
    blocks every sequence has filled (so none of them is written this step:
    a sequence that writes into a shared block has been given its own copy)."""
    n = len(lens)
    if n < 2:
        return 0
    kmax = int(lens.min()) // block_size
    if kmax == 0:
        return 0
    same = (tables[1:, :kmax] == tables[0, :kmax]).all(axis=0)
    return int(kmax if same.all() else np.argmin(same))
