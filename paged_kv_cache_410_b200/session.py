"""One decode step of one attention layer on the GPU, driven through the C ABI.

``DecodeStep`` places a workload's tensors in device memory (torch) and runs
the hot path in the order a serving engine does: copy-on-write block copies
for forked beams, append of the new tokens' K/V, then paged decode. Every
operation is a call into libpagedattn.so through ``binding``.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B

_TORCH = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.uint8}


def to_device(bits: np.ndarray, dtype: str, device) -> torch.Tensor:
    """Bit patterns (uint16 / uint8 numpy) -> device tensor of the storage dtype."""
    if dtype == "e4m3":
        return torch.from_numpy(np.ascontiguousarray(bits)).to(device)
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)
    return t.view(_TORCH[dtype])


def to_bits(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> host bit patterns (uint16 for 16-bit types, uint8 for E4M3)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.uint8:
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


class DecodeStep:
    """`shared_prefix_blocks` > 0 decodes through pa_decode_shared_prefix (the
    workload's tables must all start with those blocks); `window` > 0 through
    pa_decode_sliding_window; `fused` runs append and decode as one
    pa_append_decode launch."""

    def __init__(self, w, device="cuda", partition_tokens: int = 0, stream=None,
                 shared_prefix_blocks: int = 0, window: int = 0, fused: bool = False):
        if sum(map(bool, (shared_prefix_blocks, window, fused))) > 1:
            raise ValueError("shared prefix, sliding window and fused append are separate paths")
        self.w = w
        self.device = torch.device(device)
        self.stream = stream
        self.partition_tokens = partition_tokens
        self.shared_prefix_blocks = shared_prefix_blocks
        self.window = window
        self.fused = fused
        dev = self.device
        cshape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
        if w.cache_dtype == "e4m3":
            self.k_scale = torch.from_numpy(w.k_scale).to(dev)
            self.v_scale = torch.from_numpy(w.v_scale).to(dev)
            self.k_inv_scale = torch.from_numpy(w.k_inv_scale).to(dev)
            self.v_inv_scale = torch.from_numpy(w.v_inv_scale).to(dev)
            self.k_cache = torch.zeros(cshape, dtype=torch.uint8, device=dev)
            self.v_cache = torch.zeros(cshape, dtype=torch.uint8, device=dev)
        else:
            self.k_scale = self.v_scale = self.k_inv_scale = self.v_inv_scale = None
            self.k_cache = to_device(w.k_pool, w.cache_dtype, dev)
            self.v_cache = to_device(w.v_pool, w.cache_dtype, dev)
        self.cache = B.PagedCache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim,
                                  self.k_cache.dtype, self.k_scale, self.v_scale,
                                  self.k_inv_scale, self.v_inv_scale)
        self.q = to_device(w.q, w.io_dtype, dev)
        self.k_new = to_device(w.k_new, w.io_dtype, dev)
        self.v_new = to_device(w.v_new, w.io_dtype, dev)
        self.slot_mapping = torch.from_numpy(w.slot_mapping).to(dev)
        self.block_tables = torch.from_numpy(w.block_tables).to(dev)
        self.context_lens = torch.from_numpy(w.context_lens).to(dev)
        self.copy_pairs = np.ascontiguousarray(w.copy_pairs, dtype=np.int32)
        self.out = torch.empty((w.batch, w.num_q_heads, w.head_dim), dtype=self.q.dtype,
                               device=dev)
        self.max_context = w.max_context
        if shared_prefix_blocks:
            ws = B.pa_decode_shared_prefix_workspace_size(w.batch, w.num_q_heads,
                                                          self.max_context, shared_prefix_blocks,
                                                          self.cache, partition_tokens)
        elif window:
            ws = B.pa_decode_sliding_window_workspace_size(w.batch, w.num_q_heads,
                                                           self.max_context, window, self.cache,
                                                           partition_tokens)
        else:
            ws = B.pa_decode_workspace_size(w.batch, w.num_q_heads, self.max_context,
                                            self.cache, partition_tokens)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev) if ws else None
        if w.cache_dtype == "e4m3" and w.fill_slots is not None and len(w.fill_slots):
            # history tokens are quantised into the pool by the library's append
            fk = to_device(w.fill_k, w.io_dtype, dev)
            fv = to_device(w.fill_v, w.io_dtype, dev)
            fs = torch.from_numpy(w.fill_slots).to(dev)
            B.pa_append_kv(fk, fv, fs, self.k_cache, self.v_cache, self.cache, stream)
            del fk, fv, fs

    # the three operations of a step
    def copy(self):
        if len(self.copy_pairs):
            B.pa_copy_blocks(self.copy_pairs, self.k_cache, self.v_cache, self.cache, self.stream)

    def append(self):
        B.pa_append_kv(self.k_new, self.v_new, self.slot_mapping, self.k_cache, self.v_cache,
                       self.cache, self.stream)

    def decode(self):
        if self.shared_prefix_blocks:
            B.pa_decode_shared_prefix(self.q, self.k_cache, self.v_cache, self.block_tables,
                                      self.context_lens, float(self.w.scale), self.out,
                                      self.cache, self.max_context, self.shared_prefix_blocks,
                                      self.partition_tokens, self.workspace, self.stream)
            return
        if self.window:
            B.pa_decode_sliding_window(self.q, self.k_cache, self.v_cache, self.block_tables,
                                       self.context_lens, float(self.w.scale), self.out,
                                       self.cache, self.max_context, self.window,
                                       self.partition_tokens, self.workspace, self.stream)
            return
        B.pa_decode(self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                    float(self.w.scale), self.out, self.cache, self.max_context,
                    self.partition_tokens, self.workspace, self.stream)

    def append_decode(self):
        B.pa_append_decode(self.q, self.k_new, self.v_new, self.slot_mapping, self.k_cache,
                           self.v_cache, self.block_tables, self.context_lens,
                           float(self.w.scale), self.out, self.cache, self.max_context,
                           self.partition_tokens, self.workspace, self.stream)

    def run(self):
        self.copy()
        if self.fused:
            self.append_decode()
            return
        self.append()
        self.decode()

    def device_errors(self) -> int:
        return B.pa_get_device_error(self.stream)

    def out_f64(self) -> np.ndarray:
        return self.out.double().cpu().numpy()
