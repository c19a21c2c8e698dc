"""End to end on the GPU with the host block manager deciding placement:
requests share a system prompt through the prefix cache, beams fork and copy
their partial last block on write, and every step appends and decodes. The
oracle replays the same appends, copies and decodes on its own pool (the
block manager only supplies slots, tables and copy pairs to both sides)."""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.block_manager import BlockManager

from helpers import TOL, max_abs_err

pytestmark = pytest.mark.gpu

BS, NB, HQ, HKV, D = 16, 400, 8, 2, 128


class Pair:
    """The GPU caches and the oracle's caches, driven in lockstep."""

    def __init__(self, rng):
        self.rng = rng
        shape = (NB, BS, HKV, D)
        self.kc = np.zeros(shape, np.uint16)
        self.vc = np.zeros(shape, np.uint16)
        self.gk = torch.zeros(shape, dtype=torch.float16, device="cuda")
        self.gv = torch.zeros(shape, dtype=torch.float16, device="cuda")
        self.cache = B.PagedCache(NB, BS, HKV, D, torch.float16)

    def append(self, slots):
        slots = np.asarray(slots, np.int64)
        k = W.normal_bits(self.rng, (len(slots), HKV, D), "f16")
        v = W.normal_bits(self.rng, (len(slots), HKV, D), "f16")
        oracle.append_kv(k, v, "f16", slots, self.kc, self.vc, "f16", BS)
        t = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.float16)
        B.pa_append_kv(t(k), t(v), torch.from_numpy(slots).cuda(), self.gk, self.gv, self.cache)

    def copy(self, pairs):
        if pairs:
            oracle.copy_blocks(np.asarray(pairs, np.int32), self.kc, self.vc, "f16")
            B.pa_copy_blocks(pairs, self.gk, self.gv, self.cache)

    def decode_and_compare(self, tables, lens, shared_prefix_blocks=0):
        q = W.normal_bits(self.rng, (len(lens), HQ, D), "f16")
        scale = np.float32(1 / math.sqrt(D))
        want = oracle.decode(q, "f16", self.kc, self.vc, "f16", tables, lens, scale)
        gq = torch.from_numpy(q.view(np.int16)).cuda().view(torch.float16)
        out = torch.empty_like(gq)
        gt = torch.from_numpy(tables).cuda()
        gl = torch.from_numpy(lens).cuda()
        maxc = int(lens.max())
        if shared_prefix_blocks:
            ws = B.pa_decode_shared_prefix_workspace_size(len(lens), HQ, maxc,
                                                          shared_prefix_blocks, self.cache)
            wst = torch.empty(ws, dtype=torch.uint8, device="cuda")
            B.pa_decode_shared_prefix(gq, self.gk, self.gv, gt, gl, scale, out, self.cache, maxc,
                                      shared_prefix_blocks, workspace=wst)
        else:
            ws = B.pa_decode_workspace_size(len(lens), HQ, maxc, self.cache)
            wst = torch.empty(ws, dtype=torch.uint8, device="cuda") if ws else None
            B.pa_decode(gq, self.gk, self.gv, gt, gl, scale, out, self.cache, maxc,
                        workspace=wst)
        torch.cuda.synchronize()
        assert B.pa_get_device_error() == 0
        err = max_abs_err(out.double().cpu().numpy(), want)
        assert err <= TOL["f16"], err
        # the caches agree bit for bit as well
        gk = self.gk.cpu().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(gk, self.kc)


def test_serving_steps_through_the_block_manager():
    rng = np.random.default_rng(5)
    bm = BlockManager(NB, BS, prefix_cache=True)
    pair = Pair(rng)
    system = list(range(1000, 1048))                 # 48 tokens = 3 full blocks
    users = {0: [1] * 5, 1: [2] * 20, 2: [3] * 33, 3: []}
    for sid, extra in users.items():
        prompt = system + extra
        cached = bm.add_sequence(sid, prompt)
        assert cached == (0 if sid == 0 else 48)
        n = len(prompt) - cached                     # prefill only what is not cached
        if n:
            pair.append(bm.slots(sid, cached, n))
    # beams of request 1 (68 tokens: its last block is partial)
    for child in (10, 11, 12):
        bm.fork(1, child)
    seqs = [0, 1, 2, 3, 10, 11, 12]
    for step in range(20):
        slots, pairs = [], []
        for sid in seqs:
            slot, cow = bm.append_token(sid, 500 + step)
            slots.append(slot)
            if cow:
                pairs.append(cow)
        if step == 0:
            assert len(pairs) == 3                   # three beams copy, one writes in place
        pair.copy(pairs)
        pair.append(slots)
        tables, lens = bm.block_tables(seqs, 16)
        pair.decode_and_compare(tables, lens, shared_prefix_blocks=3 if step % 2 else 0)
    # finished requests release their blocks; a new request still reuses the prompt
    for sid in (0, 2):
        bm.free_sequence(sid)
    assert bm.add_sequence(20, system + [9]) == 48
    pair.append(bm.slots(20, 48, 1))
    tables, lens = bm.block_tables([1, 20, 11], 16)
    pair.decode_and_compare(tables, lens, shared_prefix_blocks=3)
