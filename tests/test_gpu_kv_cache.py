"""PagedKVCache (paged_kv_cache_410_b200/kv_cache.py) end to end on the GPU.

A two-layer serving loop through the real library: prompts placed by the host
block manager (later prompts served from its prefix cache), a beam fork whose
first step copies the shared partial block in every layer
(pa_copy_blocks_layers), then decode steps through each layer's entry point:
pa_append_decode, the shared-prefix decode when every table starts with the
same run of at least 32 filled blocks, or the sliding-window decode with the
blocks the window left behind released. A float64 oracle keeps its own copy
of every layer's K and V caches, applying the same stores and block copies;
after every layer of every step the device caches must equal it bit for bit
and the decode output must match the oracle's decode over it (2e-3 for fp16
outputs, 1e-2 for bf16)."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200.kv_cache import PagedKVCache
from paged_kv_cache_410_b200.session import to_bits

from helpers import TOL, max_abs_err

pytestmark = pytest.mark.gpu

BS, D = 16, 128


class Shadow:
    """The oracle's copy of one layer's caches."""

    def __init__(self, oracle, shape, cache_dtype, io_dtype, scales=None):
        self.o = oracle
        dt = np.uint8 if cache_dtype == "e4m3" else np.uint16
        self.k = np.zeros(shape, dt)
        self.v = np.zeros(shape, dt)
        self.cd, self.io = cache_dtype, io_dtype
        self.sc = scales  # (k_scale, v_scale, k_inv, v_inv) float32 numpy, E4M3 only

    def store(self, k, v, slots):
        inv = (self.sc[2], self.sc[3]) if self.sc else (None, None)
        self.o.append_kv(to_bits(k), to_bits(v), self.io, slots.cpu().numpy(), self.k, self.v,
                         self.cd, BS, *inv)

    def copy(self, pairs):
        if len(pairs):
            self.o.copy_blocks(np.asarray(pairs, np.int32), self.k, self.v, self.cd)

    def decode(self, q, tables, lens, scale, window=0):
        ks, vs = (self.sc[0], self.sc[1]) if self.sc else (None, None)
        return self.o.decode(to_bits(q), self.io, self.k, self.v, self.cd, tables, lens, scale,
                             k_scale=ks, v_scale=vs, window=window)


MODES = {
    # mode: (cache dtype, io dtype, kv heads, q heads, system prompt tokens, window)
    "fused": ("f16", "f16", 2, 8, 40, 0),
    "shared_prefix": ("bf16", "bf16", 2, 16, 33 * BS + 3, 0),
    "window": ("f16", "f16", 2, 8, 40, 48),
    "e4m3": ("e4m3", "f16", 2, 8, 40, 0),
}
TORCH = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.uint8}


@pytest.mark.parametrize("mode", list(MODES))
def test_serving_loop_matches_the_oracle_every_step(oracle_mod, mode):
    cdt, io, hkv, hq, sys_len, window = MODES[mode]
    layers, nb = 2, 256
    rng = np.random.default_rng(41 + len(mode))
    dev = torch.device("cuda")
    scales = None
    if cdt == "e4m3":
        ks = [rng.uniform(0.005, 0.02, (hkv, D)).astype(np.float32) for _ in range(layers)]
        vs = [rng.uniform(0.005, 0.02, (hkv, D)).astype(np.float32) for _ in range(layers)]
    cache = PagedKVCache(nb, BS, hkv, D, num_layers=layers, dtype=TORCH[cdt],
                         io_dtype=TORCH[io], device=dev, max_batch=8, max_blocks_per_seq=64,
                         window=window,
                         k_scales=[torch.from_numpy(x) for x in ks] if cdt == "e4m3" else None,
                         v_scales=[torch.from_numpy(x) for x in vs] if cdt == "e4m3" else None)
    shadows = []
    for l in range(layers):
        if cdt == "e4m3":
            c = cache.layers[l]
            scales = tuple(t.cpu().numpy() for t in (c.k_scale, c.v_scale, c.k_inv_scale,
                                                     c.v_inv_scale))
        shadows.append(Shadow(oracle_mod, tuple(cache.k[l].shape), cdt, io, scales))

    def rand(*shape):
        return torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(
            TORCH[io]).to(dev)

    def check_caches(what):
        torch.cuda.synchronize()
        for l in range(layers):
            assert np.array_equal(to_bits(cache.k[l]), shadows[l].k), f"{what}: K layer {l}"
            assert np.array_equal(to_bits(cache.v[l]), shadows[l].v), f"{what}: V layer {l}"

    system = list(range(1000, 1000 + sys_len))
    cached_counts = []
    for sid in range(4):
        prompt = system + [sid] * (3 + sid)
        cached, slots = cache.add_sequence(sid, prompt)
        cached_counts.append(cached)
        for l in range(layers):
            k, v = rand(len(slots), hkv, D), rand(len(slots), hkv, D)
            cache.store_prompt(l, slots, k, v)
            shadows[l].store(k, v, slots)
    # later prompts reuse the system prompt's full blocks from the prefix cache
    assert cached_counts[0] == 0 and all(c == sys_len // BS * BS for c in cached_counts[1:])
    check_caches("prompts")
    cache.fork(1, 4)                                   # a beam sharing sequence 1's blocks
    ids = [0, 1, 2, 3, 4]
    scale = float(np.float32(1 / np.sqrt(D)))
    paths, pairs_seen = set(), 0
    for step in range(8):
        plan = cache.begin_step(ids, [step] * len(ids))
        pairs_seen += len(plan.copy_pairs)
        for l in range(layers):
            shadows[l].copy(plan.copy_pairs)
        tables = plan.block_tables.cpu().numpy()
        lens = plan.context_lens.cpu().numpy()
        cascade = plan.shared_prefix_blocks >= cache.shared_prefix_min_blocks
        paths.add("window" if window else "shared_prefix" if cascade else "fused")
        for l in range(layers):
            q, k, v = rand(len(ids), hq, D), rand(len(ids), hkv, D), rand(len(ids), hkv, D)
            out = cache.attend(plan, l, q, k, v, scale=scale)
            shadows[l].store(k, v, plan.slot_mapping)
            want = shadows[l].decode(q, tables, lens, scale, window)
            check_caches(f"step {step} layer {l}")
            err = max_abs_err(out.double().cpu().numpy(), want)
            assert err <= TOL[io], f"{mode} step {step} layer {l}: max abs err {err}"
        assert cache.bm.length(0) == len(system) + 3 + step + 1
    assert pairs_seen >= 1                             # the fork copied its partial block
    assert paths == {{"fused": "fused", "e4m3": "fused"}.get(mode, mode)}
    if window:
        # each sequence keeps at most the blocks its window spans (+1 partial)
        held = len(ids) * (-(-window // BS) + 1)
        assert cache.bm.num_free_blocks + cache.bm.num_cached_blocks >= nb - held
