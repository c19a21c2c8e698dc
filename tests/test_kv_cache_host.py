"""PagedKVCache (paged_kv_cache_410_b200/kv_cache.py) on the CPU.

With a recording stand-in for the CUDA library (the block manager is the
real C++ one): the step plans it uploads follow the block manager exactly
(slots, copy-on-write pairs, tables, lengths), copies reach every layer, and
each layer's decode is the expected entry point on the plan's tensors.

With the float64 oracle standing in for each entry point: a serving loop
(two layers, prompts through the prefix cache, a beam fork, nine steps) in
the fused, shared-prefix and sliding-window modes gives, for every sequence,
layer and head, the attention computed straight from that sequence's logical
history. No GPU and no kernel is involved: the kernels' own parity is the
GPU tests' subject."""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200.block_manager import BlockManager
from paged_kv_cache_410_b200.kv_cache import PagedKVCache


class Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(B, "load_library", lambda *a, **k: r)
    monkeypatch.setattr(B, "_on_device", lambda t: True)
    return r


NB, BS, HKV, D, HQ, LAYERS, MB = 64, 4, 2, 64, 8, 3, 16


def kv(n):
    return torch.zeros((n, HKV, D), dtype=torch.float16)


def test_steps_follow_the_block_manager(rec):
    cache = PagedKVCache(NB, BS, HKV, D, num_layers=LAYERS, device="cpu", max_batch=8, stream=0,
                         max_blocks_per_seq=MB)
    twin = BlockManager(NB, BS, prefix_cache=True)
    prompt = list(range(10))                          # 2 full blocks + 2 tokens
    cached, slots = cache.add_sequence(0, prompt)
    twin.add_sequence(0, prompt)
    assert cached == 0 and slots.tolist() == twin.slots(0, 0, 10).tolist()
    for layer in range(LAYERS):
        cache.store_prompt(layer, slots, kv(10), kv(10))
    stores = [a for n, a in rec.calls if n == "pa_append_kv"]
    assert [a[5] for a in stores] == [t.data_ptr() for t in cache.k]  # one store per layer
    for c in (1, 2):                                  # two beams share every block
        cache.fork(0, c)
        twin.fork(0, c)
    order = [[0, 1, 2], [2, 0, 1], [1, 2, 0], [0, 1, 2], [2, 1, 0]]
    for step, ids in enumerate(order):
        toks = [100 * step + i for i in ids]
        rec.calls.clear()
        plan = cache.begin_step(ids, toks)
        want_slots, want_pairs = [], []
        for sid, t in zip(ids, toks):
            s, cow = twin.append_token(sid, t)
            want_slots.append(s)
            if cow:
                want_pairs.append(list(cow))
        assert plan.slot_mapping.tolist() == want_slots, step
        assert plan.copy_pairs.tolist() == want_pairs, step
        tables, lens = twin.block_tables(ids, MB)
        assert np.array_equal(plan.block_tables.numpy(), tables), step
        assert plan.context_lens.tolist() == lens.tolist() and plan.max_context == lens.max()
        copies = [a for n, a in rec.calls if n == "pa_copy_blocks_layers"]
        if want_pairs:                                # one call for all layers
            assert len(copies) == 1 and copies[0][1] == len(want_pairs) and copies[0][4] == LAYERS
            assert [copies[0][2][i] for i in range(LAYERS)] == [t.data_ptr() for t in cache.k]
        else:
            assert copies == []
        if step == 0:
            assert len(want_pairs) == 2               # two beams copy, the last writes in place
        rec.calls.clear()
        for layer in range(LAYERS):
            q = torch.zeros((len(ids), HQ, D), dtype=torch.float16)
            k, v = kv(len(ids)), kv(len(ids))
            out = cache.attend(plan, layer, q, k, v)
            name, a = [c for c in rec.calls if c[0] == "pa_append_decode"][-1]
            assert a[0] == q.data_ptr() and a[1] == k.data_ptr() and a[2] == v.data_ptr()
            assert a[6] == plan.slot_mapping.data_ptr() and a[7] == cache.k[layer].data_ptr()
            assert a[10] == plan.block_tables.data_ptr() and a[11] == MB
            assert a[12] == plan.context_lens.data_ptr() and a[13] == plan.max_context
            assert abs(a[14] - 1 / 8) < 1e-12 and a[15] == out.data_ptr()


def test_prefix_cache_serves_a_second_prompt(rec):
    cache = PagedKVCache(NB, BS, HKV, D, device="cpu", max_batch=4, max_blocks_per_seq=MB,
                         stream=0)
    system = list(range(50, 58))                      # two full blocks
    c1, s1 = cache.add_sequence(1, system + [1, 2])
    c2, s2 = cache.add_sequence(2, system + [3])
    assert (c1, c2) == (0, 8) and len(s2) == 1        # only the new token's K/V is stored
    plan = cache.begin_step([1, 2], [7, 7])
    assert (plan.block_tables[0, :2] == plan.block_tables[1, :2]).all()


def test_e4m3_layers_carry_their_scales(rec):
    ks = [torch.full((HKV, D), 0.5 + l) for l in range(2)]
    vs = [torch.full((HKV, D), 2.0 + l) for l in range(2)]
    cache = PagedKVCache(NB, BS, HKV, D, num_layers=2, dtype=torch.uint8,
                         io_dtype=torch.bfloat16, device="cpu", k_scales=ks, v_scales=vs,
                         stream=0)
    assert torch.equal(cache.layers[1].k_inv_scale, 1.0 / ks[1])
    cached, slots = cache.add_sequence(0, [1, 2, 3])
    cache.store_prompt(1, slots, torch.zeros((3, HKV, D), dtype=torch.bfloat16),
                       torch.zeros((3, HKV, D), dtype=torch.bfloat16))
    d = rec.calls[-1][1][7]._obj
    assert d.cache_dtype == B.PA_E4M3 and d.k_scale == cache.layers[1].k_scale.data_ptr()
    with pytest.raises(ValueError):
        PagedKVCache(NB, BS, HKV, D, dtype=torch.uint8, device="cpu")   # no io dtype / scales


def test_batch_limit(rec):
    cache = PagedKVCache(NB, BS, HKV, D, device="cpu", max_batch=2, max_blocks_per_seq=MB,
                         stream=0)
    for s in range(3):
        cache.add_sequence(s, [s])
    with pytest.raises(ValueError):
        cache.begin_step([0, 1, 2], [0, 0, 0])


def test_common_prefix_blocks():
    from paged_kv_cache_410_b200.kv_cache import common_prefix_blocks
    t = np.array([[5, 6, 7, 8, 9], [5, 6, 7, 1, 2], [5, 6, 7, 8, 3]], np.int32)
    assert common_prefix_blocks(t, np.array([80, 80, 80]), 16) == 3
    assert common_prefix_blocks(t, np.array([80, 40, 80]), 16) == 2   # only filled blocks count
    assert common_prefix_blocks(t, np.array([80, 15, 80]), 16) == 0
    assert common_prefix_blocks(t[:1], np.array([80]), 16) == 0          # one sequence: no sharing
    assert common_prefix_blocks(t[[0, 2]], np.array([80, 80]), 16) == 4


def test_shared_system_prompt_takes_the_shared_prefix_decode(rec):
    cache = PagedKVCache(NB, BS, HKV, D, device="cpu", max_batch=8, max_blocks_per_seq=MB,
                         stream=0, shared_prefix_min_blocks=3)
    system = list(range(200, 214))                    # 3 full blocks + 2 tokens
    for sid in range(4):
        cache.add_sequence(sid, system + [sid, sid])
    plan = cache.begin_step([0, 1, 2, 3], [1, 2, 3, 4])
    assert plan.shared_prefix_blocks == 3
    rec.calls.clear()
    q = torch.zeros((4, HQ, D), dtype=torch.float16)
    out = cache.attend(plan, 0, q, kv(4), kv(4))
    names = [n for n, _ in rec.calls if n.startswith("pa_") and "size" not in n]
    assert names == ["pa_append_kv", "pa_decode_shared_prefix"]
    a = [c for c in rec.calls if c[0] == "pa_decode_shared_prefix"][0][1]
    assert a[11] == 3 and a[0] == q.data_ptr() and a[13] == out.data_ptr()
    # below the threshold, or with the path off: the fused launch
    short = PagedKVCache(NB, BS, HKV, D, device="cpu", max_batch=8, max_blocks_per_seq=MB,
                         stream=0, shared_prefix_min_blocks=0)
    for sid in range(2):
        short.add_sequence(sid, system)
    plan = short.begin_step([0, 1], [1, 2])
    rec.calls.clear()
    short.attend(plan, 0, torch.zeros((2, HQ, D), dtype=torch.float16), kv(2), kv(2))
    assert [n for n, _ in rec.calls if n in ("pa_append_decode", "pa_decode_shared_prefix")] == \
        ["pa_append_decode"]


def test_sliding_window_releases_blocks_and_decodes_the_window(rec):
    cache = PagedKVCache(NB, BS, HKV, D, device="cpu", max_batch=4, max_blocks_per_seq=MB,
                         stream=0, window=6, prefix_cache=False)
    for sid in range(2):
        cache.add_sequence(sid, [sid] * 5)           # 2 blocks each
    free0 = cache.bm.num_free_blocks
    for step in range(12):
        plan = cache.begin_step([0, 1], [step, step])
        rec.calls.clear()
        cache.attend(plan, 0, torch.zeros((2, HQ, D), dtype=torch.float16), kv(2), kv(2))
        names = [n for n, _ in rec.calls if n in ("pa_append_kv", "pa_decode_sliding_window",
                                                  "pa_append_decode", "pa_decode_shared_prefix")]
        assert names == ["pa_append_kv", "pa_decode_sliding_window"]
        a = [c for c in rec.calls if c[0] == "pa_decode_sliding_window"][0][1]
        assert a[11] == 6                            # the window
    # 17 tokens each: a window of 6 needs at most 3 blocks per sequence
    L = cache.bm.length(0)
    assert L == 17
    held = 2 * (-(-L // BS) - (L - 6) // BS)
    assert cache.bm.num_free_blocks == NB - held and held <= 6
    assert free0 == NB - 4
    with pytest.raises(ValueError):
        PagedKVCache(NB, BS, HKV, D, device="cpu", window=-1, stream=0)


# ---- end to end on the CPU: the oracle stands in for the kernels ---------------

class OracleLib:
    """Test stand-in for libpagedattn.so: every entry point PagedKVCache calls
    is carried out by the float64 oracle on the tensors behind the pointers,
    so the cache class's slots, tables, lengths, copies and call order can be
    checked against attention computed straight from each sequence's history.
    (Test infrastructure only: the product never calls the oracle.)"""

    def __init__(self, oracle):
        self.o = oracle
        self.t = {}
        self.f64 = {}   # output address -> the oracle's float64 result

    def reg(self, *ts):
        for t in ts:
            self.t[t.data_ptr()] = t

    def bits(self, ptr, rows=None):
        t = self.t[int(ptr)]
        t = t if rows is None else t[:rows]
        if t.dtype in (torch.float16, torch.bfloat16):
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()

    @staticmethod
    def dt(code):
        return {B.PA_F16: "f16", B.PA_BF16: "bf16", B.PA_E4M3: "e4m3"}[code]

    def __getattr__(self, name):
        if name.endswith("workspace_size"):
            return lambda *a: 0
        raise AttributeError(name)

    def pa_append_kv(self, k, v, dtype, n, slots, kc, vc, desc, stream):
        if n == 0:   # as the library: nothing to store (empty tensors may share an address)
            return 0
        d = desc._obj
        inv = [None if p is None else self.t[p].numpy() for p in (d.k_inv_scale, d.v_inv_scale)]
        self.o.append_kv(self.bits(k, n), self.bits(v, n), self.dt(dtype), self.bits(slots, n),
                         self.bits(kc), self.bits(vc), self.dt(d.cache_dtype), d.block_size, *inv)
        return 0

    def pa_copy_blocks_layers(self, pairs, n, kp, vp, layers, desc, stream):
        arr = np.ctypeslib.as_array((ctypes.c_int32 * (2 * n)).from_address(pairs.value))
        for l in range(layers):
            self.o.copy_blocks(arr.reshape(-1, 2).copy(), self.bits(kp[l]), self.bits(vp[l]),
                               self.dt(desc._obj.cache_dtype))
        return 0

    def _decode(self, q, qd, batch, hq, kc, vc, desc, bt, mb, lens, scale, out, window=0):
        d = desc._obj
        sc = [None if p is None else self.t[p].numpy() for p in (d.k_scale, d.v_scale)]
        tables = self.t[int(bt)][:batch].numpy()
        got = self.o.decode(self.bits(q, batch), self.dt(qd), self.bits(kc), self.bits(vc),
                            self.dt(d.cache_dtype), tables, self.t[int(lens)][:batch].numpy(),
                            scale, k_scale=sc[0], v_scale=sc[1], window=window)
        self.t[int(out)][:batch] = torch.from_numpy(got).to(self.t[int(out)].dtype)
        self.f64[int(out)] = got
        return 0

    def pa_append_decode(self, q, k, v, dt, batch, hq, slots, kc, vc, desc, bt, mb, lens, maxc,
                         scale, out, pt, ws, wsb, stream):
        self.pa_append_kv(k, v, dt, batch, slots, kc, vc, desc, stream)
        return self._decode(q, dt, batch, hq, kc, vc, desc, bt, mb, lens, scale, out)

    def pa_decode_shared_prefix(self, q, qd, batch, hq, kc, vc, desc, bt, mb, lens, maxc, pb,
                                scale, out, pt, ws, wsb, stream):
        tables = self.t[int(bt)][:batch].numpy()
        assert (tables[:, :pb] == tables[0, :pb]).all()      # the call's precondition
        assert (self.t[int(lens)][:batch].numpy() >= pb * desc._obj.block_size).all()
        self.prefix_calls = getattr(self, "prefix_calls", 0) + 1
        return self._decode(q, qd, batch, hq, kc, vc, desc, bt, mb, lens, scale, out)

    def pa_decode_sliding_window(self, q, qd, batch, hq, kc, vc, desc, bt, mb, lens, maxc, w,
                                 scale, out, pt, ws, wsb, stream):
        return self._decode(q, qd, batch, hq, kc, vc, desc, bt, mb, lens, scale, out, window=w)


def direct_attention(q, K, V, scale, window=0):
    """softmax(scale q.K^T) V for one sequence and query head, from its
    logical history (float64, no paging)."""
    if window:
        K, V = K[-window:], V[-window:]
    s = scale * (K @ q)
    w = np.exp(s - s.max())
    return (w[:, None] * V).sum(0) / w.sum()


@pytest.mark.parametrize("mode", ["fused", "shared_prefix", "window", "e4m3"])
def test_serving_loop_on_the_oracle_matches_attention_over_each_history(monkeypatch, oracle_mod,
                                                                       mode):
    lib = OracleLib(oracle_mod)
    monkeypatch.setattr(B, "load_library", lambda *a, **k: lib)
    monkeypatch.setattr(B, "_on_device", lambda t: True)
    rng = np.random.default_rng(5)
    layers, hq, window = 2, 4, 7
    e4m3 = mode == "e4m3"
    ks = [torch.from_numpy(rng.uniform(0.005, 0.02, (HKV, D)).astype(np.float32))
          for _ in range(layers)]
    vs = [torch.from_numpy(rng.uniform(0.005, 0.02, (HKV, D)).astype(np.float32))
          for _ in range(layers)]
    cache = PagedKVCache(NB, BS, HKV, D, num_layers=layers, device="cpu", max_batch=8,
                         max_blocks_per_seq=MB, stream=0,
                         shared_prefix_min_blocks=2 if mode == "shared_prefix" else 0,
                         window=window if mode == "window" else 0,
                         dtype=torch.uint8 if e4m3 else torch.float16,
                         io_dtype=torch.float16, k_scales=ks if e4m3 else None,
                         v_scales=vs if e4m3 else None)
    for l in range(layers):
        lib.reg(cache.k[l], cache.v[l])
        if e4m3:
            c = cache.layers[l]
            lib.reg(c.k_scale, c.v_scale, c.k_inv_scale, c.v_inv_scale)

    def stored(x, l, which):
        """The values the cache holds for new K or V rows x of layer l."""
        x = x.double().numpy()
        if not e4m3:
            return x
        c = cache.layers[l]
        scale = (c.k_scale if which == "k" else c.v_scale).numpy()
        inv = (c.k_inv_scale if which == "k" else c.v_inv_scale).numpy()
        codes = oracle_mod.e4m3_from_float((x.astype(np.float32) * inv).astype(np.float32))
        return oracle_mod.e4m3_to_double(codes) * scale
    lib.reg(cache._d_slots, cache._d_tables, cache._d_lens)
    half = lambda *shape: torch.from_numpy(rng.standard_normal(shape).astype(np.float16))
    hist = {}  # (seq, layer) -> (K [T, Hkv, D], V) float64, the logical history
    system = list(range(300, 309))                     # 2 full blocks + 1 token
    for sid in range(3):
        cached, slots = cache.add_sequence(sid, system + [sid])
        lib.reg(slots)
        for l in range(layers):
            if cached:                                 # the cached blocks hold sequence 0's K/V
                K0, V0 = hist[(0, l)]
                K, V = K0[:cached], V0[:cached]
            else:
                K = V = np.zeros((0, HKV, D))
            n = 10 - cached
            k, v = half(n, HKV, D), half(n, HKV, D)
            lib.reg(k, v)
            cache.store_prompt(l, slots, k, v)
            hist[(sid, l)] = (np.concatenate([K, stored(k, l, "k")]),
                              np.concatenate([V, stored(v, l, "v")]))
        assert cached == (0 if sid == 0 else 8)
    cache.fork(1, 3)                                   # beam: shares the partial block
    for l in range(layers):
        hist[(3, l)] = tuple(x.copy() for x in hist[(1, l)])
    ids = [0, 1, 2, 3]
    scale = 1 / np.sqrt(D)
    for step in range(9):
        plan = cache.begin_step(ids, [step] * 4)
        for l in range(layers):
            q, k, v = half(4, hq, D), half(4, HKV, D), half(4, HKV, D)
            out = torch.empty((4, hq, D), dtype=torch.float16)
            lib.reg(q, k, v, out)
            cache.attend(plan, l, q, k, v, out=out)
            got = lib.f64[out.data_ptr()]
            for i, sid in enumerate(ids):
                K, V = hist[(sid, l)]
                K = np.concatenate([K, stored(k[i:i + 1], l, "k")])
                V = np.concatenate([V, stored(v[i:i + 1], l, "v")])
                hist[(sid, l)] = (K, V)
                for h in range(hq):
                    want = direct_attention(q[i, h].double().numpy(), K[:, h // (hq // HKV)],
                                            V[:, h // (hq // HKV)], np.float32(scale),
                                            window if mode == "window" else 0)
                    np.testing.assert_allclose(got[i, h], want, rtol=0, atol=1e-9)
    if mode == "shared_prefix":
        assert lib.prefix_calls == 9 * layers
    if mode == "window":
        # sequences hold at most the 2 blocks their window spans; every other
        # block is free or only in the prefix cache (reclaimable)
        assert cache.bm.num_free_blocks + cache.bm.num_cached_blocks >= NB - 4 * 2


def _lockstep_worker(rank, world, port, diverge, q):
    import os
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = Recorder()
        B.load_library = lambda *a, **k: r       # this process only
        B._on_device = lambda t: True
        cache = PagedKVCache(NB, BS, HKV // world, D, device="cpu", max_batch=4,
                             max_blocks_per_seq=MB, stream=0, lockstep_group=dist.group.WORLD)
        for sid in range(3):
            prompt = [sid] * (5 + (rank if diverge and sid == 2 else 0))
            cache.add_sequence(sid, prompt)
        outcome = "ok"
        try:
            for step in range(3):
                cache.begin_step([0, 1, 2], [step] * 3)
        except RuntimeError as e:
            outcome = "lockstep" if "lockstep" in str(e) else repr(e)
        q.put((rank, outcome))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("diverge", [False, True])
def test_lockstep_check_over_two_ranks(diverge):
    """Each rank drives its own block manager; the per-step digest exchange
    passes when they agree and fails on every rank when one placed a prompt
    differently."""
    import os
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + os.getpid() % 200 + (100 if diverge else 0)
    procs = [ctx.Process(target=_lockstep_worker, args=(r, 2, port, diverge, q))
             for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o for _, o in res] == (["lockstep", "lockstep"] if diverge else ["ok", "ok"])


def _random_loop(oracle_mod, monkeypatch, seed):
    """One randomized serving loop through PagedKVCache on the oracle stand-in:
    random shapes, block size and mode; admissions (some served entirely from
    the prefix cache), forks and frees between steps. The expected history of
    a sequence's cached prefix is what was last stored in its slots (a model of
    every slot's contents: prompt stores, copies, appends)."""
    rng = np.random.default_rng(seed)
    lib = OracleLib(oracle_mod)
    monkeypatch.setattr(B, "load_library", lambda *a, **k: lib)
    monkeypatch.setattr(B, "_on_device", lambda t: True)
    bs, hkv, d = int(rng.choice([1, 4, 16])), int(rng.choice([1, 2])), 64
    hq, layers = hkv * int(rng.choice([1, 2, 4])), int(rng.integers(1, 3))
    mode = ["fused", "prefix", "window"][seed % 3]
    window = int(rng.integers(1, 30)) if mode == "window" else 0
    cache = PagedKVCache(400, bs, hkv, d, num_layers=layers, device="cpu", max_batch=8,
                         max_blocks_per_seq=256, stream=0, window=window,
                         shared_prefix_min_blocks=int(rng.integers(1, 3)) if mode == "prefix"
                         else 0)
    for l in range(layers):
        lib.reg(cache.k[l], cache.v[l])
    lib.reg(cache._d_slots, cache._d_tables, cache._d_lens)
    half = lambda *s: torch.from_numpy(rng.standard_normal(s).astype(np.float16))
    hist, content, live, nxt = {}, {}, [], 0
    system = [int(x) for x in rng.integers(0, 4, size=int(rng.integers(0, 3 * bs + 2)))]

    def admit():
        nonlocal nxt
        toks = system + [int(x) for x in rng.integers(0, 4, size=int(rng.integers(1, 2 * bs + 3)))]
        cached, slots = cache.add_sequence(nxt, toks)
        lib.reg(slots)
        pre = cache.bm.slots(nxt, 0, cached) if cached else []
        for l in range(layers):
            K0 = np.array([content[(l, int(x))][0] for x in pre]).reshape(-1, hkv, d)
            V0 = np.array([content[(l, int(x))][1] for x in pre]).reshape(-1, hkv, d)
            k, v = half(len(toks) - cached, hkv, d), half(len(toks) - cached, hkv, d)
            lib.reg(k, v)
            cache.store_prompt(l, slots, k, v)
            for j, x in enumerate(slots.tolist()):
                content[(l, x)] = (k[j].double().numpy(), v[j].double().numpy())
            hist[(nxt, l)] = (np.concatenate([K0, k.double().numpy()]),
                              np.concatenate([V0, v.double().numpy()]))
        live.append(nxt)
        nxt += 1

    for _ in range(int(rng.integers(2, 5))):
        admit()
    for step in range(10):
        r = rng.random()
        if r < 0.15 and len(live) < 7:
            admit()
        elif r < 0.3 and len(live) < 7:
            p = live[int(rng.integers(0, len(live)))]
            cache.fork(p, nxt)
            for l in range(layers):
                hist[(nxt, l)] = tuple(x.copy() for x in hist[(p, l)])
            live.append(nxt)
            nxt += 1
        elif r < 0.4 and len(live) > 2:
            cache.free_sequence(live.pop(int(rng.integers(0, len(live)))))
        ids = [int(x) for x in rng.permutation(live)]
        plan = cache.begin_step(ids, [int(x) for x in rng.integers(0, 4, size=len(ids))])
        for l in range(layers):
            for src, dst in plan.copy_pairs.tolist():
                for row in range(bs):
                    if (l, src * bs + row) in content:
                        content[(l, dst * bs + row)] = content[(l, src * bs + row)]
            n = len(ids)
            q, k, v = half(n, hq, d), half(n, hkv, d), half(n, hkv, d)
            out = torch.empty((n, hq, d), dtype=torch.float16)
            lib.reg(q, k, v, out)
            cache.attend(plan, l, q, k, v, out=out)
            got = lib.f64[out.data_ptr()]
            for i, x in enumerate(plan.slot_mapping.tolist()):
                content[(l, x)] = (k[i].double().numpy(), v[i].double().numpy())
            for i, sid in enumerate(ids):
                K = np.concatenate([hist[(sid, l)][0], k[i:i + 1].double().numpy()])
                V = np.concatenate([hist[(sid, l)][1], v[i:i + 1].double().numpy()])
                hist[(sid, l)] = (K, V)
                for h in range(hq):
                    want = direct_attention(q[i, h].double().numpy(), K[:, h // (hq // hkv)],
                                            V[:, h // (hq // hkv)], np.float32(1 / np.sqrt(d)),
                                            window)
                    np.testing.assert_allclose(got[i, h], want, rtol=0, atol=1e-9,
                                               err_msg=f"seed {seed} step {step} layer {l}")


@pytest.mark.parametrize("seed", range(24))
def test_random_serving_loops_match_attention_over_each_history(oracle_mod, monkeypatch, seed):
    _random_loop(oracle_mod, monkeypatch, seed)
