"""The Python binding's marshalling, on the CPU: every wrapper forwards the
tensors' addresses, sizes and dtypes to the C entry point of the same name,
and refuses tensors whose layout the library cannot check itself
(non-contiguous views, wrong index dtypes, tables shorter than the batch,
caches that do not match their descriptor). The library is replaced by a
recorder and the device test by a stub, so no GPU and no kernel is involved.
"""
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B


class Recorder:
    """Stands in for libpagedattn.so: records each call's arguments."""

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
    monkeypatch.setattr(B, "_on_device", lambda t: True)  # CPU tensors stand in
    return r


NB, BS, HKV, D, HQ, BATCH, MB = 12, 16, 2, 64, 4, 3, 5


def _inputs(dtype=torch.float16):
    cache = B.PagedCache(NB, BS, HKV, D, dtype)
    kc = torch.zeros((NB, BS, HKV, D), dtype=dtype)
    vc = torch.zeros_like(kc)
    q = torch.zeros((BATCH, HQ, D), dtype=dtype)
    bt = torch.zeros((BATCH, MB), dtype=torch.int32)
    lens = torch.ones(BATCH, dtype=torch.int32)
    out = torch.empty_like(q)
    return cache, kc, vc, q, bt, lens, out


def test_decode_forwards_addresses_and_sizes(rec):
    cache, kc, vc, q, bt, lens, out = _inputs()
    ws = torch.empty(1000, dtype=torch.uint8)
    B.pa_decode(q, kc, vc, bt, lens, 0.125, out, cache, 40, 64, ws, stream=7)
    name, a = rec.calls[-1]
    assert name == "pa_decode"
    assert a[0] == q.data_ptr() and a[1] == B.PA_F16 and a[2:4] == (BATCH, HQ)
    assert a[4] == kc.data_ptr() and a[5] == vc.data_ptr()
    d = a[6]._obj
    assert (d.num_blocks, d.block_size, d.num_kv_heads, d.head_dim) == (NB, BS, HKV, D)
    assert a[7] == bt.data_ptr() and a[8] == MB and a[9] == lens.data_ptr() and a[10] == 40
    assert a[11] == 0.125 and a[12] == out.data_ptr() and a[13] == 64
    assert a[14] == ws.data_ptr() and a[15] == 1000 and a[16] == 7


def test_every_decode_variant_takes_the_same_checks(rec):
    cache, kc, vc, q, bt, lens, out = _inputs(torch.bfloat16)
    knew = torch.zeros((BATCH, HKV, D), dtype=torch.bfloat16)
    slots = torch.zeros(BATCH, dtype=torch.int64)
    B.pa_decode_shared_prefix(q, kc, vc, bt, lens, 0.1, out, cache, 64, 2, stream=0)
    B.pa_decode_sliding_window(q, kc, vc, bt, lens, 0.1, out, cache, 64, 32, stream=0)
    B.pa_decode_static_workspace(q, kc, vc, bt, lens, 0.1, out, cache, 64, stream=0)
    B.pa_append_decode(q, knew, knew.clone(), slots, kc, vc, bt, lens, 0.1, out, cache, 64,
                       stream=0)
    names = [n for n, _ in rec.calls]
    assert names == ["pa_decode_shared_prefix", "pa_decode_sliding_window",
                     "pa_decode_static_workspace", "pa_append_decode"]
    for _, a in rec.calls:
        assert a[0] == q.data_ptr() and a[-1] == 0
    bad_tables = bt.to(torch.int64)
    for call in (
        lambda: B.pa_decode_shared_prefix(q, kc, vc, bad_tables, lens, 0.1, out, cache, 64, 2),
        lambda: B.pa_decode_sliding_window(q, kc, vc, bt[:2], lens, 0.1, out, cache, 64, 32),
        lambda: B.pa_decode_static_workspace(q, kc, vc, bt, lens[:2], 0.1, out, cache, 64),
        lambda: B.pa_append_decode(q, knew, knew.clone(), slots[:2], kc, vc, bt, lens, 0.1, out,
                                   cache, 64),
    ):
        with pytest.raises((TypeError, ValueError)):
            call()
    assert len(rec.calls) == 4  # nothing reached the library


@pytest.mark.parametrize("case", ["q_view", "tables_dtype", "tables_short", "lens_dtype",
                                  "out_dtype", "out_shape", "cache_blocks", "cache_dtype",
                                  "cache_view", "head_dim"])
def test_decode_rejects_what_the_library_cannot_check(rec, case):
    cache, kc, vc, q, bt, lens, out = _inputs()
    if case == "q_view":
        q = torch.zeros((HQ, BATCH, D), dtype=torch.float16).transpose(0, 1)
    elif case == "tables_dtype":
        bt = bt.to(torch.int64)
    elif case == "tables_short":
        bt = bt[:BATCH - 1]
    elif case == "lens_dtype":
        lens = lens.to(torch.int64)
    elif case == "out_dtype":
        out = out.to(torch.bfloat16)
    elif case == "out_shape":
        out = out[:, :2]
    elif case == "cache_blocks":
        kc = kc[:NB - 1]
    elif case == "cache_dtype":
        vc = vc.to(torch.bfloat16)
    elif case == "cache_view":
        kc = torch.zeros((NB, HKV, BS, D), dtype=torch.float16).transpose(1, 2)
    elif case == "head_dim":
        q = torch.zeros((BATCH, HQ, 128), dtype=torch.float16)
        out = torch.empty_like(q)
    with pytest.raises((TypeError, ValueError)):
        B.pa_decode(q, kc, vc, bt, lens, 0.1, out, cache, 40, stream=0)
    assert rec.calls == []


def test_append_and_copy_checks(rec):
    cache, kc, vc, *_ = _inputs()
    k = torch.zeros((6, HKV, D), dtype=torch.float16)
    slots = torch.arange(6, dtype=torch.int64)
    B.pa_append_kv(k, k.clone(), slots, kc, vc, cache, stream=0)
    name, a = rec.calls[-1]
    assert name == "pa_append_kv" and a[2] == B.PA_F16 and a[3] == 6
    for bad in (dict(slots=slots.to(torch.int32)), dict(slots=slots[:5]),
                dict(v=k.to(torch.bfloat16)), dict(k=k[:, :1])):
        kk, vv, ss = bad.get("k", k), bad.get("v", k.clone()), bad.get("slots", slots)
        with pytest.raises((TypeError, ValueError)):
            B.pa_append_kv(kk, vv, ss, kc, vc, cache, stream=0)
    B.pa_copy_blocks([[1, 2]], kc, vc, cache, stream=0)
    assert rec.calls[-1][0] == "pa_copy_blocks" and rec.calls[-1][1][1] == 1
    B.pa_copy_blocks_layers([[1, 2], [3, 4]], [kc, kc.clone()], [vc, vc.clone()], cache,
                            stream=0)
    name, a = rec.calls[-1]
    assert name == "pa_copy_blocks_layers" and a[1] == 2 and a[4] == 2
    assert a[2][0] == kc.data_ptr() and a[3][0] == vc.data_ptr()
    with pytest.raises(ValueError):
        B.pa_copy_blocks_layers([[1, 2]], [kc, kc[:3]], [vc, vc], cache, stream=0)


def test_e4m3_scales_are_checked(rec):
    sc = torch.ones((HKV, D), dtype=torch.float32)
    cache = B.PagedCache(NB, BS, HKV, D, torch.uint8, sc, sc, sc, sc)
    kc = torch.zeros((NB, BS, HKV, D), dtype=torch.uint8)
    k = torch.zeros((2, HKV, D), dtype=torch.float16)
    B.pa_append_kv(k, k, torch.zeros(2, dtype=torch.int64), kc, kc.clone(), cache, stream=0)
    d = rec.calls[-1][1][7]._obj
    assert d.cache_dtype == B.PA_E4M3 and d.k_scale == sc.data_ptr()
    for bad in (sc.reshape(-1), sc.double(), sc.t()):
        cache = B.PagedCache(NB, BS, HKV, D, torch.uint8, bad, sc, sc, sc)
        with pytest.raises((TypeError, ValueError)):
            B.pa_append_kv(k, k, torch.zeros(2, dtype=torch.int64), kc, kc.clone(), cache,
                           stream=0)


def test_cpu_tensors_are_refused_without_the_stub(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(B, "load_library", lambda *a, **k: r)
    cache, kc, vc, q, bt, lens, out = _inputs()
    with pytest.raises(ValueError):
        B.pa_decode(q, kc, vc, bt, lens, 0.1, out, cache, 40, stream=0)
    assert r.calls == []


def _families():
    from paged_kv_cache_410_b200 import workloads as W
    fp8 = W.fp8_beams(batch=24, beam_groups=2, median_len=40, max_len=200, min_len=16)
    return [
        ("tiny_mha", W.tiny_mha(), {}),
        ("gqa_bf16", W.custom([5, 40, 77], num_q_heads=8, num_kv_heads=2, head_dim=128,
                              dtype="bf16"), {}),
        ("window", W.custom([5, 40, 77], num_q_heads=8, num_kv_heads=2, head_dim=128),
         {"window": 32}),
        ("fused", W.custom([5, 40, 77], num_q_heads=8, num_kv_heads=2, head_dim=128),
         {"fused": True}),
        ("prefix", W.custom_shared_prefix(64, [10, 20, 30]), {"shared_prefix_blocks": 4}),
        ("fp8_beams", fp8, {}),
        ("fp8_subset", W.subset(fp8, [0, 5, 9, 20]), {"fused": True}),
        # the workloads of __graft_entry__.smoke()
        ("smoke_fp8", W.fp8_beams(batch=12, beam_groups=1, block_size=16), {}),
        ("smoke_prefix", W.custom_shared_prefix(128, [0, 5, 40, 300], num_q_heads=8,
                                                num_kv_heads=2, head_dim=128, block_size=16,
                                                dtype="bf16", seed=7),
         {"shared_prefix_blocks": 8}),
    ]


@pytest.mark.parametrize("name,w,kw", _families(), ids=lambda x: x if isinstance(x, str) else "")
def test_decode_step_of_every_workload_passes_the_checks(rec, name, w, kw):
    """The serving-step driver hands the library tensors the checks accept,
    for every workload family and path."""
    from paged_kv_cache_410_b200.session import DecodeStep
    step = DecodeStep(w, "cpu", stream=0, **kw)
    rec.calls.clear()
    step.run()
    names = [n for n, _ in rec.calls]
    decode = ("pa_append_decode" if kw.get("fused") else
              "pa_decode_shared_prefix" if kw.get("shared_prefix_blocks") else
              "pa_decode_sliding_window" if kw.get("window") else "pa_decode")
    assert names[-1] == decode
    assert ("pa_append_kv" in names) == (not kw.get("fused"))
    assert ("pa_copy_blocks" in names) == bool(len(w.copy_pairs))
