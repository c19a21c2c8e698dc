"""Host-side logic of bench.py on the CPU: the multi-rank reductions over a
2-rank gloo group, per-rank workloads, and the reference (CPU oracle) arm."""
import argparse
import json
import os
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.make_workload("tiny_mha", rank, None)
        got_max = bench.max_over_ranks(10.0 + rank)
        got_sum = bench.sum_over_ranks(float(w.batch))
        q.put((rank, got_max, got_sum, int(w.context_lens.sum())))
    finally:
        dist.destroy_process_group()


def test_rank_reductions_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]     # max over ranks, seen by every rank
    assert [r[2] for r in res] == [8.0, 8.0]       # 4 sequences per rank
    assert res[0][3] != res[1][3]                  # ranks draw different batches


def test_rank_seed_offsets_are_distinct():
    a = bench.make_workload("llama2_7b", 0, 2)
    b = bench.make_workload("llama2_7b", 1, 2)
    assert not np.array_equal(a.context_lens, b.context_lens)


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_mha", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, PYTHONPATH=ROOT, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_mha", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_on_the_fp8_beams_workload():
    # E4M3 cache: the oracle fills its own cache from the history tokens, then
    # times copies + append + decode
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "fp8_beams", "--batch", "64", "--steps", "2",
                        "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["config"]["kv_cache_dtype"] == "e4m3"


def test_oracle_step_covers_copies_append_and_decode():
    from paged_kv_cache_410_b200 import workloads as W
    w = W.fp8_beams(batch=24, beam_groups=2, median_len=40, max_len=200)
    t, s, out = bench.oracle_step_time(w, np.arange(8))
    assert out.shape == (8, w.num_q_heads, w.head_dim) and np.isfinite(out).all()
    assert t > 0 and s.batch == 8 and len(s.copy_pairs) == len(w.copy_pairs)
    kc, vc = bench.oracle_caches(w)
    assert kc.dtype == np.uint8 and kc.any()              # filled by the oracle's append
    assert bench.oracle_caches(w)[0] is kc                # made once per workload


def test_parity_summary_against_the_oracle_sample():
    """The bench line's parity check: the oracle's output for the cpu_baseline
    sample, compared with the device output of the same sequences."""
    import oracle
    from paged_kv_cache_410_b200 import workloads as W
    w = W.custom([5, 40, 77, 130], num_q_heads=8, num_kv_heads=2, head_dim=64)
    cb, seqs, want = bench.cpu_baseline(w, target_s=0.2, window=32)
    assert cb["kind"] == "oracle" and len(seqs) == 4
    # the sample's output is the oracle's windowed decode after the append
    kc, vc = bench.oracle_caches(w)
    direct = oracle.decode(w.q, "f16", kc, vc, "f16", w.block_tables, w.context_lens, w.scale,
                           window=32)
    assert np.array_equal(want, direct[seqs])
    ok = bench.parity_summary(want + 1e-3, want, "f16")
    assert ok["ok"] and abs(ok["max_abs_err"] - 1e-3) < 1e-12 and ok["sequences"] == 4
    bad = bench.parity_summary(want + 3e-3, want, "f16")
    assert not bad["ok"] and bad["tolerance"] == 2e-3
    assert bench.parity_summary(want + 3e-3, want, "bf16")["ok"]
    nan = want.copy()
    nan[0, 0, 0] = np.nan
    r = bench.parity_summary(nan, want, "f16")
    assert r["max_abs_err"] is None and not r["ok"]


def test_small_fp8_batches_scale_the_beam_groups():
    from paged_kv_cache_410_b200 import workloads as W
    orig = W.normal_bits
    W.normal_bits = lambda rng, shape, dtype, chunk=0: np.zeros(shape, np.uint16)
    try:
        w = bench.make_workload("fp8_beams", 0, 24)
        assert w.batch == 24 and w.meta["beam_groups"] == 6
        assert bench.make_workload("fp8_beams", 0, 256).meta["beam_groups"] == 16
    finally:
        W.normal_bits = orig


def test_reference_arm_config_equals_the_gpu_arms():
    """Both arms describe the same workload with the same config object, the
    decode path included, so that their lines can be compared key for key."""
    env = dict(os.environ, PYTHONPATH=ROOT)
    for extra in ([], ["--no-flush"]):
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                            "--workload", "tiny_mha", "--steps", "2", "--warmup", "3", *extra],
                           capture_output=True, text=True, env=env, timeout=300)
        assert r.returncode == 0, r.stderr
        d = json.loads(r.stdout.strip().splitlines()[-1])
        args = argparse.Namespace(steps=2, warmup=3, cascade="auto", window=0, fused=False,
                                  no_flush=bool(extra))
        w = bench.make_workload("tiny_mha", 0, None)
        want = bench.base_line(args, w, 1, bench.cascade_blocks(args, w))["config"]
        assert d["config"] == want
        assert d["config"]["decode"] == "whole history"
        assert d["config"]["l2"].startswith("not flushed" if extra else "flushed")


def test_cascade_label_for_the_shared_prefix_family():
    from paged_kv_cache_410_b200 import workloads as W
    w = W.custom_shared_prefix(64, [0, 5, 40], num_q_heads=8, num_kv_heads=2, head_dim=64,
                               block_size=16, dtype="bf16", seed=3)
    auto = argparse.Namespace(cascade="auto", window=0, fused=False)
    assert bench.cascade_blocks(auto, w) == 4
    assert bench.decode_label(auto, 4) == "shared-prefix cascade (4 blocks)"
    for other in (argparse.Namespace(cascade="off", window=0, fused=False),
                  argparse.Namespace(cascade="auto", window=64, fused=False),
                  argparse.Namespace(cascade="auto", window=0, fused=True)):
        assert bench.cascade_blocks(other, w) == 0


def test_parity_sample_takes_the_extremes_and_a_beam_group():
    from paged_kv_cache_410_b200 import workloads as W
    w = W.fp8_beams(batch=40, beam_groups=3, median_len=40, max_len=200)
    s = bench.parity_sample(w, 12)
    assert len(s) == len(set(s.tolist())) and np.all(np.diff(s) > 0)
    assert {0, 1, 2, 3} <= set(s.tolist())
    assert int(np.argmin(w.context_lens)) in s and int(np.argmax(w.context_lens)) in s
    assert len(s) <= 12 + 2
    assert np.array_equal(bench.parity_sample(w, 100), np.arange(40))
