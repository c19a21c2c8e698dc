"""GPU parity of pa_decode_sliding_window against the float64 oracle (which
attends to tokens [max(0, L - window), L) by its own gather)."""
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


def run_window(w, window, partition_tokens=0):
    step = DecodeStep(w, "cuda", partition_tokens=partition_tokens, window=window)
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    _, _, want = oracle_step(w, window=window)
    got = step.out_f64()
    err = max_abs_err(got, want)
    assert err <= TOL[w.io_dtype], f"window {window}: max abs err {err}"
    return step, got


@pytest.mark.parametrize("window", [1, 2, 15, 16, 17, 100, 513, 5000])
def test_windows(window):
    w = W.custom([1, 7, 16, 17, 40, 300, 1030], num_q_heads=8, num_kv_heads=2, head_dim=128,
                 dtype="bf16", seed=window)
    run_window(w, window)


@pytest.mark.parametrize("bs", [1, 4, 32, 128])
def test_block_sizes(bs):
    w = W.custom([5, 33, 200, 777], num_q_heads=4, num_kv_heads=4, head_dim=64, block_size=bs,
                 seed=bs)
    run_window(w, 45)


@pytest.mark.parametrize("pt", [16, 64, 0])
def test_partitions(pt):
    w = W.llama2_7b(batch=3, min_len=2000, max_len=3000)
    run_window(w, 1000, partition_tokens=pt)


def test_long_context_window_4096():
    w = W.long_context(batch=1, context_len=20000)
    run_window(w, 4096)


def test_fp8_cache():
    w = W.fp8_beams(batch=24, beam_groups=2, block_size=16)
    run_window(w, 300)


def test_blocks_before_the_window_are_never_read():
    w = W.custom([100, 250, 64], num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16)
    step, got = run_window(w, 40)
    # a caller that freed the blocks before the window may leave any value there
    bad = step.block_tables.clone()
    for b, L in enumerate(w.context_lens.tolist()):
        first = max(0, L - 40) // 16
        bad[b, :first] = -7
    out = torch.empty_like(step.out)
    B.pa_decode_sliding_window(step.q, step.k_cache, step.v_cache, bad, step.context_lens,
                               float(w.scale), out, step.cache, step.max_context, 40,
                               workspace=step.workspace)
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    assert torch.equal(out, step.out)
