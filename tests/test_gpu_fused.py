"""GPU parity of pa_append_decode (append of each sequence's new token and
paged decode in one launch) against the float64 oracle's append followed by
its decode, and against the library's own two separate calls."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep, to_bits

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


def fused_vs_oracle(w, partition_tokens=0):
    step = DecodeStep(w, "cuda", partition_tokens=partition_tokens, fused=True)
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    kc, vc, want = oracle_step(w)
    err = max_abs_err(step.out_f64(), want)
    assert err <= TOL[w.io_dtype], f"max abs err {err}"
    assert np.array_equal(to_bits(step.k_cache), kc)
    assert np.array_equal(to_bits(step.v_cache), vc)
    return step


def separate(w, partition_tokens=0):
    step = DecodeStep(w, "cuda", partition_tokens=partition_tokens)
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    return step


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("bs", [1, 4, 16, 32])
def test_16bit(dtype, bs):
    w = W.custom([1, 2, 15, 16, 17, 64, 300, 1030], num_q_heads=8, num_kv_heads=2,
                 head_dim=128, block_size=bs, dtype=dtype, seed=bs)
    fused_vs_oracle(w)


@pytest.mark.parametrize("pt", [16, 48, 0])
def test_partitions(pt):
    w = W.llama2_7b(batch=3, min_len=1000, max_len=2500)
    fused_vs_oracle(w, partition_tokens=pt)


def test_head_dim_64_mha():
    w = W.custom([3, 40, 129], num_q_heads=4, num_kv_heads=4, head_dim=64, seed=3)
    fused_vs_oracle(w)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_fp8_beams(bs):
    w = W.fp8_beams(batch=24, beam_groups=2, block_size=bs)
    fused_vs_oracle(w)


@pytest.mark.parametrize("make", [
    lambda: W.custom([1, 16, 17, 300, 1030], num_q_heads=8, num_kv_heads=2, head_dim=128,
                     dtype="bf16", seed=9),
    lambda: W.fp8_beams(batch=24, beam_groups=2, block_size=16),
    lambda: W.llama2_7b(batch=4, min_len=3000, max_len=4000),
])
def test_bitwise_equal_to_separate_calls(make):
    w = make()
    a = fused_vs_oracle(w)
    b = separate(w)
    assert torch.equal(a.out, b.out)
    assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.v_cache, b.v_cache)


def test_padding_slots_decode_only():
    w = W.custom([5, 33, 200, 777], num_q_heads=8, num_kv_heads=2, head_dim=128, seed=4)
    w.slot_mapping[[1, 3]] = -1          # no new token for these: the cache row is used
    step = fused_vs_oracle(w)
    plain = DecodeStep(w, "cuda")
    plain.copy()
    plain.append()                       # pa_append_kv skips the same -1 slots
    plain.decode()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    assert torch.equal(step.out, plain.out)


def test_wrong_slot_is_flagged_and_not_stored():
    w = W.custom([20, 40], num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16, seed=6)
    step = DecodeStep(w, "cuda", fused=True)
    before_k = step.k_cache.clone()
    bad = step.slot_mapping.clone()
    bad[0] += 1                          # not the slot of position L - 1
    B.pa_append_decode(step.q, step.k_new, step.v_new, bad, step.k_cache, step.v_cache,
                       step.block_tables, step.context_lens, float(w.scale), step.out,
                       step.cache, step.max_context, workspace=step.workspace)
    torch.cuda.synchronize()
    assert step.device_errors() & B.DEVERR_SLOT
    changed = (step.k_cache != before_k).reshape(w.num_blocks * w.block_size, -1).any(dim=1)
    # only sequence 1's slot was written
    assert changed.nonzero().flatten().tolist() == [int(w.slot_mapping[1])]
    assert step.device_errors() == 0     # the word was cleared


def test_mismatched_dtypes_rejected_on_host():
    w = W.custom([8], num_q_heads=8, num_kv_heads=2, head_dim=128, dtype="f16", seed=1)
    step = DecodeStep(w, "cuda", fused=True)
    with pytest.raises(TypeError):
        B.pa_append_decode(step.q, step.k_new.to(torch.bfloat16), step.v_new, step.slot_mapping,
                           step.k_cache, step.v_cache, step.block_tables, step.context_lens,
                           float(w.scale), step.out, step.cache, step.max_context,
                           workspace=step.workspace)
