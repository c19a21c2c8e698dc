"""GPU parity of pa_decode_shared_prefix (cascade decode over a prefix every
sequence shares) against the float64 oracle, which knows nothing of the
sharing: it gathers every sequence's blocks on its own."""
import numpy as np
import pytest
import torch

from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200 import workloads as W
from paged_kv_cache_410_b200.session import DecodeStep, to_bits

from helpers import TOL, max_abs_err, oracle_step

pytestmark = pytest.mark.gpu


def run_cascade(w, prefix_blocks, partition_tokens=0, check_caches=True):
    step = DecodeStep(w, "cuda", partition_tokens=partition_tokens,
                      shared_prefix_blocks=prefix_blocks)
    step.run()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    kc, vc, want = oracle_step(w)
    if check_caches:
        assert np.array_equal(to_bits(step.k_cache), kc)
        assert np.array_equal(to_bits(step.v_cache), vc)
    got = step.out_f64()
    err = max_abs_err(got, want)
    assert err <= TOL[w.io_dtype], f"{w.name}: max abs err {err}"
    return step, got


def test_70b_shaped_prefix_batch():
    w = W.llama2_70b_prefix(batch=6)
    run_cascade(w, w.meta["shared_prefix_blocks"])


def test_many_row_tiles():
    # 44 sequences x group 8 = 352 query rows per KV head: three 128-row
    # tiles of the tensor-core prefix kernel, the last one ragged
    w = W.llama2_70b_prefix(batch=44, prefix_len=640, max_suffix=300)
    run_cascade(w, w.meta["shared_prefix_blocks"], check_caches=False)


@pytest.mark.parametrize("pt", [16, 128, 0])
def test_suffix_partitions(pt):
    w = W.llama2_70b_prefix(batch=4, max_suffix=900)
    run_cascade(w, w.meta["shared_prefix_blocks"], partition_tokens=pt, check_caches=False)


@pytest.mark.parametrize("prefix,suffixes,hq,hkv,d,bs,dtype", [
    (64, [0, 1, 15, 16, 17, 300], 8, 2, 64, 16, "f16"),     # a sequence ends at the prefix
    (48, [1, 2, 3, 50], 32, 2, 128, 1, "bf16"),             # block size 1, group of 16
    (96, [5, 40, 97], 32, 1, 128, 32, "f16"),               # MQA: two head groups
    (1536, [1, 700, 2000], 12, 4, 128, 128, "bf16"),        # 3 prefix chunks, group of 3
    (16, [3] * 70, 8, 8, 64, 16, "f16"),                    # many sequences, one block
])
def test_shapes(prefix, suffixes, hq, hkv, d, bs, dtype):
    w = W.custom_shared_prefix(prefix, suffixes, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                               block_size=bs, dtype=dtype, seed=prefix + hq + bs)
    step, got = run_cascade(w, w.meta["shared_prefix_blocks"])
    # same numbers as the plain entry point
    plain = DecodeStep(w, "cuda")
    plain.run()
    torch.cuda.synchronize()
    assert max_abs_err(plain.out_f64(), got) <= TOL[w.io_dtype]


def test_fp8_cache_one_beam_group():
    # 16 beams of one prompt share its full blocks: a shared prefix in an E4M3 cache
    w = W.fp8_beams(batch=16, beam_groups=1, beam_width=16, block_size=16, min_len=300)
    prefix_blocks = (int(w.meta["group_lens"][0]) - 1) // w.block_size
    assert prefix_blocks > 0
    run_cascade(w, prefix_blocks)


def test_sequences_not_starting_with_the_prefix_are_flagged():
    w = W.custom_shared_prefix(64, [10, 20, 30], num_q_heads=4, num_kv_heads=4, head_dim=64)
    step = DecodeStep(w, "cuda", shared_prefix_blocks=4)
    bad = step.block_tables.clone()
    bad[2, 1] = bad[2, 4]  # sequence 2 no longer starts with the shared blocks
    B.pa_decode_shared_prefix(step.q, step.k_cache, step.v_cache, bad, step.context_lens,
                              float(w.scale), step.out, step.cache, step.max_context, 4,
                              workspace=step.workspace)
    assert step.device_errors() & B.DEVERR_PREFIX
    short = step.context_lens.clone()
    short[0] = 63  # shorter than the prefix
    B.pa_decode_shared_prefix(step.q, step.k_cache, step.v_cache, step.block_tables, short,
                              float(w.scale), step.out, step.cache, step.max_context, 4,
                              workspace=step.workspace)
    assert step.device_errors() & B.DEVERR_PREFIX
    B.pa_decode_shared_prefix(step.q, step.k_cache, step.v_cache, step.block_tables,
                              step.context_lens, float(w.scale), step.out, step.cache,
                              step.max_context, 4, workspace=step.workspace)
    assert step.device_errors() == 0


def test_dirty_workspace_and_repeat():
    # the prefix and suffix partials live in the caller's workspace: garbage
    # left in it changes nothing, and repeated calls agree bit for bit
    w = W.llama2_70b_prefix(batch=20, prefix_len=512, max_suffix=700)
    step, got = run_cascade(w, w.meta["shared_prefix_blocks"], check_caches=False)
    first = step.out.clone()
    for fill in (0x00, 0x5A, 0xFF):
        step.workspace.fill_(fill)
        step.decode()
        torch.cuda.synchronize()
        assert step.device_errors() == 0
        assert torch.equal(step.out, first)


def test_cuda_graph_capture_and_replay():
    # the 16-bit cascade chains its prefix, suffix and merge kernels on the
    # caller's stream as programmatic dependents: captured from that stream it
    # must replay to the eager result
    w = W.llama2_70b_prefix(batch=16, prefix_len=512, max_suffix=600)
    step, _ = run_cascade(w, w.meta["shared_prefix_blocks"], check_caches=False)
    eager = step.out.clone()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step.decode()  # warm up on the capture stream (plans, smem attributes)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    step.out.zero_()
    with torch.cuda.graph(graph):
        step.decode()
    graph.replay()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    assert torch.equal(step.out, eager)
    # plain split-K decode of the same batch, captured too
    plain = DecodeStep(w, "cuda", partition_tokens=64)
    plain.run()
    torch.cuda.synchronize()
    want = plain.out.clone()
    g2 = torch.cuda.CUDAGraph()
    plain.out.zero_()
    with torch.cuda.graph(g2):
        plain.decode()
    g2.replay()
    torch.cuda.synchronize()
    assert torch.equal(plain.out, want)


def test_prefix_wait_timeout_is_reported_and_recoverable():
    # the test hook withholds the tensor-core prefix kernel's scores: its
    # softmax warps' bounded waits run out (1 s), the CTA drains and the
    # device error word reports PA_DEVERR_TIMEOUT; afterwards the context
    # is still usable and a normal call matches the oracle
    w = W.custom_shared_prefix(128, [3, 20], num_q_heads=8, num_kv_heads=1, head_dim=128,
                               block_size=16, dtype="bf16", seed=3)
    step = DecodeStep(w, "cuda", shared_prefix_blocks=w.meta["shared_prefix_blocks"])
    step.copy()
    step.append()
    B.pa_testing_withhold_prefix_scores(1)
    try:
        step.decode()
        torch.cuda.synchronize()
        assert step.device_errors() & B.DEVERR_TIMEOUT
    finally:
        B.pa_testing_withhold_prefix_scores(0)
    step.decode()
    torch.cuda.synchronize()
    assert step.device_errors() == 0
    _, _, want = oracle_step(w)
    assert max_abs_err(step.out_f64(), want) <= TOL["bf16"]
