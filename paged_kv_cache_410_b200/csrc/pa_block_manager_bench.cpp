// Host benchmark of the block manager (include/pa_block_manager.h): the work
// a decode engine does around the kernels at every step, timed with the
// steady clock on one host thread.
//
//   admit:  `batch` requests whose prompts start with the same system prompt
//           (`prompt` tokens) followed by `own` tokens of their own; with the
//           prefix cache on, every request after the first reuses the system
//           prompt's full blocks;
//   step:   one token per sequence (slot, copy-on-write pairs after forks),
//           then the batch's block tables and lengths (pa_bm_block_tables,
//           the layout pa_decode reads), and the same through
//           pa_bm_block_tables_update into arrays kept across steps (only
//           rows whose block list changed are rewritten);
//   churn:  every `churn` steps, 4 sequences fork a beam and 4 beams end.
//
// The whole loop runs twice on fresh managers: once with one
// pa_bm_append_token call per sequence, once with one pa_bm_append_tokens
// call per step. Both passes must hand out the same slots and copy-on-write
// pairs at every step (compared through a per-step hash).
//
// Usage: pa_block_manager_bench [batch steps prompt own block_size churn]
// Prints one JSON line; `step_us` is the per-token appends plus the
// incremental export, `step_us_full_tables` the appends plus the full one.
// Exits non-zero if the two exports, or the two passes, ever differ.
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "pa_block_manager.h"

namespace {

double now_us() {
  using namespace std::chrono;
  return duration<double, std::micro>(steady_clock::now().time_since_epoch()).count();
}

int arg(int argc, char** argv, int i, int dflt) { return argc > i ? std::atoi(argv[i]) : dflt; }

struct Args {
  int batch, steps, prompt, own, bs, churn;
};

struct Pass {
  double admit_us = 0, append_us = 0, tables_us = 0, update_us = 0, churn_us = 0;
  int64_t cached_total = 0, appends = 0, cow_pairs = 0, forks = 0, rewritten = 0, free_left = 0;
  std::vector<uint64_t> step_hash;  // slots and copy pairs handed out at each step
};

uint64_t mix(uint64_t h, uint64_t v) { return (h ^ v) * 1099511628211ull; }

// One serving run on a fresh manager; returns 0 or a failure code.
int serve(const Args& a, bool batched, Pass& out) {
  const int max_len = a.prompt + a.own + a.steps;
  const int max_blocks = (max_len + a.bs - 1) / a.bs;
  // the shared prompt once, every sequence's own tokens, the beams' copies
  const int64_t num_blocks =
      static_cast<int64_t>(a.prompt / a.bs + 2) +
      static_cast<int64_t>(a.batch + 8) * ((a.own + a.steps + a.bs - 1) / a.bs + 2) * 2;
  pa_block_manager* bm = pa_bm_create(num_blocks, a.bs, 1);
  if (!bm) return 3;

  // ---- admit ----------------------------------------------------------------
  std::vector<int32_t> tokens(a.prompt + a.own);
  for (int i = 0; i < a.prompt; ++i) tokens[i] = 1000 + i;
  std::vector<int64_t> seqs(a.batch);
  const double t_admit = now_us();
  for (int b = 0; b < a.batch; ++b) {
    for (int i = 0; i < a.own; ++i) tokens[a.prompt + i] = 100000 + b * a.own + i;
    int32_t cached = 0;
    if (pa_bm_add_sequence(bm, b, tokens.data(), a.prompt + a.own, &cached) != PA_BM_OK) return 4;
    out.cached_total += cached;
    seqs[b] = b;
  }
  out.admit_us = now_us() - t_admit;

  // ---- decode steps -----------------------------------------------------------
  std::vector<int32_t> tables(static_cast<size_t>(a.batch) * max_blocks);
  std::vector<int32_t> lens(a.batch);
  std::vector<int32_t> kept_tables(static_cast<size_t>(a.batch) * max_blocks);
  std::vector<int32_t> kept_lens(a.batch);
  std::vector<uint64_t> versions(a.batch, 0);
  std::vector<int64_t> slots(a.batch);
  std::vector<int32_t> step_tokens(a.batch), pairs(2 * static_cast<size_t>(a.batch));
  int64_t next_id = a.batch;
  for (int s = 0; s < a.steps; ++s) {
    for (int b = 0; b < a.batch; ++b) step_tokens[b] = 7 + s;
    int32_t npairs = 0;
    const double t0 = now_us();
    if (batched) {
      if (pa_bm_append_tokens(bm, seqs.data(), step_tokens.data(), a.batch, slots.data(),
                              pairs.data(), &npairs) != PA_BM_OK)
        return 5;
    } else {
      for (int b = 0; b < a.batch; ++b) {
        int32_t src = -1, dst = -1;
        if (pa_bm_append_token(bm, seqs[b], step_tokens[b], &slots[b], &src, &dst) != PA_BM_OK)
          return 5;
        if (src >= 0) {
          pairs[2 * npairs] = src;
          pairs[2 * npairs + 1] = dst;
          ++npairs;
        }
      }
    }
    const double t1 = now_us();
    out.appends += a.batch;
    out.cow_pairs += npairs;
    uint64_t h = 1469598103934665603ull;
    for (int b = 0; b < a.batch; ++b) h = mix(h, static_cast<uint64_t>(slots[b]));
    for (int i = 0; i < 2 * npairs; ++i) h = mix(h, static_cast<uint64_t>(pairs[i]));
    out.step_hash.push_back(h);

    const double t2 = now_us();
    if (pa_bm_block_tables(bm, seqs.data(), a.batch, max_blocks, tables.data(), lens.data()) !=
        PA_BM_OK)
      return 6;
    const double t3 = now_us();
    int32_t written = 0;
    if (pa_bm_block_tables_update(bm, seqs.data(), a.batch, max_blocks, kept_tables.data(),
                                  kept_lens.data(), versions.data(), &written) != PA_BM_OK)
      return 6;
    const double t4 = now_us();
    if (kept_tables != tables || kept_lens != lens) return 9;
    out.rewritten += written;
    out.append_us += t1 - t0;
    out.tables_us += t3 - t2;
    out.update_us += t4 - t3;
    if ((s + 1) % a.churn == 0) {
      // 4 sequences fork a beam that takes the place of 4 others, which end
      const double t5 = now_us();
      for (int k = 0; k < 4; ++k) {
        const int parent = (s / a.churn * 4 + k) % a.batch;
        const int victim = (parent + a.batch / 2) % a.batch;
        if (pa_bm_fork(bm, seqs[parent], next_id) != PA_BM_OK) return 7;
        if (pa_bm_free_sequence(bm, seqs[victim]) != PA_BM_OK) return 8;
        seqs[victim] = next_id++;
        ++out.forks;
      }
      out.churn_us += now_us() - t5;
    }
  }
  out.free_left = pa_bm_num_free_blocks(bm);
  pa_bm_destroy(bm);
  return 0;
}

}  // namespace

int main(int argc, char** argv) {
  const Args a{arg(argc, argv, 1, 256), arg(argc, argv, 2, 2000), arg(argc, argv, 3, 2000),
               arg(argc, argv, 4, 64),  arg(argc, argv, 5, 16),   arg(argc, argv, 6, 100)};
  if (a.batch < 8 || a.steps < 1 || a.prompt < 0 || a.own < 1 || a.bs < 1 || a.churn < 1) {
    std::fprintf(stderr, "bad arguments\n");
    return 2;
  }
  Pass one, many;
  int rc = serve(a, false, one);
  if (rc) return rc;
  rc = serve(a, true, many);
  if (rc) return rc;
  if (one.step_hash != many.step_hash || one.free_left != many.free_left) return 10;
  const double n = static_cast<double>(one.appends);
  std::printf(
      "{\"batch\": %d, \"steps\": %d, \"prompt_tokens\": %d, \"own_tokens\": %d, "
      "\"block_size\": %d, \"admit_us_per_request\": %.3f, \"prompt_tokens_cached\": %lld, "
      "\"append_ns_per_token\": %.1f, \"append_batched_ns_per_token\": %.1f, "
      "\"block_tables_us_per_step\": %.3f, \"block_tables_update_us_per_step\": %.3f, "
      "\"rows_rewritten_per_step\": %.2f, \"step_us\": %.3f, \"step_us_full_tables\": %.3f, "
      "\"cow_pairs\": %lld, \"forks\": %lld, \"fork_free_us\": %.3f, "
      "\"free_blocks_left\": %lld}\n",
      a.batch, a.steps, a.prompt, a.own, a.bs, one.admit_us / a.batch,
      static_cast<long long>(one.cached_total), 1000.0 * one.append_us / n,
      1000.0 * many.append_us / n, one.tables_us / a.steps, one.update_us / a.steps,
      static_cast<double>(one.rewritten) / a.steps, (one.append_us + one.update_us) / a.steps,
      (one.append_us + one.tables_us) / a.steps, static_cast<long long>(one.cow_pairs),
      static_cast<long long>(one.forks), one.forks ? one.churn_us / (one.forks / 4.0) : 0.0,
      static_cast<long long>(one.free_left));
  return 0;
}
