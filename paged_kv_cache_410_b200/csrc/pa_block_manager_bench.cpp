// Host benchmark of the block manager (include/pa_block_manager.h): the work
// a decode engine does around the kernels at every step, timed with the
// steady clock on one host thread.
//
//   admit:  `batch` requests whose prompts start with the same system prompt
//           (`prompt` tokens) followed by `own` tokens of their own; with the
//           prefix cache on, every request after the first reuses the system
//           prompt's full blocks;
//   step:   one token per sequence (pa_bm_append_token: slot, copy-on-write
//           pairs after forks), then the batch's block tables and lengths
//           (pa_bm_block_tables, the layout pa_decode reads), and the same
//           through pa_bm_block_tables_update into arrays kept across steps
//           (only rows whose block list changed are rewritten);
//   churn:  every `churn` steps, 4 sequences fork a beam and 4 beams end.
//
// Usage: pa_block_manager_bench [batch steps prompt own block_size churn]
// Prints one JSON line; `step_us` is the appends plus the incremental export,
// `step_us_full_tables` the appends plus the full one. Exits non-zero if the
// two exports ever differ.
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

}  // namespace

int main(int argc, char** argv) {
  const int batch = arg(argc, argv, 1, 256);
  const int steps = arg(argc, argv, 2, 2000);
  const int prompt = arg(argc, argv, 3, 2000);
  const int own = arg(argc, argv, 4, 64);
  const int bs = arg(argc, argv, 5, 16);
  const int churn = arg(argc, argv, 6, 100);
  if (batch < 8 || steps < 1 || prompt < 0 || own < 1 || bs < 1 || churn < 1) {
    std::fprintf(stderr, "bad arguments\n");
    return 2;
  }
  const int max_len = prompt + own + steps;
  const int max_blocks = (max_len + bs - 1) / bs;
  // the shared prompt once, every sequence's own tokens, the beams' copies
  const int64_t num_blocks =
      static_cast<int64_t>(prompt / bs + 2) +
      static_cast<int64_t>(batch + 8) * ((own + steps + bs - 1) / bs + 2) * 2;
  pa_block_manager* bm = pa_bm_create(num_blocks, bs, 1);
  if (!bm) return 3;

  // ---- admit ----------------------------------------------------------------
  std::vector<int32_t> tokens(prompt + own);
  for (int i = 0; i < prompt; ++i) tokens[i] = 1000 + i;
  std::vector<int64_t> seqs(batch);
  int64_t cached_total = 0;
  const double t_admit = now_us();
  for (int b = 0; b < batch; ++b) {
    for (int i = 0; i < own; ++i) tokens[prompt + i] = 100000 + b * own + i;
    int32_t cached = 0;
    if (pa_bm_add_sequence(bm, b, tokens.data(), prompt + own, &cached) != PA_BM_OK) return 4;
    cached_total += cached;
    seqs[b] = b;
  }
  const double admit_us = now_us() - t_admit;

  // ---- decode steps -----------------------------------------------------------
  std::vector<int32_t> tables(static_cast<size_t>(batch) * max_blocks);
  std::vector<int32_t> lens(batch);
  std::vector<int32_t> kept_tables(static_cast<size_t>(batch) * max_blocks);
  std::vector<int32_t> kept_lens(batch);
  std::vector<uint64_t> versions(batch, 0);
  int64_t appends = 0, cow_pairs = 0, forks = 0, next_id = batch, rewritten = 0;
  double append_us = 0.0, tables_us = 0.0, update_us = 0.0, churn_us = 0.0;
  for (int s = 0; s < steps; ++s) {
    double t0 = now_us();
    for (int b = 0; b < batch; ++b) {
      int64_t slot = 0;
      int32_t src = -1, dst = -1;
      if (pa_bm_append_token(bm, seqs[b], 7 + s, &slot, &src, &dst) != PA_BM_OK) return 5;
      cow_pairs += src >= 0;
    }
    appends += batch;
    double t1 = now_us();
    if (pa_bm_block_tables(bm, seqs.data(), batch, max_blocks, tables.data(), lens.data()) !=
        PA_BM_OK)
      return 6;
    double t2 = now_us();
    int32_t written = 0;
    if (pa_bm_block_tables_update(bm, seqs.data(), batch, max_blocks, kept_tables.data(),
                                  kept_lens.data(), versions.data(), &written) != PA_BM_OK)
      return 6;
    double t3 = now_us();
    if (kept_tables != tables || kept_lens != lens) return 9;
    rewritten += written;
    append_us += t1 - t0;
    tables_us += t2 - t1;
    update_us += t3 - t2;
    if ((s + 1) % churn == 0) {
      // 4 sequences fork a beam that takes the place of 4 others, which end
      const double t4 = now_us();
      for (int k = 0; k < 4; ++k) {
        const int parent = (s / churn * 4 + k) % batch;
        const int victim = (parent + batch / 2) % batch;
        if (pa_bm_fork(bm, seqs[parent], next_id) != PA_BM_OK) return 7;
        if (pa_bm_free_sequence(bm, seqs[victim]) != PA_BM_OK) return 8;
        seqs[victim] = next_id++;
        ++forks;
      }
      churn_us += now_us() - t4;
    }
  }
  std::printf(
      "{\"batch\": %d, \"steps\": %d, \"prompt_tokens\": %d, \"own_tokens\": %d, "
      "\"block_size\": %d, \"admit_us_per_request\": %.3f, \"prompt_tokens_cached\": %lld, "
      "\"append_ns_per_token\": %.1f, \"block_tables_us_per_step\": %.3f, "
      "\"block_tables_update_us_per_step\": %.3f, \"rows_rewritten_per_step\": %.2f, "
      "\"step_us\": %.3f, \"step_us_full_tables\": %.3f, "
      "\"cow_pairs\": %lld, \"forks\": %lld, \"fork_free_us\": %.3f, "
      "\"free_blocks_left\": %lld}\n",
      batch, steps, prompt, own, bs, admit_us / batch, static_cast<long long>(cached_total),
      1000.0 * append_us / static_cast<double>(appends), tables_us / steps, update_us / steps,
      static_cast<double>(rewritten) / steps, (append_us + update_us) / steps,
      (append_us + tables_us) / steps, static_cast<long long>(cow_pairs),
      static_cast<long long>(forks), forks ? churn_us / (forks / 4.0) : 0.0,
      static_cast<long long>(pa_bm_num_free_blocks(bm)));
  pa_bm_destroy(bm);
  return 0;
}
