// Paged decode attention (sm_100a).
//
// Computes, for each sequence b and query head i, softmax(scale * q.K^T) V
// over the sequence's cached tokens, found through its block table
// (page "AI 陪读顶会论文（三）：KV Cache 显存占用计算与 PagedAttention 原理拆解",
// section "为什么自回归解码必须使用 KV Cache？", attention equation; section
// "PagedAttention 的破局哲学", block table over scattered physical blocks).
//
// Work decomposition. One CTA handles one (sequence, KV head, partition of
// `partition_tokens` tokens): every query head of the KV head's group
// (grouped-query attention, KV cache article section "显存账本") is served
// from one read of the partition's K and V, so KV bytes cross HBM once per
// KV head. Warps of the CTA take 16-token tiles round-robin, each with its
// own NSTAGE-deep cp.async pipeline into shared memory (no CTA-wide barrier
// in the main loop), and keep their own running max / sum / output (online
// softmax). At the end the warps merge through shared memory; a sequence
// that spans one partition writes its output directly, longer ones write
// (max, sum, normalised output) partials that the reduce kernel combines.
//
// Tensor cores, transposed products. With 16 tokens per MMA row block and up
// to 8 query heads per MMA column block:
//   S^T (16 tokens x 8 heads) = K_tile (16 x D) . Q^T (D x 8)   [m16n8k16]
//   O^T (D x 8 heads)        += V_tile^T (D x 16) . P^T (16 x 8)
// K tiles feed the A operand through ldmatrix, V tiles through
// ldmatrix.trans; Q^T stays in registers as the B operand for the whole
// partition; P^T is the S^T accumulator after the softmax, converted to
// 16 bits and transposed in registers with movmatrix. Rows of every MMA are
// tokens or channels, so no accumulator row is padding; groups of 9..16
// query heads use two column blocks.
//
// E4M3 caches. K and V codes are widened to f16 in registers (exactly:
// every E4M3 value is an f16 value) and both products run on f16 MMAs. The
// K scale is folded into the query (q' = q * k_scale), which is scaled per
// row by a power of two (max |q'| 2^e in [2^14, 2^15), so that no channel
// of it falls into f16's subnormals) and rounded to f16 once; the
// softmax's per-column log2 scale carries 2^-e, and the V scale multiplies
// the merged output.
#pragma once

#include "pa_common.cuh"

namespace pa {

struct DecodeParams {
  const void* q;
  void* out;
  const void* k_cache;
  const void* v_cache;
  const float* k_scale;
  const float* v_scale;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_o;    // [batch][num_q_heads][num_partitions][head_dim]
  float2* ws_ml;  // [batch][num_q_heads][num_partitions] (max in log2 units, sum)
  int64_t num_blocks;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int group;        // num_q_heads / num_kv_heads
  int head_groups;  // ceil(group / 16): CTAs per KV head
  int bs_log2;
  int max_blocks_per_seq;
  int max_context;
  int partition_tokens;
  int num_partitions;
  float scale_log2;  // scale * log2(e)
  // Shared-prefix (cascade) mode; all zero for a plain decode. Tokens before
  // token_start (= prefix_blocks * block_size) are the prefix every sequence
  // shares; the suffix kernel covers [token_start, L) and writes its
  // partials after `part_offset` prefix partials, always as partials.
  int prefix_blocks;
  int token_start;
  int part_offset;
  int force_partials;
  int prefix_chunk_tokens;  // prefix tokens per prefix-kernel CTA (cascade mode)
  // Sliding window (0: none): a sequence of length L attends to its tokens
  // [L - window, L) only.
  int window;
  // Fused append (null k_new: none): sequence b's new token, at position
  // L - 1, comes from k_new / v_new [batch][num_kv_heads][head_dim] (in the
  // query dtype); it is read from there, not from the cache, and the CTA of
  // the sequence's last partition stores it at slot_mapping[b].
  const void* k_new;
  const void* v_new;
  const int64_t* slot_mapping;
  const float* k_inv_scale;  // E4M3 caches
  const float* v_inv_scale;
  // Nonzero: the grid's z index visits the sequences longest first (by
  // attended length after token_start; ties by index) instead of in order.
  // Blocks are dispatched in index order, so this keeps the longest CTAs out
  // of the launch's tail. Each CTA ranks the batch itself (batch <=
  // kOrderMaxBatch).
  int longest_first;
  // Work-list mode (null: a grid of partitions x head groups x sequences):
  // pa_decode_plan_kernel writes the launch's (sequence, partition) items to
  // work_items, largest first, their count to work_count[1] and the
  // persistent grid's size (list_slots) to work_count[0]; CTA i of that grid
  // starts with unit i, and every later unit is a ticket from atomicAdd on
  // work_count[0].
  int2* work_items;
  int* work_count;
  // Work-list mode: the persistent grid's CTAs (the plan kernel sizes the
  // partitions by them), and the longest partition a CTA may be given (the
  // launch's shared memory stages that many tokens' block ids; 0: as
  // partition_tokens).
  int list_slots;
  int max_partition_tokens;
  // Steal mode (null: none; a single sequence's split decode): the CTAs of a
  // (sequence, KV head group) row share its tiles instead of each taking one
  // partition. Their warps claim chunks of kStealChunk tiles from
  // steal_ctr[row], a 64-bit counter whose bits from kStealCountBits up hold
  // the call's epoch (steal_epoch, already shifted; bit 62 always set, which
  // a work-list item, two non-negative ints, never has) and the low bits the
  // tiles claimed so far; each CTA still writes the one partial of its
  // partition column, and the merge zeroes the counters.
  unsigned long long* steal_ctr;
  unsigned long long steal_epoch;
  // Steal mode, launched cooperatively (all CTAs resident at once): each
  // row's CTAs merge the row's partials themselves once the last of them is
  // written, counting on steal_ctr[rows + row] (partials written) and
  // steal_ctr[2 rows + row] (CTAs done), and the row's last CTA zeroes its
  // three counters; no merge kernel follows. steal_withhold (test hook):
  // the row's first CTA does not count its partial, so every wait runs out.
  int steal_merge;
  int steal_withhold;
  // Partial mode (pa_decode_partial; null: off): instead of `out`, each
  // (sequence, query head) row's attention over the tokens its table lists
  // goes to cp_o[row][D] (fp32, normalised as `out` would be) and
  // cp_ml[row] = (max score in log2 units, sum of 2^(score - max)), the
  // pieces a later merge of several such calls (pa_merge_partials) needs;
  // an empty row gives (0, (-inf, 0)). The launch keeps the plain grid.
  float* cp_o;
  float2* cp_ml;
};

constexpr int kStealChunk = 4;
constexpr int kStealCountBits = 24;

// The first of n tiles newly claimed from a steal counter (one thread; n = 0
// only installs this launch's epoch). A counter of another epoch (an earlier
// call's, or bytes a workspace held before) is replaced by (epoch, n) with a
// compare-and-swap from the exact value last seen; a swap fails only when
// another claimant changed the counter in between, by its own first add of
// the launch (at most one per warp) or by installing the epoch, after which
// the counter only grows. The retries are bounded all the same: after
// kStealMaxRounds the claim gives up (claims nothing, flags
// PA_DEVERR_TIMEOUT).
constexpr int kStealMaxRounds = 1 << 20;
__device__ __forceinline__ int steal_claim(unsigned long long* ctr, unsigned long long epoch,
                                           int n) {
  const unsigned long long mask = (1ull << kStealCountBits) - 1;
  const unsigned long long add = static_cast<unsigned long long>(n);
  unsigned long long v = atomicAdd(ctr, add);
  if ((v & ~mask) == epoch) return static_cast<int>(v & mask);
  v += add;  // what this add left behind
  for (int round = 0; round < kStealMaxRounds; ++round) {
    const unsigned long long seen = atomicCAS(ctr, v, epoch | add);
    if (seen == v) return 0;
    if ((seen & ~mask) == epoch)  // installed by another claimant
      return static_cast<int>(atomicAdd(ctr, add) & mask);
    v = seen;
  }
  flag_error(PA_DEVERR_TIMEOUT);
  return 1 << 30;
}

// Steal mode with the merge in the launch: the partials of a (sequence, KV
// head group) row -- nparts of them, one per CTA of the row -- combined by
// those CTAs into `out` once all are written. CTA `part` takes an even slice
// of the row's float4 output columns (query head x 4 channels); a warp
// merges one column at a time, its lanes taking the partials lane, lane +
// 32, ... with a running max each, then combined across the warp. The wait
// for the row's last partial is bounded (1 s of %globaltimer; then
// PA_DEVERR_TIMEOUT and no merge): the launch is cooperative, so the CTAs it
// waits for are resident.
constexpr unsigned long long kStealWaitNs = 1000000000ull;
template <typename TQ, int D, int NW>
__device__ __forceinline__ void steal_merge_row(const DecodeParams& p, int b, int by, int hq0,
                                             int nrows, int nparts, int part) {
  const int64_t rows = static_cast<int64_t>(p.batch) * p.num_kv_heads * p.head_groups;
  const int64_t row = static_cast<int64_t>(b) * p.num_kv_heads * p.head_groups + by;
  unsigned long long* done = p.steal_ctr + rows + row;
  unsigned long long* gone = p.steal_ctr + 2 * rows + row;
  const unsigned long long mask = (1ull << kStealCountBits) - 1;
  __shared__ int s_ok;
  __syncthreads();  // every partial of this CTA is stored
  if (threadIdx.x == 0) {
    __threadfence();
    if (!(p.steal_withhold && part == 0)) steal_claim(done, p.steal_epoch, 1);
    unsigned long long t_start, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_start));
    int ok = 0;
    while (true) {
      unsigned long long v;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(done) : "memory");
      if ((v & ~mask) == p.steal_epoch && static_cast<int>(v & mask) >= nparts) {
        ok = 1;
        break;
      }
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t_start > kStealWaitNs) {
        flag_error(PA_DEVERR_TIMEOUT);
        break;
      }
      __nanosleep(128);
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  if (s_ok) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    constexpr int C4 = D / 4;
    const int total = nrows * C4;
    const int per = (total + nparts - 1) / nparts;
    const int hi = min(total, (part + 1) * per);
    for (int col = part * per + warp; col < hi; col += NW) {
      const int r = col / C4;
      const int c4 = col - r * C4;
      const int64_t bh = static_cast<int64_t>(b) * p.num_q_heads + hq0 + r;
      const float2* ml = p.ws_ml + bh * p.num_partitions;
      const float4* po = reinterpret_cast<const float4*>(p.ws_o + bh * p.num_partitions * D) + c4;
      float mx = -INFINITY, ws = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j0 = 0; j0 < nparts; j0 += 64) {
        // two partials per lane, both loaded before either is used
        float2 v[2];
        float4 o[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int j = j0 + lane + 32 * k;
          v[k] = make_float2(-INFINITY, 0.f);
          o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (j < nparts) {
            v[k] = __ldcg(ml + j);
            o[k] = __ldcg(po + static_cast<int64_t>(j) * C4);
          }
        }
        const float mn = fmaxf(mx, fmaxf(v[0].x, v[1].x));
        if (mn == -INFINITY) continue;  // (CTAs that got no tile: sum 0)
        const float sc = mx == -INFINITY ? 0.f : ex2(mx - mn);
        ws *= sc;
        acc.x *= sc;
        acc.y *= sc;
        acc.z *= sc;
        acc.w *= sc;
        mx = mn;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const float w = v[k].x == -INFINITY ? 0.f : v[k].y * ex2(v[k].x - mx);
          ws += w;
          acc.x += w * o[k].x;
          acc.y += w * o[k].y;
          acc.z += w * o[k].z;
          acc.w += w * o[k].w;
        }
      }
      float M = mx;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float sc = mx == -INFINITY ? 0.f : ex2(mx - M);
      ws *= sc;
      acc.x *= sc;
      acc.y *= sc;
      acc.z *= sc;
      acc.w *= sc;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ws += __shfl_xor_sync(0xffffffffu, ws, o);
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
      }
      if (lane == 0) {
        TQ* out = reinterpret_cast<TQ*>(p.out) + bh * D + 4 * c4;
        const float inv = 1.f / ws;
        out[0] = from_f32<TQ>(acc.x * inv);
        out[1] = from_f32<TQ>(acc.y * inv);
        out[2] = from_f32<TQ>(acc.z * inv);
        out[3] = from_f32<TQ>(acc.w * inv);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_ok) {
    // the row's last CTA out puts its counters back to zero (every CTA of
    // the row is past the wait by then), so that a replay of this launch
    // with the same epoch starts afresh
    if (steal_claim(gone, p.steal_epoch, 1) == nparts - 1) {
      atomicExch(p.steal_ctr + row, 0ull);
      atomicExch(done, 0ull);
      atomicExch(gone, 0ull);
    }
  }
}

constexpr int kOrderMaxBatch = 256;

// Work-list mode: where a persistent CTA stands in the list (shared memory,
// written by thread 0): the ticket of its current unit and that unit's item.
// The next ticket is taken only once the current unit's main loop is done
// (a ticket reserved earlier would tie a unit to a CTA still busy), and its
// item is loaded during the epilogue, so that both latencies hide there.
struct WorkCursor {
  int u;        // current unit: item u / hb, KV head group u % hb
  int n_units;  // items x hb
  int pt;       // the launch's partition length (the plan kernel's choice)
  int2 item;    // item of u: (sequence, partition)
};

__device__ __forceinline__ int units_per_item(const DecodeParams& p) {
  return p.num_kv_heads * p.head_groups;
}

__device__ __forceinline__ int2 cursor_item(const DecodeParams& p, const WorkCursor& c, int u) {
  return u < c.n_units ? p.work_items[u / units_per_item(p)] : make_int2(-1, -1);
}

// thread 0: move the cursor to a new ticket at once
__device__ __forceinline__ void cursor_next(const DecodeParams& p, WorkCursor& c) {
  const int u = atomicAdd(p.work_count, 1);
  c.item = cursor_item(p, c, u);
  c.u = u;
}

// 16 consecutive channels of a 16-bit input row -> 16 E4M3 codes, each
// e4m3_rn_satfinite(fp32(x) * inv_scale) (the append kernel's rounding).
template <typename TIn>
__device__ __forceinline__ uint4 quantize16(const TIn* x, const float* inv) {
  const uint4 a = *reinterpret_cast<const uint4*>(x);
  const uint4 b = *reinterpret_cast<const uint4*>(x + 8);
  const TIn* ea = reinterpret_cast<const TIn*>(&a);
  const TIn* eb = reinterpret_cast<const TIn*>(&b);
  float y[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    y[j] = __fmul_rn(to_f32<TIn>(ea[j]), inv[j]);
    y[8 + j] = __fmul_rn(to_f32<TIn>(eb[j]), inv[8 + j]);
  }
  uint4 r;
  uint32_t* w = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    w[k] = f32x2_to_e4m3x2(y[4 * k], y[4 * k + 1]) | (f32x2_to_e4m3x2(y[4 * k + 2], y[4 * k + 3]) << 16);
  return r;
}

__device__ __forceinline__ int clamp_context(const DecodeParams& p, int L) {
  const int64_t table_cap = static_cast<int64_t>(p.max_blocks_per_seq) << p.bs_log2;
  const int cap = static_cast<int>(table_cap < p.max_context ? table_cap : p.max_context);
  return L < 0 ? 0 : (L > cap ? cap : L);
}

// Tokens a CTA of this launch covers for a sequence of length L: it attends
// to [lo, L); partitions start at `base` (lo rounded down to 16 for a sliding
// window, so that tiles stay block aligned; the tokens in [base, lo) are
// masked and never read).
struct SeqSpan {
  int lo;
  int base;
};
__device__ __forceinline__ SeqSpan seq_span(const DecodeParams& p, int L) {
  SeqSpan s;
  s.lo = p.token_start;
  s.base = p.token_start;
  if (p.window > 0 && L - p.window > s.lo) {
    s.lo = L - p.window;
    s.base = s.lo & ~15;
  }
  return s;
}

// Number of split-K partials of a sequence of length L after the prefix's
// (cascade mode) ones with partitions of pt tokens, shared by the decode and
// reduce kernels.
__device__ __forceinline__ int partitions_of(const DecodeParams& p, int L, int pt) {
  const SeqSpan s = seq_span(p, L);
  const int n = L - s.base;
  return L > s.lo ? (n + pt - 1) / pt : 0;
}

// Partition length of this launch's CTAs: the host's, or in work-list mode
// the plan kernel's choice (published in work_count[2]).
__device__ __forceinline__ int launch_partition_tokens(const DecodeParams& p) {
  return p.work_count ? p.work_count[2] : p.partition_tokens;
}

enum CacheKind { kF16 = 0, kBF16 = 1, kE4M3 = 2 };


// Block ids of one partition staged in shared memory (longer slices are read
// from global memory row by row).
constexpr int kBlockIdsInSmem = 1024;

// Online softmax keeps a reference max per query and moves it only when a
// tile's max exceeds it by more than this (log2 units): the exponentials stay
// at most 2^8, exact in f16/bf16 and far from overflow in the fp32 sums, and
// the accumulator is rescaled only when the reference moves. The reference
// cancels in the final normalisation.
constexpr float kRescaleLog2 = 8.f;

template <int CK, int D>
struct TileGeom {
  static constexpr int ES = (CK == kE4M3) ? 1 : 2;  // bytes per cache element
  static constexpr int RB = D * ES;                  // bytes per token row (one head)
  static constexpr int CPR = RB / 16;                // 16-byte chunks per row
  static constexpr int TOKENS = 16;                  // rows of a tile
  static constexpr int TB = TOKENS * RB;             // one tile of K (or V)
  static_assert(CPR == 4 || CPR == 8 || CPR == 16, "unsupported row size");
  // Byte offset of 16-byte chunk `c` of row `r` inside a tile: the low three
  // chunk bits are XORed with a function of the row (a permutation within
  // each 128-byte line), chosen so that every read pattern of the kernels is
  // free of bank conflicts.
  //  * 16-bit rows (ldmatrix: 8 rows at one chunk column): r & 7.
  //  * E4M3, 128-byte rows: a warp reads 8 contiguous bytes per lane of
  //    rows g = 0..7 at chunk pair {2gq, 2gq + 1} (K), and 16 bytes of
  //    chunk g of rows 2t + c (V). XORing with r & 7 sends rows r and r ^ 1
  //    of the K read to the same pair (two-way conflicts); instead the pair
  //    index takes bit 1 of r and bit 2 XOR bit 0, which is distinct over
  //    rows 0..3, rows 4..7 (the two half-warps of the K read) and over
  //    rows {c, c + 2, c + 4, c + 6} (the V read).
  //  * E4M3, 64-byte rows (two rows per line): the same two reads are free
  //    of conflicts with 2 * ((r >> 1) & 3).
  __device__ __forceinline__ static uint32_t off(int r, int c) {
    if constexpr (ES == 2) {
      return static_cast<uint32_t>(r * RB + ((c ^ (r & 7)) << 4));
    } else if constexpr (CPR >= 8) {
      const int pair = (r & 2) | (((r >> 2) ^ r) & 1);
      return static_cast<uint32_t>(r * RB + ((c ^ ((pair << 1) | (r & 1))) << 4));
    } else {
      const int u = r * CPR + c;
      return static_cast<uint32_t>(((u & ~7) | ((u & 7) ^ (r & 6))) << 4);
    }
  }
};

template <int CK, int D, int NW, int NSTAGE>
struct DecodeSmem {
  using G = TileGeom<CK, D>;
  static constexpr int kStageBytes = 2 * G::TB;  // K tile + V tile
  static constexpr int kPipeBytes = NW * NSTAGE * kStageBytes;
  static constexpr int kMergeBytes = NW * 16 * D * 4 + NW * 16 * 3 * 4 + 32 * 4;
  static constexpr int kMainBytes = kPipeBytes > kMergeBytes ? kPipeBytes : kMergeBytes;
  // + block-table slice of the partition (int32), sized at launch
  // + (fused append into an E4M3 cache) the new token's quantised K and V
  //   rows, 16-byte aligned after the block ids
  static constexpr int kNewRowBytes = 2 * G::RB;
  __host__ __device__ static constexpr int new_rows_offset(int bt_entries) {
    return kMainBytes + (4 * bt_entries + 15) / 16 * 16;
  }
};

// Block ids of a partition staged in shared memory (the launch sizes the
// slice for this many).
__host__ __device__ inline int staged_block_ids(int partition_tokens, int bs_log2) {
  const int n = (partition_tokens >> bs_log2) + 2;
  return n < kBlockIdsInSmem ? n : kBlockIdsInSmem;
}
// ... for the longest partition a CTA of the launch may be given
__host__ __device__ inline int staged_block_ids(const DecodeParams& p) {
  return staged_block_ids(max(p.partition_tokens, p.max_partition_tokens), p.bs_log2);
}

// ---- per-warp attention math shared by the decode and prefix kernels -------
//
// A warp owns NH blocks of 8 query columns. Thread (g = lane/4, t = lane%4)
// holds the B-operand fragments of column 8*nh + g and the O^T accumulator
// o[mt][nh] = {(channel row g, columns 2t, 2t+1), (channel row g+8, same)}.

// Q^T fragments (16-bit caches): qb[kk][nh] = {channels of k-slots 2t,2t+1 ;
// 2t+8,2t+9} of the query row rows[nh] (nullptr: a padding column of zeros).
template <typename TQ, int D, int NH>
__device__ __forceinline__ void load_query_fragments(const TQ* const (&rows)[NH],
                                                     uint32_t (&qb)[D / 16][NH][2]) {
  const int t = threadIdx.x & 3;
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(rows[nh]);
    const bool ok = q32 != nullptr;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      qb[kk][nh][0] = ok ? q32[(kk * 16 + 2 * t) / 2] : 0u;
      qb[kk][nh][1] = ok ? q32[(kk * 16 + 8 + 2 * t) / 2] : 0u;
    }
  }
}

// Q^T fragments for an E4M3 cache (B operand of the f16 MMA on widened K).
// Thread (g, t) holds query row rows[nh] (column g of block nh; nullptr:
// zeros) times the K scale, q' = q * k_scale (fp32), scaled by 2^e with e
// chosen per row so that max |q'| 2^e lies in [2^14, 2^15), rounded to f16
// once. Channel order (shared with attend_tile_e4m3's K fragments): within
// each 32-channel group gq, k-step 2gq + h holds channels 8t + 4h + {0,1} in
// slots 2t, 2t+1 and 8t + 4h + {2,3} in slots 2t+8, 2t+9, so that a thread's
// K codes are 8 contiguous bytes. sl2[nh][e] = scale_log2 * 2^-e of the row
// in accumulator column 2t + e.
template <typename TQ, int D, int NH>
__device__ __forceinline__ void load_query_e4m3(const TQ* const (&rows)[NH], const float* ks,
                                                float scale_log2, uint32_t (&qb)[D / 16][NH][2],
                                                float (&sl2)[NH][2]) {
  const int t = threadIdx.x & 3;
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) {
    const TQ* qr = rows[nh];
    const bool ok = qr != nullptr;
    float x[D / 32][2][4];
    float mx = 0.f;
#pragma unroll
    for (int gq = 0; gq < D / 32; ++gq)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // channels c .. c + 3: one 8-byte load of q, one 16-byte load of the
        // scales (rows and scale arrays are 16-byte aligned)
        const int c = 32 * gq + 8 * t + 4 * h;
        uint2 qv = make_uint2(0u, 0u);
        float4 sv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ok) {
          qv = *reinterpret_cast<const uint2*>(qr + c);
          sv = *reinterpret_cast<const float4*>(ks + c);
        }
        const TQ* qe = reinterpret_cast<const TQ*>(&qv);
        x[gq][h][0] = to_f32<TQ>(qe[0]) * sv.x;
        x[gq][h][1] = to_f32<TQ>(qe[1]) * sv.y;
        x[gq][h][2] = to_f32<TQ>(qe[2]) * sv.z;
        x[gq][h][3] = to_f32<TQ>(qe[3]) * sv.w;
#pragma unroll
        for (int i = 0; i < 4; ++i) mx = fmaxf(mx, fabsf(x[gq][h][i]));
      }
    // the four threads of the group hold the row's channels between them
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    // e = 14 - floor(log2 mx) (from the exponent field; kept within a range
    // where 2^e and 2^-e are normal floats)
    int e = 0;
    if (mx > 0.f) {
      const int ex = static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127;
      e = min(max(14 - ex, -100), 100);
    }
    const float up = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);  // 2^e
#pragma unroll
    for (int gq = 0; gq < D / 32; ++gq)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        qb[2 * gq + h][nh][0] = pack2<false>(x[gq][h][0] * up, x[gq][h][1] * up);
        qb[2 * gq + h][nh][1] = pack2<false>(x[gq][h][2] * up, x[gq][h][3] * up);
      }
    // the accumulator's columns 2t, 2t + 1 are the rows of threads (2t, *) and
    // (2t + 1, *)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int ec = __shfl_sync(0xffffffffu, e, (2 * t + c) * 4);
      sl2[nh][c] = scale_log2 * __uint_as_float(static_cast<uint32_t>(127 - ec) << 23);
    }
  }
}

// Channels of O^T rows g and g + 8 in channel block mt.
template <int CK, int D>
__device__ __forceinline__ int2 accumulator_channels(int mt, int g) {
  if constexpr (CK != kE4M3) return make_int2(16 * mt + g, 16 * mt + 8 + g);
  return make_int2((D / 8) * g + 2 * mt, (D / 8) * g + 2 * mt + 1);
}

// Position of channel c of query head `head` inside its row of the warps'
// merge buffer: c XOR a value that depends on the head and on c / 32 only,
// so that each aligned run of 32 channels stays in place as a set (the
// merge reads it with consecutive threads, conflict-free) while the stores
// of the accumulators, one channel per lane from 8 lanes g x 4 heads 2t + e,
// land in 32 distinct banks: for 16-bit caches lane g holds channel
// 16 mt + g (+ 8), so the head goes to bits 3-4; for E4M3 lane g holds
// channel (D / 8) g + 2 mt (+ 1), so bits 0 .. log2(D / 32) - 1 take c / 32
// and the next two the head.
template <int CK, int D>
__device__ __forceinline__ int merge_pos(int head, int c) {
  const int h2 = (head >> 1) & 3;
  if constexpr (CK != kE4M3) {
    return c ^ (h2 << 3);
  } else {
    constexpr int kBlk = D / 32;  // 2 or 4
    constexpr int kShift = kBlk == 4 ? 2 : 1;
    return c ^ (((c >> 5) & (kBlk - 1)) | (h2 << kShift));
  }
}

// One 16-token tile of K and V of a 16-bit cache in shared memory (rows <
// nskip or >= nvalid are zero and masked; FULL: all 16 rows count) against
// the warp's query columns: S^T = K Q^T, online softmax update of the
// per-column running max / sum (log2 domain), O^T += V^T P^T.
template <int CK, int D, int NH, bool FULL>
__device__ __forceinline__ void attend_tile(uint32_t sk_a, uint32_t sv_a, int nvalid, int nskip,
                                            float scale_log2,
                                            const uint32_t (&qb)[D / 16][NH][2],
                                            float (&o)[D / 16][NH][4], float (&m_run)[NH][2],
                                            float (&l_run)[NH][2]) {
  static_assert(CK != kE4M3, "E4M3 tiles: attend_tile_e4m3");
  using G = TileGeom<CK, D>;
  constexpr bool kMmaBF16 = (CK == kBF16);  // MMA operand type
  constexpr int KSTEPS = D / 16;
  constexpr int MT = D / 16;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;

  // S^T = K Q^T: s[nh] = {(token g, columns 2t, 2t+1), (token g+8, same)}
  float s[NH][4];
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) s[nh][0] = s[nh][1] = s[nh][2] = s[nh][3] = 0.f;
  {
    const int mi = lane >> 3;
    const int tok = (lane & 7) + 8 * (mi & 1);
    const int chk = mi >> 1;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      uint32_t a[4];
      ldmatrix_x4(a[0], a[1], a[2], a[3], sk_a + G::off(tok, 2 * kk + chk));
#pragma unroll
      for (int nh = 0; nh < NH; ++nh) mma_16816<kMmaBF16>(s[nh], a, qb[kk][nh][0], qb[kk][nh][1]);
    }
  }

  // online softmax per column; the max is reduced over the 16 tokens
  // (lanes with the same t, both row halves) on the raw scores (the scale is
  // positive), and each exponent is one FFMA: s * scale_log2 - m_ref
  const bool va = FULL || (g < nvalid && g >= nskip);
  const bool vb = FULL || (g + 8 < nvalid && g + 8 >= nskip);
  uint32_t pb[NH][2];
  bool grew = false;
  float alpha[NH][2];
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) {
    float pr[2][2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float mx = fmaxf(va ? s[nh][e] : -INFINITY, vb ? s[nh][2 + e] : -INFINITY);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      mx *= scale_log2;
      // mx is finite (token 0 of the tile exists), so the first tile always
      // sets the reference
      const bool up = mx > m_run[nh][e] + kRescaleLog2;
      grew |= up;
      const float m_ref = up ? mx : m_run[nh][e];
      alpha[nh][e] = up ? ex2(m_run[nh][e] - m_ref) : 1.f;  // exactly 1 when unchanged
      const float p0 = ex2(fmaf(s[nh][e], scale_log2, -m_ref));
      const float p1 = ex2(fmaf(s[nh][2 + e], scale_log2, -m_ref));
      pr[0][e] = va ? p0 : 0.f;
      pr[1][e] = vb ? p1 : 0.f;
      l_run[nh][e] = l_run[nh][e] * alpha[nh][e] + (pr[0][e] + pr[1][e]);
      m_run[nh][e] = m_ref;
    }
    // (token, column) 8x8 blocks -> transposed: column g, tokens 2t,2t+1 | 2t+8,2t+9
    pb[nh][0] = movmatrix_trans(pack2<kMmaBF16>(pr[0][0], pr[0][1]));
    pb[nh][1] = movmatrix_trans(pack2<kMmaBF16>(pr[1][0], pr[1][1]));
  }
  if (__any_sync(0xffffffffu, grew)) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nh = 0; nh < NH; ++nh) {
        o[mt][nh][0] *= alpha[nh][0];
        o[mt][nh][1] *= alpha[nh][1];
        o[mt][nh][2] *= alpha[nh][0];
        o[mt][nh][3] *= alpha[nh][1];
      }
  }

  // O^T += V^T P^T
  {
    const int mi = lane >> 3;
    const int tok = (lane & 7) + 8 * (mi >> 1);
    const int chk = mi & 1;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      uint32_t a[4];
      ldmatrix_x4_trans(a[0], a[1], a[2], a[3], sv_a + G::off(tok, 2 * mt + chk));
#pragma unroll
      for (int nh = 0; nh < NH; ++nh) mma_16816<kMmaBF16>(o[mt][nh], a, pb[nh][0], pb[nh][1]);
    }
  }
}

// One 16-token tile of K and V of an E4M3 cache (rows < nskip or >= nvalid
// are zero and masked; FULL: all 16 rows count): S^T = K Q^T with K widened
// to f16 in registers, s[nh] = {(token g, columns 2t, 2t+1), (token g + 8,
// same)}; online softmax as attend_tile, with the per-column log2 scale sl2;
// O^T += V^T P^T with V widened to f16.
template <int D, int NH, bool FULL>
__device__ __forceinline__ void attend_tile_e4m3(uint32_t sk_a, uint32_t sv_a, int nvalid,
                                                 int nskip, const float (&sl2)[NH][2],
                                                 const uint32_t (&qb)[D / 16][NH][2],
                                                 float (&o)[D / 16][NH][4], float (&m_run)[NH][2],
                                                 float (&l_run)[NH][2]) {
  using G = TileGeom<kE4M3, D>;
  constexpr int MT = D / 16;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;

  float s[NH][4];
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) s[nh][0] = s[nh][1] = s[nh][2] = s[nh][3] = 0.f;
  // thread (g, t) reads 8 contiguous channel bytes of tokens g and g + 8 in
  // each 32-channel group gq (the query's channel order)
#pragma unroll
  for (int gq = 0; gq < D / 32; ++gq) {
    const int c = 2 * gq + (t >> 1);
    const int bo = (t & 1) * 8;
    const uint2 wl = lds64(sk_a + G::off(g, c) + bo);      // token g
    const uint2 wh = lds64(sk_a + G::off(g + 8, c) + bo);  // token g + 8
    uint32_t a0[4], a1[4];
    e4m3x4_to_f16x2x2(wl.x, a0[0], a0[2]);
    e4m3x4_to_f16x2x2(wh.x, a0[1], a0[3]);
    e4m3x4_to_f16x2x2(wl.y, a1[0], a1[2]);
    e4m3x4_to_f16x2x2(wh.y, a1[1], a1[3]);
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) {
      mma_16816<false>(s[nh], a0, qb[2 * gq][nh][0], qb[2 * gq][nh][1]);
      mma_16816<false>(s[nh], a1, qb[2 * gq + 1][nh][0], qb[2 * gq + 1][nh][1]);
    }
  }

  const bool va = FULL || (g < nvalid && g >= nskip);
  const bool vb = FULL || (g + 8 < nvalid && g + 8 >= nskip);
  uint32_t pb[NH][2];
  bool grew = false;
  float alpha[NH][2];
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) {
    float pr[2][2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float mx = fmaxf(va ? s[nh][e] : -INFINITY, vb ? s[nh][2 + e] : -INFINITY);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float sc = sl2[nh][e];
      mx *= sc;
      // mx is finite (some row of the tile exists), so the first tile always
      // sets the reference
      const bool up = mx > m_run[nh][e] + kRescaleLog2;
      grew |= up;
      const float m_ref = up ? mx : m_run[nh][e];
      alpha[nh][e] = up ? ex2(m_run[nh][e] - m_ref) : 1.f;
      const float p0 = ex2(fmaf(s[nh][e], sc, -m_ref));
      const float p1 = ex2(fmaf(s[nh][2 + e], sc, -m_ref));
      pr[0][e] = va ? p0 : 0.f;
      pr[1][e] = vb ? p1 : 0.f;
      l_run[nh][e] = l_run[nh][e] * alpha[nh][e] + (pr[0][e] + pr[1][e]);
      m_run[nh][e] = m_ref;
    }
    pb[nh][0] = movmatrix_trans(pack2<false>(pr[0][0], pr[0][1]));
    pb[nh][1] = movmatrix_trans(pack2<false>(pr[1][0], pr[1][1]));
  }
  if (__any_sync(0xffffffffu, grew)) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nh = 0; nh < NH; ++nh) {
        o[mt][nh][0] *= alpha[nh][0];
        o[mt][nh][1] *= alpha[nh][1];
        o[mt][nh][2] *= alpha[nh][0];
        o[mt][nh][3] *= alpha[nh][1];
      }
  }

  // O^T += V^T P^T. Row m of O^T block mt is channel DPT*g + 2*mt (m = g) or
  // that + 1 (m = g + 8): this thread reads channels [DPT*g, DPT*g + DPT) of
  // token rows 2t, 2t+1, 2t+8, 2t+9 and pairs tokens with byte permutes.
  constexpr int DPT = D / 8;
  constexpr int WORDS = DPT / 4;
  uint32_t ra[4][WORDS];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    const int r = 2 * t + (q4 & 1) + 8 * (q4 >> 1);
    const int byte0 = DPT * g;
    const uint32_t addr = sv_a + G::off(r, byte0 >> 4) + (byte0 & 15);
    if constexpr (WORDS == 4) {
      const uint4 w = lds128(addr);
      ra[q4][0] = w.x;
      ra[q4][1] = w.y;
      ra[q4][2] = w.z;
      ra[q4][3] = w.w;
    } else {
      const uint2 w = lds64(addr);
      ra[q4][0] = w.x;
      ra[q4][1] = w.y;
    }
  }
#pragma unroll
  for (int w = 0; w < WORDS; ++w) {
    uint32_t f[4], e[4];
    e4m3x4_to_f16x2x2(__byte_perm(ra[0][w], ra[1][w], 0x5140), f[0], f[1]);
    e4m3x4_to_f16x2x2(__byte_perm(ra[0][w], ra[1][w], 0x7362), f[2], f[3]);
    e4m3x4_to_f16x2x2(__byte_perm(ra[2][w], ra[3][w], 0x5140), e[0], e[1]);
    e4m3x4_to_f16x2x2(__byte_perm(ra[2][w], ra[3][w], 0x7362), e[2], e[3]);
    const uint32_t a0[4] = {f[0], f[1], e[0], e[1]};  // channel block 2w
    const uint32_t a1[4] = {f[2], f[3], e[2], e[3]};  // channel block 2w+1
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) {
      mma_16816<false>(o[2 * w][nh], a0, pb[nh][0], pb[nh][1]);
      mma_16816<false>(o[2 * w + 1][nh], a1, pb[nh][0], pb[nh][1]);
    }
  }
}

// NH: 8-head column blocks per CTA (1 for groups of up to 8 query heads, 2
// for 9..16).
//
// One decode CTA: partition `part` of sequence `b`, for KV head / head group
// `by` (= kv_head * head_groups + head_group).
// FUSED: the launch also appends each sequence's new token (pa_append_decode).
// PT: the launch's partition length (p.partition_tokens, or in work-list
// mode the plan kernel's). cursor (work-list mode, else null): thread 0 takes
// the next ticket once the main loop is done, loads its item during the
// epilogue and moves the cursor before returning.
// STEAL: steal mode (p.steal_ctr set; 16-bit caches with blocks of 16 tokens
// or more, one head group per KV head, no fused append, grid mode).
template <typename TQ, int CK, int D, int NW, int NSTAGE, int NH, bool FUSED = false,
          bool STEAL = false>
__device__ __forceinline__ void decode_cta(const DecodeParams& p, const int part, const int by,
                                           const int b, const int PT,
                                           WorkCursor* cursor = nullptr) {
  using S = DecodeSmem<CK, D, NW, NSTAGE>;
  using G = typename S::G;
  constexpr bool kE4 = (CK == kE4M3);
  constexpr int TOK = G::TOKENS;            // tokens per tile
  constexpr int KSTEPS = D / 16;            // k-steps of S^T = K Q^T (16-bit)
  constexpr int MT = D / 16;                // 16-channel row blocks of O^T
  constexpr int RPI = 32 / G::CPR;          // tile rows one load instruction covers
  constexpr int LITERS = TOK / RPI;         // load instructions per lane per tile and tensor

  extern __shared__ __align__(128) uint8_t smem[];
  int* s_bt = reinterpret_cast<int*>(smem + S::kMainBytes);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane >> 2;  // MMA group id
  const int t = lane & 3;   // thread in group

  const int hk = by / p.head_groups;
  const int hgrp = by - hk * p.head_groups;
  const int row0 = hgrp * 16;
  const int nrows = min(16, p.group - row0);  // query heads of this CTA
  const int hq0 = hk * p.group + row0;

  // ---- sequence length, checked against what the launch covers ----------
  const int L_in = p.context_lens[b];
  const int L = clamp_context(p, L_in);
  if (L != L_in && threadIdx.x == 0 && part == 0 && by == 0)
    flag_error(PA_DEVERR_CONTEXT_LEN);
  if (p.prefix_blocks > 0 && part == 0 && by == 0) {
    // cascade mode: this sequence must start with the shared prefix blocks
    const int32_t* row = p.block_tables + static_cast<int64_t>(b) * p.max_blocks_per_seq;
    bool bad = L < p.token_start;
    for (int i = threadIdx.x; i < p.prefix_blocks; i += NW * 32)
      bad |= row[i] != p.block_tables[i];
    if (bad) flag_error(PA_DEVERR_PREFIX);
  }
  const int nparts = partitions_of(p, L, PT);
  const bool steer = cursor != nullptr && threadIdx.x == 0;  // this thread moves the cursor
  if (part >= (nparts > 0 || p.force_partials ? nparts : 1)) {
    if (steer) cursor_next(p, *cursor);
    return;
  }

  TQ* out = reinterpret_cast<TQ*>(p.out);
  if (L == 0) {  // (plain mode only: a cascade launch has no partition here)
    for (int i = threadIdx.x; i < nrows * D; i += NW * 32) {
      const int64_t bh = static_cast<int64_t>(b) * p.num_q_heads + hq0 + i / D;
      if (p.cp_o) {
        p.cp_o[bh * D + (i % D)] = 0.f;
        if (i % D == 0) p.cp_ml[bh] = make_float2(-INFINITY, 0.f);
      } else {
        out[bh * D + (i % D)] = from_f32<TQ>(0.f);
      }
    }
    if (steer) cursor_next(p, *cursor);
    return;
  }
  const SeqSpan span = seq_span(p, L);
  const int lo = span.lo;  // first attended token
  // the partition; in steal mode the row's whole attended range
  const int t0 = STEAL ? span.base : span.base + part * PT;
  const int t1 = STEAL ? L : min(t0 + PT, L);
  const int ntiles = (t1 - t0 + TOK - 1) / TOK;

  // ---- block ids of this partition -> shared memory ----------------------
  // (as many as the launch staged room for, at most kBlockIdsInSmem; a
  // longer slice is read from global memory per row instead). Blocks before
  // `lo` are never looked up: a sliding-window caller may have freed them.
  const int bt0 = max(t0, lo) >> p.bs_log2;
  const int nbt = ((t1 - 1) >> p.bs_log2) - bt0 + 1;
  const bool bt_in_smem = !STEAL && nbt <= staged_block_ids(p);
  const int32_t* gbt = p.block_tables + static_cast<int64_t>(b) * p.max_blocks_per_seq + bt0;
  if (bt_in_smem) {
    for (int i = threadIdx.x; i < nbt; i += NW * 32) {
      int id = gbt[i];
      if (id < 0 || id >= p.num_blocks) {
        flag_error(PA_DEVERR_BLOCK_ID);
        id = -1;
      }
      s_bt[i] = id;
    }
  }

  // ---- Q^T fragments (B operand: k = channel, n = query head) -------------
  const TQ* qbase = reinterpret_cast<const TQ*>(p.q) +
                    (static_cast<int64_t>(b) * p.num_q_heads + hq0) * D;
  uint32_t qb[KSTEPS][NH][2];
  float sl2[NH][2];  // E4M3: per-column log2 scale
  {
    const TQ* rows[NH];
#pragma unroll
    for (int nh = 0; nh < NH; ++nh)
      rows[nh] = 8 * nh + g < nrows ? qbase + (8 * nh + g) * D : nullptr;
    if constexpr (kE4)
      load_query_e4m3<TQ, D, NH>(rows, p.k_scale + static_cast<int64_t>(hk) * D, p.scale_log2,
                                 qb, sl2);
    else
      load_query_fragments<TQ, D, NH>(rows, qb);
  }
  __syncthreads();  // s_bt ready

  // ---- per-warp pipeline over this warp's tiles ---------------------------
  uint8_t* wbuf = smem + warp * NSTAGE * S::kStageBytes;
  const uint8_t* kc = reinterpret_cast<const uint8_t*>(p.k_cache);
  const uint8_t* vc = reinterpret_cast<const uint8_t*>(p.v_cache);
  const int64_t slot_stride = static_cast<int64_t>(p.num_kv_heads) * G::RB;
  const int bs_mask = (1 << p.bs_log2) - 1;
  const bool block_aligned = p.bs_log2 >= 4;  // a 16-token tile lies inside one block
  // this lane's load slots: rows lrow + i*RPI, 16-byte chunk lch
  const int lrow = lane / G::CPR;
  const int lch = lane % G::CPR;
  const int64_t lane_goff = static_cast<int64_t>(hk) * G::RB + lch * 16;

  auto block_id = [&](int bi) -> int {
    if (bt_in_smem) return s_bt[bi];
    int id = __ldg(gbt + bi);
    if (id < 0 || id >= p.num_blocks) {
      flag_error(PA_DEVERR_BLOCK_ID);
      id = -1;
    }
    return id;
  };

  // ---- fused append: the new token (position L - 1) comes from the input --
  const bool has_new = FUSED && p.slot_mapping[b] >= 0;
  const int jnew = has_new ? L - 1 : -1;
  const int64_t new_row = (static_cast<int64_t>(b) * p.num_kv_heads + hk) * D;  // elements
  const TQ* knew = has_new ? reinterpret_cast<const TQ*>(p.k_new) + new_row : nullptr;
  const TQ* vnew = has_new ? reinterpret_cast<const TQ*>(p.v_new) + new_row : nullptr;
  // E4M3: the new token's rows, quantised once (e4m3_rn_satfinite(x *
  // inv_scale), as pa_append_kv does) into shared memory, for the tile that
  // holds the token and for the store at the end
  const uint32_t s_new =
      smem_addr(smem) + S::new_rows_offset(staged_block_ids(p));
  if constexpr (FUSED && kE4) {
    if (has_new && jnew >= max(t0, lo) && jnew < t1 && threadIdx.x < 2 * G::CPR) {
      const bool is_v = threadIdx.x >= G::CPR;
      const int ch = threadIdx.x - (is_v ? G::CPR : 0);
      const uint4 qv = quantize16<TQ>((is_v ? vnew : knew) + 16 * ch,
                                      (is_v ? p.v_inv_scale : p.k_inv_scale) + hk * D + 16 * ch);
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(
                       s_new + (is_v ? G::RB : 0) + 16 * ch),
                   "r"(qv.x), "r"(qv.y), "r"(qv.z), "r"(qv.w)
                   : "memory");
    }
    __syncthreads();
  }
  // Store the new token in the cache, as pa_append_kv would; the slot must
  // be the one the table gives position L - 1. Done by the CTA of the last
  // partition (first head group); nothing in this launch reads the slot.
  auto store_new_token = [&]() {
    if (!(has_new && part == nparts - 1 && hgrp == 0)) return;
    const int64_t slot = p.slot_mapping[b];
    const int64_t expect =
        (static_cast<int64_t>(p.block_tables[static_cast<int64_t>(b) * p.max_blocks_per_seq +
                                             (jnew >> p.bs_log2)])
         << p.bs_log2) +
        (jnew & ((1 << p.bs_log2) - 1));
    if (slot != expect || slot >= (static_cast<int64_t>(p.num_blocks) << p.bs_log2)) {
      if (threadIdx.x == 0) flag_error(PA_DEVERR_SLOT);
    } else if (threadIdx.x < 2 * G::CPR) {
      const bool is_v = threadIdx.x >= G::CPR;
      const int ch = threadIdx.x - (is_v ? G::CPR : 0);
      // (the fused entry point passes writable caches)
      uint8_t* dst = static_cast<uint8_t*>(const_cast<void*>(is_v ? p.v_cache : p.k_cache)) +
                     (slot * p.num_kv_heads + hk) * G::RB + ch * 16;
      const TQ* src = is_v ? vnew : knew;
      if constexpr (CK == kE4M3) {
        *reinterpret_cast<uint4*>(dst) = lds128(s_new + (is_v ? G::RB : 0) + 16 * ch);
      } else {
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src + 8 * ch);
      }
    }
  };
  // a 16-bit row is a plain copy: done up front; the E4M3 row is stored at
  // the end of the CTA, from the quantised copy in shared memory
  if constexpr (FUSED && CK != kE4M3) store_new_token();

  // One 16-byte chunk of row r: from the cache at `off`, or from the fused
  // new token (16-bit: the same bytes by cp.async; E4M3: the quantised row
  // from shared memory).
  auto load_chunk = [&](uint32_t sk_a, uint32_t sv_a, int r, int j, bool ok, int64_t off) {
    const uint32_t so = G::off(r, lch);
    if (FUSED && j == jnew) {
      if constexpr (CK != kE4M3) {
        cp_async_16(sk_a + so, knew + 8 * lch, 16u);
        cp_async_16(sv_a + so, vnew + 8 * lch, 16u);
      } else {
        const uint4 kq = lds128(s_new + 16 * lch);
        const uint4 vq = lds128(s_new + G::RB + 16 * lch);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(sk_a + so), "r"(kq.x),
                     "r"(kq.y), "r"(kq.z), "r"(kq.w)
                     : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(sv_a + so), "r"(vq.x),
                     "r"(vq.y), "r"(vq.z), "r"(vq.w)
                     : "memory");
      }
      return;
    }
    cp_async_16(sk_a + so, kc + off, ok ? 16u : 0u);
    cp_async_16(sv_a + so, vc + off, ok ? 16u : 0u);
  };
  // (blk_given: the tile's block id where the caller has it already, as in
  // steal mode; kLookUp: look it up here)
  constexpr int kLookUp = -2;
  auto load_tile = [&](int tile, int stage, int blk_given) {
    const uint32_t sk_a = smem_addr(wbuf + stage * S::kStageBytes);
    const uint32_t sv_a = sk_a + G::TB;
    const int tb = t0 + tile * TOK;
    if (block_aligned) {
      const int blk = blk_given != kLookUp ? blk_given : block_id((tb >> p.bs_log2) - bt0);
      const int64_t base =
          ((static_cast<int64_t>(blk) << p.bs_log2) + (tb & bs_mask) + lrow) * slot_stride +
          lane_goff;
#pragma unroll
      for (int i = 0; i < LITERS; ++i) {
        const int r = lrow + i * RPI;
        const bool ok = blk >= 0 && tb + r < t1 && tb + r >= lo;
        const int64_t off = ok ? base + static_cast<int64_t>(i * RPI) * slot_stride : 0;
        load_chunk(sk_a, sv_a, r, tb + r, ok, off);
      }
    } else {
#pragma unroll
      for (int i = 0; i < LITERS; ++i) {
        const int r = lrow + i * RPI;
        const int j = tb + r;
        const int blk = (j < t1 && j >= lo && j != jnew) ? block_id((j >> p.bs_log2) - bt0) : -1;
        const bool ok = blk >= 0;
        const int64_t off =
            ok ? ((static_cast<int64_t>(blk) << p.bs_log2) + (j & bs_mask)) * slot_stride +
                     lane_goff
               : 0;
        load_chunk(sk_a, sv_a, r, j, ok, off);
      }
    }
  };

  float o[MT][NH][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) o[mt][nh][0] = o[mt][nh][1] = o[mt][nh][2] = o[mt][nh][3] = 0.f;
  float m_run[NH][2], l_run[NH][2];
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) {
    m_run[nh][0] = m_run[nh][1] = -INFINITY;
    l_run[nh][0] = l_run[nh][1] = 0.f;
  }

  // One tile from pipeline stage `stage` into the warp's running state.
  auto attend = [&](int tile, int stage) {
    const uint32_t sk_a = smem_addr(wbuf + stage * S::kStageBytes);
    const uint32_t sv_a = sk_a + G::TB;
    const int ts = t0 + tile * TOK;
    const int nvalid = t1 - ts;         // rows of the tile below the end (>= 1)
    const int nskip = max(lo - ts, 0);  // rows before the window (first tile only)
    if constexpr (kE4) {
      if (nvalid >= TOK && nskip == 0)
        attend_tile_e4m3<D, NH, true>(sk_a, sv_a, nvalid, 0, sl2, qb, o, m_run, l_run);
      else
        attend_tile_e4m3<D, NH, false>(sk_a, sv_a, nvalid, nskip, sl2, qb, o, m_run, l_run);
    } else {
      if (nvalid >= TOK && nskip == 0)
        attend_tile<CK, D, NH, true>(sk_a, sv_a, nvalid, 0, p.scale_log2, qb, o, m_run, l_run);
      else
        attend_tile<CK, D, NH, false>(sk_a, sv_a, nvalid, nskip, p.scale_log2, qb, o, m_run,
                                      l_run);
    }
  };

  if constexpr (!STEAL) {
    // the warp's tiles: warp, warp + NW, ... of the partition
    const int my_tiles = warp < ntiles ? (ntiles - warp + NW - 1) / NW : 0;
#pragma unroll
    for (int s = 0; s < NSTAGE - 1; ++s) {
      if (s < my_tiles) load_tile(warp + s * NW, s, kLookUp);
      cp_async_commit();
    }
    for (int it = 0; it < my_tiles; ++it) {
      {
        const int nxt = it + NSTAGE - 1;
        if (nxt < my_tiles) load_tile(warp + nxt * NW, nxt % NSTAGE, kLookUp);
        cp_async_commit();
      }
      cp_async_wait<NSTAGE - 1>();
      __syncwarp();
      attend(warp + it * NW, it % NSTAGE);
      __syncwarp();  // this stage is reloaded by the next iteration
    }
  } else {
    // The row's tiles in chunks of kStealChunk: first each CTA's own share
    // (about half the row split evenly, its chunks round robin over the
    // warps), then a pool of the rest that the warps of all the row's CTAs
    // claim chunk by chunk from the counter, so that CTAs which finish their
    // share early take more of it. The shares keep the claims away from the
    // launch's first microseconds, when every warp of the row would contend
    // on the counter, and the row's first CTA installs the launch's epoch
    // meanwhile. A warp works one chunk while the next one's block ids load
    // (its first lanes read them when the chunk is chosen).
    unsigned long long* ctr =
        p.steal_ctr + (static_cast<int64_t>(b) * p.num_kv_heads * p.head_groups + by);
    const int share = ((ntiles / 2) / nparts) & ~(kStealChunk * NW - 1);
    const int share_chunks = share / (kStealChunk * NW);  // per warp
    const int pool = nparts * share;                       // first tile of the pool
    if (part == 0 && threadIdx.x == 0) {
      steal_claim(ctr, p.steal_epoch, 0);
      if (p.steal_merge) {  // and the in-launch merge's two counters
        const int64_t rows = static_cast<int64_t>(p.batch) * p.num_kv_heads * p.head_groups;
        steal_claim(ctr + rows, p.steal_epoch, 0);
        steal_claim(ctr + 2 * rows, p.steal_epoch, 0);
      }
    }
    int k_share = 0;
    // first tile of the warp's next chunk (>= ntiles: none left), and the
    // chunk's block ids in lanes 0 .. kStealChunk - 1
    auto next_chunk = [&](int& id) -> int {
      int c;
      if (k_share < share_chunks) {
        c = part * share + (k_share++ * NW + warp) * kStealChunk;
      } else {
        int off = 0;
        if (lane == 0) off = steal_claim(ctr, p.steal_epoch, kStealChunk);
        c = pool + __shfl_sync(0xffffffffu, off, 0);
      }
      id = -1;
      if (lane < kStealChunk && c + lane < ntiles)
        id = block_id(((t0 + (c + lane) * TOK) >> p.bs_log2) - bt0);
      return c;
    };
    int id_cur = -1, id_nxt = -1;  // block id of tile (chunk + lane), lanes < kStealChunk
    int c_cur = next_chunk(id_cur);                           // current chunk
    int c_nxt = c_cur < ntiles ? next_chunk(id_nxt) : c_cur;  // next chunk
    int c_k = 0;  // tiles of the current chunk handed out
    // the warp's next tile (-1: none left) and its block id
    auto next_tile = [&](int& blk) -> int {
      while (c_cur < ntiles) {
        if (c_k < kStealChunk && c_cur + c_k < ntiles) {
          blk = __shfl_sync(0xffffffffu, id_cur, c_k);
          return c_cur + c_k++;
        }
        c_cur = c_nxt;
        id_cur = id_nxt;
        c_k = 0;
        if (c_cur < ntiles) c_nxt = next_chunk(id_nxt);
      }
      blk = -1;
      return -1;
    };
    // tiles loaded ahead, in order (pend[0]: the next iteration's)
    int pend[NSTAGE - 1], pblk[NSTAGE - 1];
#pragma unroll
    for (int s = 0; s < NSTAGE - 1; ++s) {
      pend[s] = next_tile(pblk[s]);
      if (pend[s] >= 0) load_tile(pend[s], s, pblk[s]);
      cp_async_commit();
    }
    for (int it = 0; pend[0] >= 0; ++it) {
      const int tile = pend[0];
#pragma unroll
      for (int s = 0; s + 1 < NSTAGE - 1; ++s) {
        pend[s] = pend[s + 1];
        pblk[s] = pblk[s + 1];
      }
      {
        int& nt = pend[NSTAGE - 2];
        nt = next_tile(pblk[NSTAGE - 2]);
        if (nt >= 0) load_tile(nt, (it + NSTAGE - 1) % NSTAGE, pblk[NSTAGE - 2]);
        cp_async_commit();
      }
      cp_async_wait<NSTAGE - 1>();
      __syncwarp();
      attend(tile, it % NSTAGE);
      __syncwarp();  // this stage is reloaded by the next iteration
    }
  }
  cp_async_wait<0>();
  const int ticket = steer ? atomicAdd(p.work_count, 1) : 0;

  // ---- merge the warps ------------------------------------------------------
#pragma unroll
  for (int nh = 0; nh < NH; ++nh)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      l_run[nh][e] += __shfl_xor_sync(0xffffffffu, l_run[nh][e], 4);
      l_run[nh][e] += __shfl_xor_sync(0xffffffffu, l_run[nh][e], 8);
      l_run[nh][e] += __shfl_xor_sync(0xffffffffu, l_run[nh][e], 16);
    }
  __syncthreads();  // pipeline buffers are reused below
  float* w_o = reinterpret_cast<float*>(smem);  // [NW][16][D]
  float* w_m = w_o + NW * 16 * D;               // [NW][16]
  float* w_l = w_m + NW * 16;                   // [NW][16]
  float* r_w = w_l + NW * 16;                   // [NW][16] merge weights
  float* r_stat = r_w + NW * 16;                // [16][2] merged max, sum
#pragma unroll
  for (int nh = 0; nh < NH; ++nh) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int head = 8 * nh + 2 * t + e;
      if (head < nrows) {
        float* dst = w_o + (warp * 16 + head) * D;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int2 ch = accumulator_channels<CK, D>(mt, g);
          dst[merge_pos<CK, D>(head, ch.x)] = o[mt][nh][e];
          dst[merge_pos<CK, D>(head, ch.y)] = o[mt][nh][2 + e];
        }
        if (g == 0) {
          w_m[warp * 16 + head] = m_run[nh][e];
          w_l[warp * 16 + head] = l_run[nh][e];
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < nrows) {
    const int row = threadIdx.x;
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, w_m[w * 16 + row]);
    float lsum = 0.f;
    for (int w = 0; w < NW; ++w) {
      const float wt = (w_m[w * 16 + row] == -INFINITY) ? 0.f : ex2(w_m[w * 16 + row] - M);
      r_w[w * 16 + row] = wt;
      lsum += wt * w_l[w * 16 + row];
    }
    r_stat[2 * row] = M;
    r_stat[2 * row + 1] = lsum;
  }
  __syncthreads();

  // (the ticket has arrived by now; its item loads while the output is written)
  const int2 next_item = steer ? cursor_item(p, *cursor, ticket) : make_int2(-1, -1);
  const bool direct = nparts == 1 && !p.force_partials;
  const int slot = p.part_offset + part;
  const uint64_t keep = direct ? 0 : l2_evict_last_policy();  // partials: kept for the merge
  const float* vs = (CK == kE4M3) ? p.v_scale + static_cast<int64_t>(hk) * D : nullptr;
  for (int i = threadIdx.x; i < nrows * D; i += NW * 32) {
    const int row = i / D;
    const int c = i - row * D;
    float acc = 0.f;
    const int pc = merge_pos<CK, D>(row, c);
#pragma unroll
    for (int w = 0; w < NW; ++w) acc += r_w[w * 16 + row] * w_o[(w * 16 + row) * D + pc];
    const float lsum_row = r_stat[2 * row + 1];  // 0: a steal-mode CTA that got no tile
    float val = lsum_row > 0.f ? acc / lsum_row : 0.f;
    if constexpr (CK == kE4M3) val *= vs[c];
    const int64_t bh = static_cast<int64_t>(b) * p.num_q_heads + hq0 + row;
    if (direct && p.cp_o) {
      p.cp_o[bh * D + c] = val;
      if (c == 0) p.cp_ml[bh] = make_float2(r_stat[2 * row], r_stat[2 * row + 1]);
    } else if (direct) {
      out[bh * D + c] = from_f32<TQ>(val);
    } else {
      st_hint(p.ws_o + (bh * p.num_partitions + slot) * D + c, val, keep);
      if (c == 0)
        st_hint(p.ws_ml + bh * p.num_partitions + slot,
                make_float2(r_stat[2 * row], r_stat[2 * row + 1]), keep);
    }
  }
  if constexpr (FUSED && CK == kE4M3) store_new_token();
  if constexpr (STEAL) {
    if (p.steal_merge && !direct) steal_merge_row<TQ, D, NW>(p, b, by, hq0, nrows, nparts, part);
  }
  if (steer) {
    cursor->u = ticket;
    cursor->item = next_item;
  }
}

// One decode CTA of the launch. Grid mode: the CTA (part, by, b) of the
// grid, with the sequence taken longest first when asked. Work-list mode:
// units (item u / hb, KV head group u % hb) taken from the ticket counter
// until the list is exhausted; each computes exactly what the CTA (part, by,
// b) of a full grid would. In cascade mode the CTA ends with the wait for the
// prefix grid.
template <typename TQ, int CK, int D, int NW, int NSTAGE, int NH, bool FUSED, bool STEAL = false>
__device__ __forceinline__ void decode_launch_cta(const DecodeParams& p) {
  // a kernel launched after this one as its programmatic dependent (the
  // split-K merge) may start as soon as every CTA here has started; it waits
  // for this grid's completion before reading anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ WorkCursor cur;
  const bool list = p.work_items != nullptr;
  int part = static_cast<int>(blockIdx.x);
  int by = static_cast<int>(blockIdx.y);
  int b = static_cast<int>(blockIdx.z);
  if (list) {
    // the plan kernel, this launch's programmatic predecessor, wrote the list
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) {
      // (batch x partitions x hb < 2^31: the host checks the bound)
      cur.n_units = min(p.work_count[1], p.batch * p.num_partitions) * units_per_item(p);
      cur.pt = launch_partition_tokens(p);
      // the first unit is the CTA's own index: no ticket to wait for
      const int u = static_cast<int>(blockIdx.x);
      cur.item = cursor_item(p, cur, u);
      cur.u = u;
    }
    __syncthreads();
  } else if (p.longest_first) {
    // the sequence of rank z in decreasing attended length
    __shared__ int s_key[kOrderMaxBatch];
    __shared__ int s_pick;
    for (int i = threadIdx.x; i < p.batch; i += NW * 32)
      s_key[i] = max(clamp_context(p, p.context_lens[i]) - p.token_start, 0);
    __syncthreads();
    for (int i = threadIdx.x; i < p.batch; i += NW * 32) {
      const int ki = s_key[i];
      int rank = 0;
      for (int j = 0; j < p.batch; ++j) rank += (s_key[j] > ki) || (s_key[j] == ki && j < i);
      if (rank == b) s_pick = i;
    }
    __syncthreads();
    b = s_pick;
  }
  while (true) {
    if (list) {
      const int u = cur.u;
      if (u >= cur.n_units) break;
      b = cur.item.x;
      part = cur.item.y;
      by = u % units_per_item(p);
      __syncthreads();  // every thread has read the cursor before it moves
      if (b < 0 || b >= p.batch || part < 0 || part >= p.num_partitions ||
          cur.pt < p.partition_tokens || cur.pt > max(p.partition_tokens, p.max_partition_tokens) ||
          (cur.pt & 15) != 0) {
        // not what the plan kernel wrote (the workspace was changed under the
        // launch): nothing is read through it
        if (threadIdx.x == 0) cursor_next(p, cur);
        __syncthreads();
        continue;
      }
    }
    decode_cta<TQ, CK, D, NW, NSTAGE, NH, FUSED, STEAL>(p, part, by, b,
                                                 list ? cur.pt : p.partition_tokens,
                                                 list ? &cur : nullptr);
    if (!list) break;
    __syncthreads();  // the cursor has moved; shared memory is free again
  }
  // cascade mode: the shared-prefix kernel runs before this one in the stream
  // with this launch as its programmatic dependent, so this grid started
  // early; it completes only after the prefix grid has, so that the merge,
  // which waits for this grid, also sees the prefix partials
  if (p.prefix_blocks > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Minimum resident CTAs per SM asked of the compiler (0: none). The
// two-column-block decode at head_dim 128 is held to 3 CTAs per SM (at most
// 170 registers; left alone the compiler takes up to 255 and the SM holds
// two); the others are left to the compiler's choice, which keeps them at
// <= 128 registers (an explicit minimum of one CTA made it take 173 for the
// one-block 16-bit decode and cost the SM its third CTA). The steal-mode
// decode at head_dim 128 is held to 3 as well.
template <int CK, int D, int NH, bool STEAL = false>
constexpr int decode_min_ctas() {
  return (D == 128 && (NH == 2 || STEAL)) ? 3 : 0;
}

// grid: (partitions, num_kv_heads * head_groups, batch), or work-list mode
// (STEAL: steal mode, a grid over one sequence)
template <typename TQ, int CK, int D, int NW, int NSTAGE, int NH, bool FUSED, bool STEAL = false>
__global__ void __launch_bounds__(NW * 32, (decode_min_ctas<CK, D, NH, STEAL>()))
    pa_decode_kernel(const DecodeParams p) {
  decode_launch_cta<TQ, CK, D, NW, NSTAGE, NH, FUSED, STEAL>(p);
}

// The same for an E4M3 cache and up to 8 query heads per KV head, held to 5
// CTAs per SM (at most 102 registers a thread): that decode is bound by
// instruction latency, and the extra warps pay (measured).
template <typename TQ, int D, int NW, int NSTAGE, bool FUSED>
__global__ void __launch_bounds__(NW * 32, 5) pa_decode_e4m3_kernel(const DecodeParams p) {
  decode_launch_cta<TQ, kE4M3, D, NW, NSTAGE, 1, FUSED>(p);
}

// ---- work list for batches of mixed lengths --------------------------------
//
// In a (partitions x head groups x sequences) grid every sequence gets as
// many partition CTAs as the longest one needs; the CTAs past a shorter
// sequence's end exit at once but still take a slot and a dispatch each, and
// the CTAs are dispatched in index order whatever their size, so the longest
// may start last. One CTA of this kernel lists the (sequence, partition)
// items instead, sorted by size (tokens of the partition) into
// kPlanBuckets classes, largest first, so that a persistent grid taking
// units from a counter starts the long ones first and ends on the short ones.
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 64;

// Size class of an item of `tiles` 16-token tiles: kPlanBuckets for a full
// partition down to 1; 0 for an empty sequence (its item writes a zero row).
__device__ __forceinline__ int plan_bucket(int tiles, int full_tiles) {
  if (tiles <= 0) return 0;
  return 1 + min(kPlanBuckets - 1, static_cast<int>(static_cast<int64_t>(tiles - 1) *
                                                    kPlanBuckets / full_tiles));
}

__global__ void __launch_bounds__(kPlanThreads) pa_decode_plan_kernel(const DecodeParams p) {
  __shared__ int s_hist[kPlanBuckets + 1];
  __shared__ int s_start[kPlanBuckets + 1];
  __shared__ unsigned long long s_work;
  __shared__ int s_span;
  __shared__ int s_pt;
  // the decode grid may be placed now; it waits for this grid to complete
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int i = threadIdx.x; i <= kPlanBuckets; i += kPlanThreads) s_hist[i] = 0;
  if (threadIdx.x == 0) {
    s_work = 0;
    s_span = 0;
  }
  __syncthreads();
  // The partition length. When one partition can hold every sequence's
  // attended span (within the room the launch staged for block ids, up to
  // 8 times the host's length) and the batch still has 4 waves of units
  // (sequences x head groups against the grid's CTAs), that: no sequence is
  // split and there is nothing to merge. Otherwise the host's times 1, 2 or
  // 4, the longest whose item is at most 3/2 of a slot's share of the
  // batch's tokens x head groups. Longer partitions mean fewer units and
  // partials; the largest items still start first.
  // (each thread keeps the length of its first sequence: the passes below
  // read it again, and a batch of up to kPlanThreads has no other)
  const int my_len = threadIdx.x < p.batch ? clamp_context(p, p.context_lens[threadIdx.x]) : 0;
  auto seq_len = [&](int b) {
    return b == static_cast<int>(threadIdx.x) ? my_len : clamp_context(p, p.context_lens[b]);
  };
  {
    unsigned long long mine = 0;
    int span = 0;
    for (int b = threadIdx.x; b < p.batch; b += kPlanThreads) {
      const int L = seq_len(b);
      if (L > 0) {
        const int n = L - seq_span(p, L).base;
        mine += static_cast<unsigned long long>(n);
        span = max(span, n);
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      mine += __shfl_xor_sync(0xffffffffu, mine, o);
      span = max(span, __shfl_xor_sync(0xffffffffu, span, o));
    }
    if ((threadIdx.x & 31) == 0) {
      atomicAdd(&s_work, mine);
      atomicMax(&s_span, span);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int host = p.partition_tokens;
    const int cap = max(host, p.max_partition_tokens);
    const int whole = (s_span + 15) & ~15;
    int pt = host;
    if (whole > host && whole <= cap &&
        static_cast<int64_t>(p.batch) * units_per_item(p) >= 4ll * max(p.list_slots, 1)) {
      pt = whole;
    } else {
      const unsigned long long share =
          s_work * static_cast<unsigned long long>(units_per_item(p)) * 3 /
          (2ull * static_cast<unsigned long long>(max(p.list_slots, 1)));
      const int cap4 = min(cap, 4 * host);
      while (2 * pt <= cap4 && static_cast<unsigned long long>(2 * pt) <= share) pt *= 2;
    }
    s_pt = pt;
  }
  __syncthreads();
  const int pt = s_pt;
  const int full_tiles = max(pt / 16, 1);
  // items of sequence b: np partitions, all full but the last (class bk)
  auto shape = [&](int b, int& np, int& bk) {
    const int L = seq_len(b);
    np = partitions_of(p, L, pt);
    if (np == 0) {  // L == 0: one item, the zero row
      np = 1;
      bk = 0;
      return;
    }
    const int last = (L - seq_span(p, L).base) - (np - 1) * pt;
    bk = plan_bucket((last + 15) / 16, full_tiles);
  };
  for (int b = threadIdx.x; b < p.batch; b += kPlanThreads) {
    int np, bk;
    shape(b, np, bk);
    if (np > 1) atomicAdd(&s_hist[kPlanBuckets], np - 1);
    atomicAdd(&s_hist[bk], 1);
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // each class's first slot, largest class first: an exclusive scan of the
    // histogram taken from bucket kPlanBuckets down, by one warp (lane l
    // holds positions PER*l .. PER*l + PER - 1 of that order)
    constexpr int PER = (kPlanBuckets + 1 + 31) / 32;
    const int lane = threadIdx.x;
    int v[PER];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int r = lane * PER + j;
      v[j] = r <= kPlanBuckets ? s_hist[kPlanBuckets - r] : 0;
      sum += v[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int at = incl - sum;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int r = lane * PER + j;
      if (r <= kPlanBuckets) s_start[kPlanBuckets - r] = at;
      at += v[j];
    }
    if (lane == 31) {
      p.work_count[0] = p.list_slots;  // the decode's ticket counter, past the first units
      p.work_count[1] = incl;  // items
      p.work_count[2] = pt;    // partition length
    }
  }
  __syncthreads();
  // (the order within a class is whatever the atomics give: every item is
  // computed the same wherever it lands)
  for (int b = threadIdx.x; b < p.batch; b += kPlanThreads) {
    int np, bk;
    shape(b, np, bk);
    if (np > 1) {
      const int at = atomicAdd(&s_start[kPlanBuckets], np - 1);
      for (int j = 0; j < np - 1; ++j) p.work_items[at + j] = make_int2(b, j);
    }
    p.work_items[atomicAdd(&s_start[bk], 1)] = make_int2(b, np - 1);
  }
}

// A merged row's four channels of lane `lane`: to `out` in TQ, or in partial
// mode (PARTIAL) to cp_o / cp_ml as fp32 with the row's (max, sum).
template <typename TQ, int D, bool PARTIAL>
__device__ __forceinline__ void write_merged(const DecodeParams& p, int64_t row, int lane,
                                             float4 a, float ws, float M) {
  const float inv = 1.f / ws;
  if constexpr (PARTIAL) {
    reinterpret_cast<float4*>(p.cp_o + row * D)[lane] =
        make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
    if (lane == 0) p.cp_ml[row] = make_float2(M, ws);
    return;
  }
  TQ* out = reinterpret_cast<TQ*>(p.out) + row * D + 4 * lane;
  out[0] = from_f32<TQ>(a.x * inv);
  out[1] = from_f32<TQ>(a.y * inv);
  out[2] = from_f32<TQ>(a.z * inv);
  out[3] = from_f32<TQ>(a.w * inv);
}

// Merge split-K partials: with per-partition max m_p (log2 units), sum l_p
// and normalised output o_p, out = sum_p w_p o_p / sum_p w_p where
// w_p = l_p * 2^(m_p - max_p m_p).
//
// A CTA has NWARPS warps; WPR warps merge one (sequence, query head) row, so
// a CTA covers NWARPS / WPR rows (the host picks WPR from the number of
// partials so that a warp has at most NL of them, up to 32 warps per row).
// Lane l owns channels 4l .. 4l+3 (float4 loads of the partial outputs).
// With one warp per row, the lanes hold the row's (max, sum) pairs and every
// load is issued before any is used. With several, each warp loads its
// partials' pairs and outputs together, weights them by its own max, and the
// WPR warps' sums are rescaled to the row's max and added in shared memory:
// the partials arrive in one round trip either way.
//
// The kernel is launched as the programmatic dependent of the kernels that
// write the partials: it waits for them to complete before reading.
template <typename TQ, int D, int WPR, int NL, int NWARPS, bool PARTIAL = false>
__global__ void __launch_bounds__(NWARPS * 32) pa_decode_reduce_kernel(const DecodeParams p) {
  static_assert(D % 4 == 0 && D <= 128, "one float4 per lane");
  static_assert(NWARPS % WPR == 0, "whole rows per CTA");
  constexpr int RPC = NWARPS / WPR;  // rows per CTA
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (p.steal_ctr && blockIdx.x == 0) {
    // the decode grid has completed: its steal counters go back to zero, so
    // that a replay of the same launch (same epoch) starts afresh
    const int n = p.batch * p.num_kv_heads * p.head_groups;
    for (int i = threadIdx.x; i < n; i += NWARPS * 32) p.steal_ctr[i] = 0ull;
  }
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int rloc = warp / WPR;
  const int wsub = warp - rloc * WPR;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * RPC + rloc;  // b * Hq + head
  const int64_t rows = static_cast<int64_t>(p.batch) * p.num_q_heads;

  __shared__ float4 s_acc[NWARPS][D / 4];
  __shared__ float s_wsum[NWARPS];
  __shared__ float s_max[NWARPS];

  int nparts = 0;
  if (row < rows) {
    const int b = static_cast<int>(row / p.num_q_heads);
    nparts = p.part_offset +
             partitions_of(p, clamp_context(p, p.context_lens[b]), launch_partition_tokens(p));
  }
  const bool work = nparts > 1 || (nparts == 1 && p.force_partials);
  const bool active = lane < D / 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if constexpr (WPR == 1) {
    // at most NL partials (the launch picks WPR = 1 only then)
    if (work) {
      const float2* ml = p.ws_ml + row * p.num_partitions;
      const float4* po = reinterpret_cast<const float4*>(p.ws_o + row * p.num_partitions * D);
      const uint64_t once = l2_evict_first_policy();  // the partials' one reader
      const float2 mine = lane < nparts ? ld_hint(ml + lane, once) : make_float2(-INFINITY, 0.f);
      // unconditional loads (indexes clamped to the row's partials and to
      // the row's D / 4 lanes; the clamped copies get weight 0 or are not
      // stored), so that they are all issued together
      const int lc = active ? lane : D / 4 - 1;
      float4 x[NL];
#pragma unroll
      for (int i = 0; i < NL; ++i)
        x[i] = ld_hint(po + static_cast<int64_t>(min(i, nparts - 1)) * (D / 4) + lc, once);
      float M = mine.x;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float wl = lane < nparts ? mine.y * ex2(mine.x - M) : 0.f;
      wsum = wl;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
#pragma unroll
      for (int i = 0; i < NL; ++i) {
        const float w = __shfl_sync(0xffffffffu, wl, i);
        acc.x += w * x[i].x;
        acc.y += w * x[i].y;
        acc.z += w * x[i].z;
        acc.w += w * x[i].w;
      }
      if (active) {
        if constexpr (PARTIAL) {
          write_merged<TQ, D, PARTIAL>(p, row, lane, acc, wsum, M);
        } else {
          TQ* out = reinterpret_cast<TQ*>(p.out) + row * D + 4 * lane;
          const float inv = 1.f / wsum;
          out[0] = from_f32<TQ>(acc.x * inv);
          out[1] = from_f32<TQ>(acc.y * inv);
          out[2] = from_f32<TQ>(acc.z * inv);
          out[3] = from_f32<TQ>(acc.w * inv);
        }
      }
    }
    return;
  }
  float mw = -INFINITY;  // this warp's max over its partials
  if (work) {
    const float2* ml = p.ws_ml + row * p.num_partitions;
    const float4* po = reinterpret_cast<const float4*>(p.ws_o + row * p.num_partitions * D);
    const uint64_t once = l2_evict_first_policy();  // the partials' last reads
    const int lc = active ? lane : D / 4 - 1;
    // this warp's partials wsub, wsub + WPR, ..., NL of them at a time: all
    // loads of a batch are issued before any is used (the row may have fewer
    // partials than the launch's plan: those past its count are not read and
    // get weight 0), and the batch is weighted by the warp's own running max,
    // so that the partials' (max, sum) pairs and outputs arrive in one round
    // trip
    for (int i0 = wsub; i0 < nparts; i0 += NL * WPR) {
      float2 mk[NL];
      float4 xk[NL];
#pragma unroll
      for (int k = 0; k < NL; ++k) {
        const int i = i0 + k * WPR;
        mk[k] = make_float2(-INFINITY, 0.f);
        xk[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < nparts) {
          mk[k] = ld_hint(ml + i, once);
          xk[k] = ld_hint(po + static_cast<int64_t>(i) * (D / 4) + lc, once);
        }
      }
      float mb = mw;
#pragma unroll
      for (int k = 0; k < NL; ++k) mb = fmaxf(mb, mk[k].x);
      // rescale what the earlier batches summed to the new max
      const float r = (mw == -INFINITY) ? 0.f : ex2(mw - mb);
      acc.x *= r;
      acc.y *= r;
      acc.z *= r;
      acc.w *= r;
      wsum *= r;
      mw = mb;
#pragma unroll
      for (int k = 0; k < NL; ++k) {
        // (an empty partial has max -inf and sum 0: weight 0)
        const float w = mk[k].x != -INFINITY ? mk[k].y * ex2(mk[k].x - mb) : 0.f;
        wsum += w;
        acc.x += w * xk[k].x;
        acc.y += w * xk[k].y;
        acc.z += w * xk[k].z;
        acc.w += w * xk[k].w;
      }
    }
  }
  if (active) s_acc[warp][lane] = acc;
  if (lane == 0) {
    s_wsum[warp] = wsum;
    s_max[warp] = mw;
  }
  __syncthreads();
  if (work && wsub == 0 && active) {
    // the row's WPR warps, each scaled from its own max to the row's
    float M = s_max[warp];
#pragma unroll
    for (int k = 1; k < WPR; ++k) M = fmaxf(M, s_max[warp + k]);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    float ws = 0.f;
#pragma unroll
    for (int k = 0; k < WPR; ++k) {
      const float mk = s_max[warp + k];
      const float r = (mk == -INFINITY) ? 0.f : ex2(mk - M);
      const float4 b4 = s_acc[warp + k][lane];
      a.x += r * b4.x;
      a.y += r * b4.y;
      a.z += r * b4.z;
      a.w += r * b4.w;
      ws += r * s_wsum[warp + k];
    }
    write_merged<TQ, D, PARTIAL>(p, row, lane, a, ws, M);
  }
}

// Merge of several pa_decode_partial results (context parallelism: each
// call covered a disjoint part of every sequence's tokens): part n of row r
// is part_o[n][r][D] with (max, sum) part_ml[n][r], in the log2 units
// pa_decode_partial writes; out[r] = sum_n w_n o_n / sum_n w_n with
// w_n = sum_n 2^(max_n - max over n). A warp per row, lane l owning channels
// 4l .. 4l+3; a part with sum 0 (no tokens) weighs nothing.
template <typename TQ, int D>
__global__ void __launch_bounds__(256) pa_merge_partials_kernel(const float* part_o,
                                                               const float2* part_ml,
                                                               int num_parts, int64_t rows,
                                                               TQ* out) {
  static_assert(D % 4 == 0 && D <= 128, "one float4 per lane");
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows || lane >= D / 4) return;
  float M = -INFINITY;
  for (int n = 0; n < num_parts; ++n) {
    const float2 v = part_ml[n * rows + r];
    if (v.y > 0.f) M = fmaxf(M, v.x);
  }
  float ws = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int n = 0; n < num_parts; ++n) {
    const float2 v = part_ml[n * rows + r];
    if (!(v.y > 0.f)) continue;
    const float w = v.y * ex2(v.x - M);
    const float4 o = reinterpret_cast<const float4*>(part_o + (n * rows + r) * D)[lane];
    ws += w;
    acc.x += w * o.x;
    acc.y += w * o.y;
    acc.z += w * o.z;
    acc.w += w * o.w;
  }
  const float inv = ws > 0.f ? 1.f / ws : 0.f;  // no part with tokens: a zero row
  TQ* o = out + r * D + 4 * lane;
  o[0] = from_f32<TQ>(acc.x * inv);
  o[1] = from_f32<TQ>(acc.y * inv);
  o[2] = from_f32<TQ>(acc.z * inv);
  o[3] = from_f32<TQ>(acc.w * inv);
}

}  // namespace pa
