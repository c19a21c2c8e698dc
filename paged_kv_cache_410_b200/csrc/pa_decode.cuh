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
// Tensor cores. Rows of the m16n8k16 MMA are the group's query heads (up to
// 16; padding rows are zero), columns are 8 tokens: S = Q K^T with K tiles
// loaded by ldmatrix, then O += P V with P taken straight from the S
// accumulators and V tiles loaded by ldmatrix.trans. For an E4M3 cache the
// codes are widened to f16 (exactly) in registers; the K scale is folded into
// the query (as an f16 hi + lo pair so the fold costs no precision) and the V
// scale is applied to the merged output.
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
};

enum CacheKind { kF16 = 0, kBF16 = 1, kE4M3 = 2 };

// Block ids of one partition staged in shared memory (longer slices are read
// from global memory row by row).
constexpr int kBlockIdsInSmem = 1024;

template <int CK, int D>
struct TileGeom {
  static constexpr int ES = (CK == kE4M3) ? 1 : 2;  // bytes per cache element
  static constexpr int RB = D * ES;                  // bytes per token row (one head)
  static constexpr int CPR = RB / 16;                // 16-byte chunks per row
  static constexpr int TB = 16 * RB;                 // one 16-token tile of K (or V)
  static_assert(CPR == 4 || CPR == 8 || CPR == 16, "unsupported row size");
  // Byte offset of 16-byte chunk `c` of row `r` inside a tile. Rows of 128 B
  // or more XOR the low three chunk bits with the row, so that 8 rows read
  // at one chunk column hit 8 distinct bank groups; 64-byte rows are
  // swizzled per 128-byte line instead.
  __device__ __forceinline__ static uint32_t off(int r, int c) {
    if constexpr (CPR >= 8) {
      return static_cast<uint32_t>(r * RB + ((c ^ (r & 7)) << 4));
    } else {
      const int u = r * CPR + c;
      const int line = r >> 1;
      return static_cast<uint32_t>(((u & ~7) | ((u & 7) ^ (line & 7))) << 4);
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
};

template <typename TQ, int CK, int D, int NW, int NSTAGE, bool TWO_ROWS>
__global__ void __launch_bounds__(NW * 32)
    pa_decode_kernel(const DecodeParams p) {
  using G = TileGeom<CK, D>;
  using S = DecodeSmem<CK, D, NW, NSTAGE>;
  constexpr bool kMmaBF16 = (CK == kBF16);  // MMA operand type (E4M3 widens to f16)
  constexpr int KSTEPS = D / 16;
  constexpr int NT = D / 8;  // n-tiles of the P.V product

  extern __shared__ __align__(128) uint8_t smem[];
  int* s_bt = reinterpret_cast<int*>(smem + S::kMainBytes);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane >> 2;  // MMA group id: query-head row / token column
  const int t = lane & 3;   // thread in group

  const int b = blockIdx.z;
  const int hk = blockIdx.y / p.head_groups;
  const int hgrp = blockIdx.y - hk * p.head_groups;
  const int part = blockIdx.x;
  const int row0 = hgrp * 16;
  const int nrows = min(16, p.group - row0);
  const int hq0 = hk * p.group + row0;

  // ---- sequence length, checked against what the launch covers ----------
  int L = p.context_lens[b];
  const int64_t table_cap = static_cast<int64_t>(p.max_blocks_per_seq) << p.bs_log2;
  const int cap = static_cast<int>(table_cap < p.max_context ? table_cap : p.max_context);
  if (L < 0 || L > cap) {
    if (threadIdx.x == 0 && part == 0 && blockIdx.y == 0) flag_error(PA_DEVERR_CONTEXT_LEN);
    L = L < 0 ? 0 : cap;
  }
  const int PT = p.partition_tokens;
  const int nparts = (L + PT - 1) / PT;
  if (part >= (nparts > 0 ? nparts : 1)) return;

  TQ* out = reinterpret_cast<TQ*>(p.out);
  if (L == 0) {
    for (int i = threadIdx.x; i < nrows * D; i += NW * 32)
      out[(static_cast<int64_t>(b) * p.num_q_heads + hq0 + i / D) * D + (i % D)] =
          from_f32<TQ>(0.f);
    return;
  }
  const int t0 = part * PT;
  const int t1 = min(t0 + PT, L);
  const int ntiles = (t1 - t0 + 15) >> 4;

  // ---- block ids of this partition -> shared memory ----------------------
  // (up to kBlockIdsInSmem of them; a longer slice is read from global
  // memory per row instead)
  const int bt0 = t0 >> p.bs_log2;
  const int nbt = ((t1 - 1) >> p.bs_log2) - bt0 + 1;
  const bool bt_in_smem = nbt <= kBlockIdsInSmem;
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

  // ---- query fragments (A operand, rows = query heads) -------------------
  const TQ* qbase = reinterpret_cast<const TQ*>(p.q) +
                    (static_cast<int64_t>(b) * p.num_q_heads + hq0) * D;
  const bool rlo = g < nrows;
  const bool rhi = TWO_ROWS && (g + 8 < nrows);
  uint32_t qa[KSTEPS][4];
  uint32_t qlo[CK == kE4M3 ? KSTEPS : 1][4];
  if constexpr (CK != kE4M3) {
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const int c0 = kk * 16 + 2 * t;
      const uint32_t* r0 = reinterpret_cast<const uint32_t*>(qbase + g * D);
      const uint32_t* r1 = reinterpret_cast<const uint32_t*>(qbase + (g + 8) * D);
      qa[kk][0] = rlo ? r0[c0 / 2] : 0u;
      qa[kk][1] = rhi ? r1[c0 / 2] : 0u;
      qa[kk][2] = rlo ? r0[(c0 + 8) / 2] : 0u;
      qa[kk][3] = rhi ? r1[(c0 + 8) / 2] : 0u;
    }
  } else {
    // E4M3: q' = q * k_scale[hk][:], split into f16 hi + lo. K-slot mapping
    // per 32-channel group gq: k-step 2gq holds channels 8t+{0,1} (slots
    // 2t,2t+1) and 8t+{2,3} (slots 2t+8,2t+9); k-step 2gq+1 holds 8t+{4,5}
    // and 8t+{6,7}. The K fragments below use the same mapping.
    const float* ks = p.k_scale + static_cast<int64_t>(hk) * D;
#pragma unroll
    for (int gq = 0; gq < D / 32; ++gq) {
#pragma unroll
      for (int half_ = 0; half_ < 2; ++half_) {
        const int kk = 2 * gq + half_;
        const int cA = gq * 32 + 8 * t + 4 * half_;  // channels cA, cA+1 | cA+2, cA+3
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const bool ok = rr == 0 ? rlo : rhi;
          const TQ* qr = qbase + (g + 8 * rr) * D;
          float x[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) x[e] = ok ? to_f32<TQ>(qr[cA + e]) * ks[cA + e] : 0.f;
          float h[4], l[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            h[e] = __half2float(__float2half_rn(x[e]));
            l[e] = x[e] - h[e];
          }
          qa[kk][rr] = pack2<false>(h[0], h[1]);
          qa[kk][2 + rr] = pack2<false>(h[2], h[3]);
          qlo[kk][rr] = pack2<false>(l[0], l[1]);
          qlo[kk][2 + rr] = pack2<false>(l[2], l[3]);
        }
      }
    }
  }
  __syncthreads();  // s_bt ready

  // ---- per-warp pipeline over this warp's tiles ---------------------------
  uint8_t* wbuf = smem + warp * NSTAGE * S::kStageBytes;
  const uint8_t* kc = reinterpret_cast<const uint8_t*>(p.k_cache);
  const uint8_t* vc = reinterpret_cast<const uint8_t*>(p.v_cache);
  const int64_t head_off = static_cast<int64_t>(hk) * G::RB;
  const int64_t slot_stride = static_cast<int64_t>(p.num_kv_heads) * G::RB;
  const int bs_mask = (1 << p.bs_log2) - 1;

  auto load_tile = [&](int tile, int stage) {
    uint8_t* sk = wbuf + stage * S::kStageBytes;
    const uint32_t sk_a = smem_addr(sk);
    const uint32_t sv_a = sk_a + G::TB;
    const int tb = t0 + tile * 16;
#pragma unroll
    for (int i = 0; i < G::CPR / 2; ++i) {
      const int c = lane + 32 * i;
      const int r = c / G::CPR;
      const int ch = c % G::CPR;
      const int j = tb + r;
      int blk = -1;
      if (j < t1) {
        const int bi = (j >> p.bs_log2) - bt0;
        if (bt_in_smem) {
          blk = s_bt[bi];
        } else {
          blk = __ldg(gbt + bi);
          if (blk < 0 || blk >= p.num_blocks) {
            flag_error(PA_DEVERR_BLOCK_ID);
            blk = -1;
          }
        }
      }
      const bool ok = blk >= 0;
      const int64_t off = ok ? ((static_cast<int64_t>(blk) << p.bs_log2) + (j & bs_mask)) *
                                       slot_stride +
                                   head_off + ch * 16
                             : 0;
      const uint32_t so = G::off(r, ch);
      cp_async_16(sk_a + so, kc + off, ok ? 16u : 0u);
      cp_async_16(sv_a + so, vc + off, ok ? 16u : 0u);
    }
  };

  float o[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};

  const int my_tiles = warp < ntiles ? (ntiles - warp + NW - 1) / NW : 0;
#pragma unroll
  for (int s = 0; s < NSTAGE - 1; ++s) {
    if (s < my_tiles) load_tile(warp + s * NW, s);
    cp_async_commit();
  }

  for (int it = 0; it < my_tiles; ++it) {
    {
      const int nxt = it + NSTAGE - 1;
      if (nxt < my_tiles) load_tile(warp + nxt * NW, nxt % NSTAGE);
      cp_async_commit();
    }
    cp_async_wait<NSTAGE - 1>();
    __syncwarp();

    const int stage = it % NSTAGE;
    const uint32_t sk_a = smem_addr(wbuf + stage * S::kStageBytes);
    const uint32_t sv_a = sk_a + G::TB;
    const int tile = warp + it * NW;
    const int nvalid = t1 - (t0 + tile * 16);  // tokens of this tile that exist (>= 1)

    // S = Q K^T for 16 tokens: s[nt] covers tokens 8nt .. 8nt+7
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    if constexpr (CK != kE4M3) {
      const int lr = (lane & 7) + ((lane >> 4) << 3);
      const int lc = (lane >> 3) & 1;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        uint32_t k0, k1, k2, k3;
        ldmatrix_x4(k0, k1, k2, k3, sk_a + G::off(lr, 2 * kk + lc));
        mma_16816<kMmaBF16>(s[0], qa[kk], k0, k1);
        mma_16816<kMmaBF16>(s[1], qa[kk], k2, k3);
      }
    } else {
#pragma unroll
      for (int gq = 0; gq < D / 32; ++gq) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int r = g + 8 * nt;
          const uint2 w = lds64(sk_a + G::off(r, 2 * gq + (t >> 1)) + (t & 1) * 8);
          uint32_t a0, a1, b0, b1;
          e4m3x4_to_f16x2x2(w.x, a0, a1);
          e4m3x4_to_f16x2x2(w.y, b0, b1);
          mma_16816<false>(s[nt], qa[2 * gq], a0, a1);
          mma_16816<false>(s[nt], qlo[2 * gq], a0, a1);
          mma_16816<false>(s[nt], qa[2 * gq + 1], b0, b1);
          mma_16816<false>(s[nt], qlo[2 * gq + 1], b0, b1);
        }
      }
    }

    // online softmax over the tile (log2 domain); row halves rr: g, g + 8
    uint32_t pa[4];
#pragma unroll
    for (int rr = 0; rr < (TWO_ROWS ? 2 : 1); ++rr) {
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = (e >> 1) * 8 + 2 * t + (e & 1);
        const float v = s[e >> 1][2 * rr + (e & 1)] * p.scale_log2;
        x[e] = tok < nvalid ? v : -INFINITY;
      }
      float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[rr], mx);  // finite: token 0 of the tile exists
      const float alpha = ex2(m_run[rr] - m_new);
      float pe[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pe[e] = ex2(x[e] - m_new);
      l_run[rr] = l_run[rr] * alpha + (pe[0] + pe[1]) + (pe[2] + pe[3]);
      m_run[rr] = m_new;
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        o[i][2 * rr] *= alpha;
        o[i][2 * rr + 1] *= alpha;
      }
      pa[rr] = pack2<kMmaBF16>(pe[0], pe[1]);      // tokens 2t, 2t+1
      pa[2 + rr] = pack2<kMmaBF16>(pe[2], pe[3]);  // tokens 8+2t, 9+2t
    }
    if constexpr (!TWO_ROWS) {
      pa[1] = 0u;
      pa[3] = 0u;
    }

    // O += P V
    if constexpr (CK != kE4M3) {
      const int lr = (lane & 7) + (((lane >> 3) & 1) << 3);
      const int lc = lane >> 4;
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t v0, v1, v2, v3;
        ldmatrix_x4_trans(v0, v1, v2, v3, sv_a + G::off(lr, 2 * c + lc));
        mma_16816<kMmaBF16>(o[2 * c], pa, v0, v1);
        mma_16816<kMmaBF16>(o[2 * c + 1], pa, v2, v3);
      }
    } else {
      // n-tile i, column n <-> channel NT*n + i: this thread (column g) owns
      // channels [NT*g, NT*g + NT) of token rows 2t, 2t+1, 2t+8, 2t+9.
      constexpr int WORDS = NT / 4;
      uint32_t ra[4][WORDS];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int r = 2 * t + (q4 & 1) + 8 * (q4 >> 1);
        const int byte0 = NT * g;
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
        uint32_t lo01, hi01, lo89, hi89, f0, f1, f2, f3, e0, e1, e2, e3;
        lo01 = __byte_perm(ra[0][w], ra[1][w], 0x5140);
        hi01 = __byte_perm(ra[0][w], ra[1][w], 0x7362);
        lo89 = __byte_perm(ra[2][w], ra[3][w], 0x5140);
        hi89 = __byte_perm(ra[2][w], ra[3][w], 0x7362);
        e4m3x4_to_f16x2x2(lo01, f0, f1);
        e4m3x4_to_f16x2x2(hi01, f2, f3);
        e4m3x4_to_f16x2x2(lo89, e0, e1);
        e4m3x4_to_f16x2x2(hi89, e2, e3);
        mma_16816<false>(o[4 * w + 0], pa, f0, e0);
        mma_16816<false>(o[4 * w + 1], pa, f1, e1);
        mma_16816<false>(o[4 * w + 2], pa, f2, e2);
        mma_16816<false>(o[4 * w + 3], pa, f3, e3);
      }
    }
    __syncwarp();  // this stage is reloaded by the next iteration
  }
  cp_async_wait<0>();

  // ---- merge the warps ------------------------------------------------------
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 1);
    l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 2);
  }
  __syncthreads();  // pipeline buffers are reused below
  float* w_o = reinterpret_cast<float*>(smem);  // [NW][16][D]
  float* w_m = w_o + NW * 16 * D;               // [NW][16]
  float* w_l = w_m + NW * 16;                   // [NW][16]
  float* r_w = w_l + NW * 16;                   // [NW][16] merge weights
  float* r_stat = r_w + NW * 16;                // [16][2] merged max, 1/sum
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int row = g + 8 * rr;
    if (rr == 1 && !TWO_ROWS) break;
    if (row < nrows) {
      float* dst = w_o + (warp * 16 + row) * D;
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        int c0, c1;
        if constexpr (CK != kE4M3) {
          c0 = 8 * i + 2 * t;
          c1 = c0 + 1;
        } else {
          c0 = NT * (2 * t) + i;
          c1 = NT * (2 * t + 1) + i;
        }
        dst[c0] = o[i][2 * rr];
        dst[c1] = o[i][2 * rr + 1];
      }
      if (t == 0) {
        w_m[warp * 16 + row] = m_run[rr];
        w_l[warp * 16 + row] = l_run[rr];
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

  const bool direct = nparts == 1;
  const float* vs = (CK == kE4M3) ? p.v_scale + static_cast<int64_t>(hk) * D : nullptr;
  for (int i = threadIdx.x; i < nrows * D; i += NW * 32) {
    const int row = i / D;
    const int c = i - row * D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) acc += r_w[w * 16 + row] * w_o[(w * 16 + row) * D + c];
    float val = acc / r_stat[2 * row + 1];
    if constexpr (CK == kE4M3) val *= vs[c];
    const int64_t bh = static_cast<int64_t>(b) * p.num_q_heads + hq0 + row;
    if (direct) {
      out[bh * D + c] = from_f32<TQ>(val);
    } else {
      p.ws_o[(bh * p.num_partitions + part) * D + c] = val;
      if (c == 0)
        p.ws_ml[bh * p.num_partitions + part] =
            make_float2(r_stat[2 * row], r_stat[2 * row + 1]);
    }
  }
}

// Merge split-K partials: with per-partition max m_p (log2 units), sum l_p
// and normalised output o_p, out = sum_p w_p o_p / sum_p w_p where
// w_p = l_p * 2^(m_p - max_p m_p).
template <typename TQ, int D>
__global__ void __launch_bounds__(128) pa_decode_reduce_kernel(const DecodeParams p) {
  const int hq = blockIdx.x;
  const int b = blockIdx.y;
  int L = p.context_lens[b];
  const int64_t table_cap = static_cast<int64_t>(p.max_blocks_per_seq) << p.bs_log2;
  const int cap = static_cast<int>(table_cap < p.max_context ? table_cap : p.max_context);
  L = L < 0 ? 0 : (L > cap ? cap : L);
  const int nparts = (L + p.partition_tokens - 1) / p.partition_tokens;
  if (nparts <= 1) return;
  const int64_t bh = static_cast<int64_t>(b) * p.num_q_heads + hq;
  const float2* ml = p.ws_ml + bh * p.num_partitions;
  const float* po = p.ws_o + bh * p.num_partitions * D;

  __shared__ float s_w[256];
  __shared__ float s_red[4];
  // max over partitions
  float M = -INFINITY;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) M = fmaxf(M, ml[i].x);
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = M;
  __syncthreads();
  M = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
  __syncthreads();

  float acc[(D + 127) / 128] = {};
  float wsum = 0.f;
  for (int base = 0; base < nparts; base += 256) {
    const int n = min(256, nparts - base);
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const float2 v = ml[base + i];
      s_w[i] = v.y * ex2(v.x - M);
    }
    __syncthreads();
    for (int i = 0; i < n; ++i) {
      const float w = s_w[i];
      wsum += w;
#pragma unroll
      for (int k = 0; k < (D + 127) / 128; ++k) {
        const int c = threadIdx.x + 128 * k;
        if (c < D) acc[k] += w * po[static_cast<int64_t>(base + i) * D + c];
      }
    }
    __syncthreads();
  }
  TQ* out = reinterpret_cast<TQ*>(p.out);
#pragma unroll
  for (int k = 0; k < (D + 127) / 128; ++k) {
    const int c = threadIdx.x + 128 * k;
    if (c < D) out[bh * D + c] = from_f32<TQ>(acc[k] / wsum);
  }
}

}  // namespace pa
