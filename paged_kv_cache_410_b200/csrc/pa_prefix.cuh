// Shared-prefix (cascade) decode: the attention of every sequence over a
// prefix that all sequences of the batch share (KV cache article, section
// "PagedAttention：把操作系统的老智慧搬进推理引擎": a common system prompt is
// stored once, in blocks every sequence references).
//
// With the prefix's blocks shared, the batch's queries for one KV head form
// one dense problem: (batch x group) query rows against the same prefix
// tokens. A prefix CTA owns one KV head, one chunk of prefix tokens and
// 16 * NWP query rows (16 per warp, possibly from several sequences); its
// warps share each K/V tile through one CTA-wide cp.async pipeline. Per warp
// the layout is the row one -- all 16 MMA rows are real queries:
//   S (16 queries x 16 tokens) = Q (16 x D) . K_tile^T     [m16n8k16, 2 n-tiles]
//   O (16 x D)                += P (16 x 16) . V_tile       [P straight from S]
// Each query row's result over the chunk is a split-K partial.
//
// pa_cascade_kernel runs these prefix CTAs and the per-sequence suffix CTAs
// (decode_cta in cascade mode) in one launch, prefix CTAs first, so the
// tensor-core-heavy prefix work overlaps the HBM-bound suffix work with no
// dependency between the two; pa_decode_reduce_kernel then merges both kinds
// of partials.
#pragma once

#include "pa_decode.cuh"

namespace pa {

// A prefix stage holds one block of 16 * NSUB tokens of K and of V.
template <int CK, int D, int NSP, int NSUB>
struct PrefixSmem {
  using G = TileGeom<CK, D>;
  static constexpr int kBlockTokens = 16 * NSUB;
  static constexpr int kKBytes = NSUB * G::TB;
  static constexpr int kStageBytes = 2 * kKBytes;
  static constexpr int kPipeBytes = NSP * kStageBytes;
  // + block ids of the chunk (int32), sized at launch
};

// Rows per prefix pipeline block: 64 for 16-bit caches; 32 for E4M3, whose
// hi + lo query fragments leave fewer registers for the scores.
template <int CK>
__host__ __device__ constexpr int prefix_subtiles() {
  return CK == kE4M3 ? 2 : 4;
}

// A fragments of 16 query rows: qa[kk] = {row g | row g+8} x {k-slots 2t,2t+1 |
// 2t+8,2t+9}. E4M3: q' = q * k_scale as f16 hi + lo, with channels permuted
// within each 32-channel group gq so that a thread's K codes are contiguous:
// k-step 2gq + h holds channels 8t + 4h + {0,1} in slots 2t, 2t+1 and
// 8t + 4h + {2,3} in slots 2t+8, 2t+9.
template <typename TQ, int CK, int D>
__device__ __forceinline__ void load_query_rows(const TQ* row_g, const TQ* row_g8,
                                                const float* k_scale_row,
                                                uint32_t (&qa)[D / 16][4],
                                                uint32_t (&qalo)[CK == kE4M3 ? D / 16 : 1][4]) {
  const int t = threadIdx.x & 3;
  const TQ* rows[2] = {row_g, row_g8};
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const TQ* qr = rows[rr];
    const bool ok = qr != nullptr;
    if constexpr (CK != kE4M3) {
      const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qr);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        qa[kk][rr] = ok ? q32[(kk * 16 + 2 * t) / 2] : 0u;
        qa[kk][2 + rr] = ok ? q32[(kk * 16 + 8 + 2 * t) / 2] : 0u;
      }
    } else {
#pragma unroll
      for (int gq = 0; gq < D / 32; ++gq) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int kk = 2 * gq + h;
          const int c = gq * 32 + 8 * t + 4 * h;
          float x[4], hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x[e] = ok ? to_f32<TQ>(qr[c + e]) * k_scale_row[c + e] : 0.f;
            hi[e] = __half2float(__float2half_rn(x[e]));
            lo[e] = x[e] - hi[e];
          }
          qa[kk][rr] = pack2<false>(hi[0], hi[1]);
          qa[kk][2 + rr] = pack2<false>(hi[2], hi[3]);
          qalo[kk][rr] = pack2<false>(lo[0], lo[1]);
          qalo[kk][2 + rr] = pack2<false>(lo[2], lo[3]);
        }
      }
    }
  }
}

// Channels of output n-tile i, accumulator columns 2t and 2t+1.
template <int CK, int D>
__device__ __forceinline__ int2 row_layout_channels(int i, int t) {
  if constexpr (CK != kE4M3) return make_int2(8 * i + 2 * t, 8 * i + 2 * t + 1);
  return make_int2((D / 8) * (2 * t) + i, (D / 8) * (2 * t + 1) + i);
}

// One block of 16 * NSUB K/V rows against the warp's 16 query rows (row
// layout), with one softmax round for the whole block (FULL: all rows exist).
template <int CK, int D, int NSUB, bool FULL>
__device__ __forceinline__ void attend_block_rows(uint32_t sk_a, uint32_t sv_a, int nvalid,
                                                  float scale_log2,
                                                  const uint32_t (&qa)[D / 16][4],
                                                  const uint32_t (&qalo)[CK == kE4M3 ? D / 16 : 1][4],
                                                  float (&o)[D / 8][4], float (&m_run)[2],
                                                  float (&l_run)[2]) {
  using G = TileGeom<CK, D>;
  constexpr bool kMmaBF16 = (CK == kBF16);
  constexpr int NT = D / 8;
  constexpr int NS = 2 * NSUB;  // 8-token column tiles of S
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;

  // S = Q K^T: s[n] = {(row g, tokens 8n+2t, +1), (row g+8, same)}
  float s[NS][4];
#pragma unroll
  for (int n = 0; n < NS; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
  for (int sub = 0; sub < NSUB; ++sub) {
    if constexpr (CK != kE4M3) {
      const int lr = 16 * sub + (lane & 7) + ((lane >> 4) << 3);
      const int lc = (lane >> 3) & 1;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t k0, k1, k2, k3;
        ldmatrix_x4(k0, k1, k2, k3, sk_a + G::off(lr, 2 * kk + lc));
        mma_16816<kMmaBF16>(s[2 * sub], qa[kk], k0, k1);
        mma_16816<kMmaBF16>(s[2 * sub + 1], qa[kk], k2, k3);
      }
    } else {
#pragma unroll
      for (int gq = 0; gq < D / 32; ++gq) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const uint2 w =
              lds64(sk_a + G::off(16 * sub + g + 8 * nt, 2 * gq + (t >> 1)) + (t & 1) * 8);
          uint32_t a0, a1, b0, b1;
          e4m3x4_to_f16x2x2(w.x, a0, a1);
          e4m3x4_to_f16x2x2(w.y, b0, b1);
          mma_16816<false>(s[2 * sub + nt], qa[2 * gq], a0, a1);
          mma_16816<false>(s[2 * sub + nt], qalo[2 * gq], a0, a1);
          mma_16816<false>(s[2 * sub + nt], qa[2 * gq + 1], b0, b1);
          mma_16816<false>(s[2 * sub + nt], qalo[2 * gq + 1], b0, b1);
        }
      }
    }
  }

  // online softmax per row (log2 domain); the max is reduced over the 4
  // threads of the row group, on raw scores (the scale is positive), and each
  // exponent is one FFMA. The reference max moves only when the block max
  // exceeds it by more than kRescaleLog2, so P <= 2^kRescaleLog2 and the
  // accumulator is rarely rescaled.
  uint32_t pa[NSUB][4];
  bool grew = false;
  float alpha[2];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    float mx = -INFINITY;
#pragma unroll
    for (int n = 0; n < NS; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = FULL || 8 * n + 2 * t + e < nvalid;
        mx = fmaxf(mx, ok ? s[n][2 * rr + e] : -INFINITY);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    mx *= scale_log2;
    const bool up = mx > m_run[rr] + kRescaleLog2;  // the first block always moves it
    grew |= up;
    const float m_ref = up ? mx : m_run[rr];
    alpha[rr] = up ? ex2(m_run[rr] - m_ref) : 1.f;
    float sum = 0.f;
#pragma unroll
    for (int n = 0; n < NS; ++n) {
      float p0 = ex2(fmaf(s[n][2 * rr], scale_log2, -m_ref));
      float p1 = ex2(fmaf(s[n][2 * rr + 1], scale_log2, -m_ref));
      if constexpr (!FULL) {
        p0 = 8 * n + 2 * t < nvalid ? p0 : 0.f;
        p1 = 8 * n + 2 * t + 1 < nvalid ? p1 : 0.f;
      }
      sum += p0 + p1;
      // A fragment of k-step n/2: rows g (rr=0) / g+8 (rr=1), tokens 2t,2t+1 (+8)
      pa[n >> 1][rr + 2 * (n & 1)] = pack2<kMmaBF16>(p0, p1);
    }
    l_run[rr] = l_run[rr] * alpha[rr] + sum;
    m_run[rr] = m_ref;
  }
  if (__any_sync(0xffffffffu, grew)) {
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
  }

  // O += P V
#pragma unroll
  for (int sub = 0; sub < NSUB; ++sub) {
    if constexpr (CK != kE4M3) {
      const int lr = 16 * sub + (lane & 7) + (((lane >> 3) & 1) << 3);
      const int lc = lane >> 4;
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t v0, v1, v2, v3;
        ldmatrix_x4_trans(v0, v1, v2, v3, sv_a + G::off(lr, 2 * c + lc));
        mma_16816<kMmaBF16>(o[2 * c], pa[sub], v0, v1);
        mma_16816<kMmaBF16>(o[2 * c + 1], pa[sub], v2, v3);
      }
    } else {
      // n-tile i, column n <-> channel NT*n + i: this thread (column g) reads
      // channels [NT*g, NT*g + NT) of token rows 2t, 2t+1, 2t+8, 2t+9.
      constexpr int WORDS = NT / 4;
      uint32_t ra[4][WORDS];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int r = 16 * sub + 2 * t + (q4 & 1) + 8 * (q4 >> 1);
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
        uint32_t f[4], e[4];
        e4m3x4_to_f16x2x2(__byte_perm(ra[0][w], ra[1][w], 0x5140), f[0], f[1]);
        e4m3x4_to_f16x2x2(__byte_perm(ra[0][w], ra[1][w], 0x7362), f[2], f[3]);
        e4m3x4_to_f16x2x2(__byte_perm(ra[2][w], ra[3][w], 0x5140), e[0], e[1]);
        e4m3x4_to_f16x2x2(__byte_perm(ra[2][w], ra[3][w], 0x7362), e[2], e[3]);
#pragma unroll
        for (int k = 0; k < 4; ++k) mma_16816<false>(o[4 * w + k], pa[sub], f[k], e[k]);
      }
    }
  }
}

// One prefix CTA: KV head hk, prefix chunk `chunk`, query rows
// [16 * (colblock * NWP + warp), + 16) of the flattened (sequence, head of
// the group) rows.
template <typename TQ, int CK, int D, int NWP, int NSP>
__device__ __forceinline__ void prefix_cta(const DecodeParams& p, const int chunk,
                                           const int colblock, const int hk) {
  using G = TileGeom<CK, D>;
  constexpr int NSUB = prefix_subtiles<CK>();
  using S = PrefixSmem<CK, D, NSP, NSUB>;
  constexpr int NT = D / 8;
  constexpr int BT = S::kBlockTokens;

  extern __shared__ __align__(128) uint8_t smem[];
  int* s_bt = reinterpret_cast<int*>(smem + S::kPipeBytes);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int nrows_all = p.batch * p.group;
  const int row0 = (colblock * NWP + warp) * 16;  // this warp's first query row
  const int c0 = chunk * p.prefix_chunk_tokens;
  const int c1 = min(c0 + p.prefix_chunk_tokens, p.token_start);
  if (c0 >= c1) return;  // whole CTA: the grid covers exactly the prefix
  const int ntiles = (c1 - c0 + BT - 1) / BT;

  // ---- block ids of the chunk (the prefix entries of sequence 0's table) ---
  const int bt0 = c0 >> p.bs_log2;
  const int nbt = ((c1 - 1) >> p.bs_log2) - bt0 + 1;
  const bool bt_in_smem = nbt <= kBlockIdsInSmem;
  const int32_t* gbt = p.block_tables + bt0;
  if (bt_in_smem) {
    for (int i = threadIdx.x; i < nbt; i += NWP * 32) {
      int id = gbt[i];
      if (id < 0 || id >= p.num_blocks) {
        flag_error(PA_DEVERR_BLOCK_ID);
        id = -1;
      }
      s_bt[i] = id;
    }
  }
  auto block_id = [&](int bi) -> int {
    if (bt_in_smem) return s_bt[bi];
    int id = __ldg(gbt + bi);
    if (id < 0 || id >= p.num_blocks) {
      flag_error(PA_DEVERR_BLOCK_ID);
      id = -1;
    }
    return id;
  };

  // ---- query rows: row n is (sequence n / group, head n % group) ----------
  auto qrow = [&](int n) -> const TQ* {
    if (n >= nrows_all) return nullptr;
    const int bq = n / p.group;
    const int i = n - bq * p.group;
    return reinterpret_cast<const TQ*>(p.q) +
           (static_cast<int64_t>(bq) * p.num_q_heads + hk * p.group + i) * D;
  };
  uint32_t qa[D / 16][4];
  uint32_t qalo[CK == kE4M3 ? D / 16 : 1][4];
  load_query_rows<TQ, CK, D>(qrow(row0 + g), qrow(row0 + g + 8),
                             CK == kE4M3 ? p.k_scale + static_cast<int64_t>(hk) * D : nullptr,
                             qa, qalo);
  __syncthreads();  // s_bt ready

  // ---- CTA-wide pipeline: every warp consumes every tile -------------------
  const uint8_t* kc = reinterpret_cast<const uint8_t*>(p.k_cache);
  const uint8_t* vc = reinterpret_cast<const uint8_t*>(p.v_cache);
  const int64_t slot_stride = static_cast<int64_t>(p.num_kv_heads) * G::RB;
  const int64_t head_off = static_cast<int64_t>(hk) * G::RB;
  const int bs_mask = (1 << p.bs_log2) - 1;
  auto load_tile = [&](int tile, int stage) {
    const uint32_t sk_a = smem_addr(smem + stage * S::kStageBytes);
    const uint32_t sv_a = sk_a + S::kKBytes;
    const int tb = c0 + tile * BT;
    for (int c = threadIdx.x; c < BT * G::CPR; c += NWP * 32) {
      const int r = c / G::CPR;
      const int ch = c % G::CPR;
      const int j = tb + r;
      const int blk = j < c1 ? block_id((j >> p.bs_log2) - bt0) : -1;
      const bool ok = blk >= 0;
      const int64_t off =
          ok ? ((static_cast<int64_t>(blk) << p.bs_log2) + (j & bs_mask)) * slot_stride +
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

#pragma unroll
  for (int s = 0; s < NSP - 1; ++s) {
    if (s < ntiles) load_tile(s, s);
    cp_async_commit();
  }
  for (int it = 0; it < ntiles; ++it) {
    {
      const int nxt = it + NSP - 1;
      if (nxt < ntiles) load_tile(nxt, nxt % NSP);
      cp_async_commit();
    }
    cp_async_wait<NSP - 1>();
    __syncthreads();  // tile `it` landed for every thread's copies
    const uint32_t sk_a = smem_addr(smem + (it % NSP) * S::kStageBytes);
    const int nvalid = c1 - (c0 + it * BT);
    if (nvalid >= BT)
      attend_block_rows<CK, D, NSUB, true>(sk_a, sk_a + S::kKBytes, nvalid, p.scale_log2, qa,
                                           qalo, o, m_run, l_run);
    else
      attend_block_rows<CK, D, NSUB, false>(sk_a, sk_a + S::kKBytes, nvalid, p.scale_log2, qa,
                                            qalo, o, m_run, l_run);
    __syncthreads();  // every warp is done with the stage before it is refilled
  }
  cp_async_wait<0>();

  // ---- one partial per query row ---------------------------------------------
  const float* vs = (CK == kE4M3) ? p.v_scale + static_cast<int64_t>(hk) * D : nullptr;
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    float l = l_run[rr];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int n = row0 + g + 8 * rr;
    if (n < nrows_all) {
      const int bq = n / p.group;
      const int i = n - bq * p.group;
      const int64_t bh = static_cast<int64_t>(bq) * p.num_q_heads + hk * p.group + i;
      const float inv = 1.f / l;
      float* dst = p.ws_o + (bh * p.num_partitions + chunk) * D;
#pragma unroll
      for (int k = 0; k < NT; ++k) {
        const int2 ch = row_layout_channels<CK, D>(k, t);
        float v0 = o[k][2 * rr] * inv;
        float v1 = o[k][2 * rr + 1] * inv;
        if constexpr (CK == kE4M3) {
          v0 *= vs[ch.x];
          v1 *= vs[ch.y];
        }
        dst[ch.x] = v0;
        dst[ch.y] = v1;
      }
      if (t == 0) p.ws_ml[bh * p.num_partitions + chunk] = make_float2(m_run[rr], l);
    }
  }
}

// Cascade launch: n_prefix prefix CTAs (chunk fastest, then query-row block,
// then KV head) and n_suffix suffix CTAs (partition fastest, then KV head /
// head group, then sequence) share one grid. Blocks are dispatched roughly
// in index order, so the prefix CTAs are spread through it: prefix CTA j
// sits at block j * (ratio + 1), ratio = n_suffix / n_prefix, and the suffix
// CTAs fill the other blocks in order.
struct CascadeGrid {
  int n_prefix;
  int n_suffix;
  int ratio;
  int n_chunks;
  int n_rowblocks;
  int n_suffix_parts;
};

// Three CTAs per SM (the decode CTAs' shared-memory limit) for 16-bit caches;
// two for E4M3, whose hi + lo query fragments need more registers.
template <typename TQ, int CK, int D, int NW, int NSTAGE, int NH, int NWP, int NSP>
__global__ void __launch_bounds__(NW * 32, CK == kE4M3 ? 2 : 3)
    pa_cascade_kernel(const DecodeParams p, const CascadeGrid cg) {
  static_assert(NW == NWP, "one block size for both kinds of CTA");
  const int bid = blockIdx.x;
  const int j = bid / (cg.ratio + 1);
  if (j < cg.n_prefix && bid - j * (cg.ratio + 1) == 0) {
    const int chunk = j % cg.n_chunks;
    const int r = j / cg.n_chunks;
    prefix_cta<TQ, CK, D, NWP, NSP>(p, chunk, r % cg.n_rowblocks, r / cg.n_rowblocks);
  } else {
    const int sid = bid - min(j + 1, cg.n_prefix);  // prefix blocks before this one
    const int part = sid % cg.n_suffix_parts;
    const int r = sid / cg.n_suffix_parts;
    const int ny = p.num_kv_heads * p.head_groups;
    decode_cta<TQ, CK, D, NW, NSTAGE, NH>(p, part, r % ny, r / ny, p.partition_tokens);
  }
}

}  // namespace pa
