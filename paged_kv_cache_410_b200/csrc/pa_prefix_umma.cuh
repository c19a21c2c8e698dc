// Shared-prefix attention on the 5th-generation tensor cores (tcgen05 MMA,
// accumulators in tensor memory), for 16-bit caches.
//
// Every sequence of the batch references the same physical blocks for the
// first token_start tokens (KV cache article, section
// "PagedAttention：把操作系统的老智慧搬进推理引擎": a common prompt is stored
// once and shared). For one KV head the batch's query rows against those
// tokens are one dense problem, so a CTA takes NT tiles of 128 query rows
// (of any sequences) and one chunk of prefix tokens, 64 tokens per step;
// per tile:
//   S (128 x 64, f32, TMEM)  = Q (128 x D, smem) . K_tile^T (64 x D, smem)
//   P (128 x 64, 16-bit, TMEM) = 2^(S * scale * log2(e) - m)     [one row per thread]
//   O (128 x D, f32, TMEM)  += P (TMEM) . V_tile (64 x D, smem)
// and writes, per query row, the normalised partial (O / l, m, l) that the
// split-K merge combines with the row's suffix partials. P is written over
// the S buffer it was computed from (two 16-bit values per 32-bit column)
// and is the A operand of the P.V MMA straight from tensor memory, so P
// needs no shared memory: the CTA's tiles take 128 KB at head_dim 128, and a
// suffix decode CTA fits on the same SM.
//
// Shared-memory tiles use the 128-byte swizzle (rows of 128 bytes, 16-byte
// chunk c of row r stored at chunk c ^ (r % 8), 8-row atoms of 1024 bytes);
// a D-channel row is split into D/64 slabs of 64 channels. Q and K are
// K-major operands (channels contiguous); V is read MN-major straight from
// its token-major tile. A producer warp moves the tiles with
// TMA (3-D tensor maps over q [batch][Hq][D] and the caches [slot][Hkv][D],
// one box per cache block of >= 8 tokens and 64-channel slab, no
// multicast), one thread of an MMA warp issues the MMAs, and the partial
// outputs leave through TMA stores; every wait on a copy or an MMA is
// bounded in time. The kernel shares the GPU with the suffix decode that is
// launched after it as its programmatic dependent.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "pa_decode.cuh"

namespace pa {

constexpr int kUmmaRows = 128;    // query rows per MMA tile (M)
constexpr int kUmmaTokens = 64;   // prefix tokens per step (N of S, K of P.V)
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

// A CTA holds NT row tiles of 128 query rows, all against the same K / V
// stages (so that each stage serves NT * 128 rows), NSTAGE stages deep.
// Warps 0 .. 4*NT-1 run the softmax (warp w: tile w / 4, TMEM lanes
// 32 * (w % 4) ..), then one TMA producer warp and one MMA warp.
template <int D, int NT, int NSTAGE>
struct UmmaCfg {
  static constexpr int kSoftmaxWarps = 4 * NT;
  static constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
  static constexpr int kProducerWarp = kSoftmaxWarps;
  static constexpr int kMmaWarp = kSoftmaxWarps + 1;
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
  // TMEM columns: S of tile t, buffer b at t*128 + b*64 (P(it), 16-bit
  // pairs, over the first 32 columns of S(it)'s buffer); O of tile t at
  // NT*128 + t*D; allocated as a power of two
  static constexpr int kOCol = NT * 2 * kUmmaTokens;
  static constexpr int kColsUsed = kOCol + NT * D;
  static constexpr int kTmemCols = kColsUsed <= 256 ? 256 : 512;
  // shared memory: 1024-byte aligned pieces
  static constexpr int kSlabs = D / 64;
  static constexpr int kQTile = kSlabs * kUmmaRows * 128;     // one row tile of Q
  static constexpr int kTileSlab = kUmmaTokens * 128;          // one slab of a K/V stage
  static constexpr int kTileBytes = kSlabs * kTileSlab;        // one K or V stage
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + NT * kQTile;
  static constexpr int kV = kK + NSTAGE * kTileBytes;
  static constexpr int kBytes = kV + NSTAGE * kTileBytes;
  // the epilogue stages each tile's partial outputs (128 rows x D f32) over
  // the tiles
  static_assert(NT * kUmmaRows * D * 4 <= kBytes, "epilogue staging fits in the tiles");
  static constexpr int kSmall = 256;  // mbarriers, TMEM address, abort flag
  // requested: the tiles plus slack to align them to 1024 bytes (the small
  // items live in the slack when it has room, else after the tiles)
  static constexpr int kRequest = kBytes + 1024;
  static_assert(kColsUsed <= 512, "TMEM holds 512 columns");
};

struct UmmaGrid {
  int n_chunks;
  int n_rowtiles;     // CTAs per (KV head, chunk): NT row tiles each
  int seqs_per_tile;  // a row tile holds seqs_per_tile x group query rows (<= 128)
  int withhold_scores;  // test hook: the MMA warp issues nothing, so the softmax
                        // warps' bounded waits run out (PA_DEVERR_TIMEOUT)
  int unit_tokens;    // tokens per TMA box: min(block_size, 64)
  int num_slots;      // num_blocks * block_size (an out-of-range slot loads zeros)
};

// ---- PTX wrappers -----------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "  selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}
// Wait for the phase with parity `parity` to complete; false after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// As mbar_wait, but also gives up as soon as the CTA's abort flag (shared
// u32 at `abort`) is set, and sets it on a timeout, so that after one
// failed wait every role drains at once.
__device__ __forceinline__ bool mbar_wait_or_abort(uint32_t bar, uint32_t parity,
                                                   uint32_t abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    uint32_t a;
    asm volatile("ld.volatile.shared.u32 %0, [%1];\n" : "=r"(a) : "r"(abort));
    if (a) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      asm volatile("st.volatile.shared.u32 [%0], %1;\n" ::"r"(abort), "r"(1u) : "memory");
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
// 3-D tiled TMA load of one box at coordinates (x, y, z) into shared memory,
// completing `bar`'s transaction bytes.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%3, %4, %5}], [%2];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 4-D tiled TMA store of one box from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int x, int y,
                                             int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], "
      "[%1];\n" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_and_wait() {
  asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
  asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
}
// Barrier `id` over `count` threads that also returns whether `pred` held in
// all of them.
__device__ __forceinline__ bool bar_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n"
      "  .reg .pred p, q;\n"
      "  setp.ne.u32 p, %1, 0;\n"
      "  bar.red.and.pred q, %2, %3, p;\n"
      "  selp.u32 %0, 1, 0, q;\n"
      "}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(slot),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// Make this thread's generic-proxy shared-memory writes (st.shared,
// cp.async) visible to the tensor core's reads.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// D (TMEM) (+)= A (smem) . B (smem)^T, 16-bit inputs, f32 accumulate.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  setp.ne.b32 p, %4, 0;\n"
      "  tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D (TMEM) (+)= A (TMEM) . B (smem), 16-bit inputs, f32 accumulate; A is
// M x K with row i in TMEM lane i and two 16-bit K elements per 32-bit
// column (K = 16: 8 columns from a_tmem).
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  setp.ne.b32 p, %4, 0;\n"
      "  tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
      : "memory");
}

#define PA_R32(X)                                                                             \
  X(0), X(1), X(2), X(3), X(4), X(5), X(6), X(7), X(8), X(9), X(10), X(11), X(12), X(13),   \
      X(14), X(15), X(16), X(17), X(18), X(19), X(20), X(21), X(22), X(23), X(24), X(25),   \
      X(26), X(27), X(28), X(29), X(30), X(31)
#define PA_OUT(i) "=r"(r[i])
#define PA_IN(i) "r"(r[i])

// This warp's 32 TMEM lanes, 32 consecutive 32-bit columns from `taddr`:
// v[j] = column j of the calling thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];\n"
      : PA_R32(PA_OUT)
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};\n" ::"r"(taddr),
      PA_R32(PA_IN)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  uint32_t r[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
  tmem_st32u(taddr, r);
}
#undef PA_R32
#undef PA_OUT
#undef PA_IN
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading
// and stride byte offsets (16-byte units), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of a kind::f16 MMA with f32 accumulation, M = 128:
// A K-major, B K-major or MN-major, N columns.
template <bool BF16, int N, bool B_MN>
__host__ __device__ constexpr uint32_t umma_idesc() {
  return (1u << 4) | ((BF16 ? 1u : 0u) << 7) | ((BF16 ? 1u : 0u) << 10) |
         ((B_MN ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(kUmmaRows >> 4) << 24);
}

// ---- the kernel ---------------------------------------------------------------

// Grid: n_chunks * n_rowtiles * num_kv_heads CTAs (chunk fastest, then the
// row block, then the KV head). Roles (UmmaCfg):
//   softmax warps: thread i of tile t owns query row i of the tile (TMEM
//              lane i): sequence (rt * NT + t) * seqs_per_tile + i / group,
//              head i % group of the KV head's group;
//   producer:  TMA loads of Q and of the K and V stages, each stage refilled
//              as soon as the MMAs that read it are done;
//   MMA warp:  S(it+1) of all tiles is issued before P.V(it), so the tensor
//              core computes the next scores while the softmax warps work;
//              S(it+1) goes into the buffer that held P(it-1), so it is issued
//              once P.V(it-1) has completed.
// The roles meet only at mbarriers (full / free per stage, S full, P written,
// P.V done); every wait is bounded and a timeout aborts all roles.
template <typename TQ, int D, int NT, int NSTAGE>
__global__ void __launch_bounds__(UmmaCfg<D, NT, NSTAGE>::kThreads, 1)
    pa_prefix_umma_kernel(const DecodeParams p, const UmmaGrid ug,
                          const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_o) {
  // the suffix decode, launched after this kernel as its programmatic
  // dependent, may start on the SMs this grid leaves free as soon as every
  // CTA here has started
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr bool BF16 = std::is_same<TQ, __nv_bfloat16>::value;
  using C = UmmaCfg<D, NT, NSTAGE>;
  constexpr int SLABS = C::kSlabs;
  constexpr uint32_t kIdescS = umma_idesc<BF16, kUmmaTokens, false>();
  constexpr uint32_t kIdescPV = umma_idesc<BF16, D, true>();

  extern __shared__ __align__(128) uint8_t smem[];  // tiles aligned to 1024 below
  const uint32_t raw = smem_addr(smem);
  const uint32_t base = (raw + 1023u) & ~1023u;
  // barriers, the TMEM address, the abort flag and the chunk's block ids: in
  // the alignment slack when it holds the fixed part, else after the tiles
  const uint32_t small = (base - raw >= static_cast<uint32_t>(C::kSmall)) ? raw : base + C::kBytes;
  const uint32_t small_end = small == raw ? base : raw + C::kRequest;
  const uint32_t bar_q = small;
  const uint32_t bar_kfull = small + 8;      // + 8 * stage (<= 4 stages)
  const uint32_t bar_vfull = small + 40;     // + 8 * stage
  const uint32_t bar_kfree = small + 72;     // + 8 * stage
  const uint32_t bar_vfree = small + 104;    // + 8 * stage
  const uint32_t bar_sfull = small + 136;    // + 8 * S buffer
  const uint32_t bar_pfull = small + 168;
  const uint32_t bar_pv = small + 176;
  const uint32_t bar_done = small + 184;
  const uint32_t tmem_slot = small + 192;
  const uint32_t abort = small + 196;
  const uint32_t s_bt = small + C::kSmall;
  const uint32_t sQ = base + C::kQ;
  const uint32_t sK = base + C::kK;
  const uint32_t sV = base + C::kV;
  static_assert(NSTAGE >= 2 && NSTAGE <= 4, "stages");

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int chunk = blockIdx.x % ug.n_chunks;
  const int rt = (blockIdx.x / ug.n_chunks) % ug.n_rowtiles;
  const int hk = blockIdx.x / (ug.n_chunks * ug.n_rowtiles);
  const int c0 = chunk * p.prefix_chunk_tokens;
  const int c1 = min(c0 + p.prefix_chunk_tokens, p.token_start);
  if (c0 >= c1) return;  // uniform over the CTA, before anything is allocated
  const int nsteps = (c1 - c0 + kUmmaTokens - 1) / kUmmaTokens;
  // use i of a stage-indexed barrier completes once per NSTAGE steps
  auto stage_parity = [](int it) { return static_cast<uint32_t>((it / NSTAGE) & 1); };

  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (tid == C::kMmaWarp * 32) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(bar_kfull + 8 * i, 1);
      mbar_init(bar_vfull + 8 * i, 1);
      mbar_init(bar_kfree + 8 * i, 1);
      mbar_init(bar_vfree + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(bar_sfull + 8 * i, 1);
    mbar_init(bar_pfull, C::kSoftmaxThreads);
    mbar_init(bar_pv, 1);
    mbar_init(bar_done, 1);
    asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(abort), "r"(0u) : "memory");
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint32_t tmem;
  asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(tmem) : "r"(tmem_slot));
  bool ok = true;

  if (warp == C::kProducerWarp) {
    // ---- producer ---------------------------------------------------------
    // block ids of the chunk (prefix entries of sequence 0's table): staged
    // in shared memory when they fit in the space left, else read when used
    const int bt0 = c0 >> p.bs_log2;
    const int nbt = ((c1 - 1) >> p.bs_log2) - bt0 + 1;
    const bool bt_in_smem = s_bt + 4u * static_cast<uint32_t>(nbt) <= small_end;
    if (bt_in_smem) {
      for (int i = lane; i < nbt; i += 32) {
        int id = __ldg(p.block_tables + bt0 + i);
        if (id < 0 || id >= p.num_blocks) {
          flag_error(PA_DEVERR_BLOCK_ID);
          id = -1;
        }
        asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(s_bt + 4u * i), "r"(id) : "memory");
      }
    }
    __syncwarp();
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tm_k)) : "memory");
      asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tm_v)) : "memory");
    }
    auto block_id = [&](int j) -> int {
      const int bi = (j >> p.bs_log2) - bt0;
      int id;
      if (bt_in_smem) {
        asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(id) : "r"(s_bt + 4u * bi));
        return id;
      }
      id = __ldg(p.block_tables + bt0 + bi);
      if (id < 0 || id >= p.num_blocks) {
        flag_error(PA_DEVERR_BLOCK_ID);
        id = -1;
      }
      return id;
    };
    // One tile: a box of unit_tokens rows per (unit, slab); the warp's lanes
    // issue the boxes together, lane i the box (unit i / SLABS, slab
    // i % SLABS). Units past the chunk (and blocks with a bad id) are read at
    // an out-of-range slot: zeros.
    const int bs_mask = (1 << p.bs_log2) - 1;
    const int nbox = (kUmmaTokens / ug.unit_tokens) * SLABS;  // <= 16
    auto load_tile = [&](const CUtensorMap* map, uint32_t dst, uint32_t bar, int it) {
      if (lane == 0) mbar_arrive_expect_tx(bar, C::kTileBytes);
      if (lane < nbox) {
        const int u0 = (lane / SLABS) * ug.unit_tokens;
        const int sl = lane % SLABS;
        const int j = c0 + it * kUmmaTokens + u0;
        int slot = ug.num_slots;
        if (j < c1) {
          const int blk = block_id(j);
          if (blk >= 0) slot = (blk << p.bs_log2) + (j & bs_mask);
        }
        tma_load_3d(dst + sl * C::kTileSlab + u0 * 128, map, bar, sl * 64, hk, slot);
      }
    };
    const int qrows = ug.seqs_per_tile * p.group;
    if (lane == 0) mbar_arrive_expect_tx(bar_q, NT * SLABS * qrows * 128);
    if (lane < NT * SLABS) {
      const int t = lane / SLABS;
      const int sl = lane % SLABS;
      tma_load_3d(sQ + t * C::kQTile + sl * (kUmmaRows * 128), &tm_q, bar_q, sl * 64,
                  hk * p.group, (rt * NT + t) * ug.seqs_per_tile);
    }
    int issued = 0;  // tiles (K and V) issued so far
    for (int it = 0; it < nsteps; ++it) {
      const int st = it % NSTAGE;
      const uint32_t par = stage_parity(it - NSTAGE);
      if (it >= NSTAGE &&
          !__all_sync(0xffffffffu, mbar_wait_or_abort(bar_kfree + 8 * st, par, abort)))
        break;
      load_tile(&tm_k, sK + st * C::kTileBytes, bar_kfull + 8 * st, it);
      if (it >= NSTAGE &&
          !__all_sync(0xffffffffu, mbar_wait_or_abort(bar_vfree + 8 * st, par, abort))) {
        issued = 2 * it + 1;
        break;
      }
      load_tile(&tm_v, sV + st * C::kTileBytes, bar_vfull + 8 * st, it);
      issued = 2 * it + 2;
    }
    // every issued copy has landed before the CTA can exit (normally the
    // MMA warp has waited for all of them already)
    if (lane == 0) {
      for (int i = issued - 2 * NSTAGE > 0 ? issued - 2 * NSTAGE : 0; i < issued; ++i) {
        const int it = i >> 1;
        const uint32_t bar = ((i & 1) ? bar_vfull : bar_kfull) + 8 * (it % NSTAGE);
        mbar_wait(bar, stage_parity(it));
      }
      mbar_wait(bar_q, 0);
    }
  } else if (warp == C::kMmaWarp) {
    // ---- MMA issue --------------------------------------------------------
    if (lane == 0) {
      auto issue_s = [&](int i) -> bool {
        if (!mbar_wait_or_abort(bar_kfull + 8 * (i % NSTAGE), stage_parity(i), abort))
          return false;
        // S buffer i & 1 holds P(i - 2) until P.V(i - 2) has read it
        if (i >= 2 && !mbar_wait_or_abort(bar_pv, static_cast<uint32_t>((i - 2) & 1), abort))
          return false;
        tc_fence_after();
        const uint32_t kst = sK + (i % NSTAGE) * C::kTileBytes;
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sw128_desc(
                sQ + t * C::kQTile + (kk >> 2) * (kUmmaRows * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t b =
                sw128_desc(kst + (kk >> 2) * C::kTileSlab + (kk & 3) * 32, 16, 1024);
            umma_f16(tmem + t * 2 * kUmmaTokens + (i & 1) * kUmmaTokens, a, b, kIdescS, kk > 0);
          }
        umma_commit(bar_sfull + 8 * (i & 1));
        umma_commit(bar_kfree + 8 * (i % NSTAGE));
        return true;
      };
      ok = mbar_wait_or_abort(bar_q, 0, abort) && !ug.withhold_scores && issue_s(0);
      for (int it = 0; ok && it < nsteps; ++it) {
        if (it + 1 < nsteps && !issue_s(it + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait_or_abort(bar_pfull, static_cast<uint32_t>(it & 1), abort) ||
            !mbar_wait_or_abort(bar_vfull + 8 * (it % NSTAGE), stage_parity(it), abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t vst = sV + (it % NSTAGE) * C::kTileBytes;
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int kk = 0; kk < kUmmaTokens / 16; ++kk) {
            // P(it): 16 tokens = 8 columns of tile t's S buffer it & 1
            const uint32_t a = tmem + t * 2 * kUmmaTokens + (it & 1) * kUmmaTokens + kk * 8;
            const uint64_t b = sw128_desc(vst + kk * 16 * 128, C::kTileSlab, 1024);
            umma_f16_tmem_a(tmem + C::kOCol + t * D, a, b, kIdescPV, (it > 0 || kk > 0) ? 1u : 0u);
          }
        umma_commit(bar_pv);
        umma_commit(bar_vfree + 8 * (it % NSTAGE));
      }
      // every issued MMA has completed before TMEM is released
      umma_commit(bar_done);
      mbar_wait(bar_done, 0);
    }
  } else {
    // ---- softmax warps --------------------------------------------------------
    const int tile = warp >> 2;
    const int my_row = tid & (kUmmaRows - 1);  // row within the tile = TMEM lane
    const uint32_t t_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + t_lane + tile * 2 * kUmmaTokens;
    const uint32_t tO = tmem + t_lane + C::kOCol + tile * D;
    float m_run = -INFINITY;
    float l_run = 0.f;
    for (int it = 0; it < nsteps; ++it) {
      ok = __all_sync(0xffffffffu, mbar_wait_or_abort(bar_sfull + 8 * (it & 1),
                                                      static_cast<uint32_t>((it >> 1) & 1), abort));
      if (!ok) break;
      tc_fence_after();
      float s[kUmmaTokens];
      {
        float h[32];
        tmem_ld32(tS + (it & 1) * kUmmaTokens, h);
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = h[j];
        tmem_ld32(tS + (it & 1) * kUmmaTokens + 32, h);
#pragma unroll
        for (int j = 0; j < 32; ++j) s[32 + j] = h[j];
        tmem_ld_wait();
      }

      const int nvalid = c1 - (c0 + it * kUmmaTokens);
      const bool full = nvalid >= kUmmaTokens;  // every step but a chunk's ragged last one
      // row max as a tree of 8 independent partial maxima (a thread owns the
      // whole row, so a single running max would be a 64-long dependency chain)
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = -INFINITY;
      if (full) {
#pragma unroll
        for (int j = 0; j < kUmmaTokens; ++j) m8[j & 7] = fmaxf(m8[j & 7], s[j]);
      } else {
#pragma unroll
        for (int j = 0; j < kUmmaTokens; ++j)
          m8[j & 7] = fmaxf(m8[j & 7], j < nvalid ? s[j] : -INFINITY);
      }
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      mx *= p.scale_log2;
      const bool up = mx > m_run + kRescaleLog2;  // the first step always moves it
      const float m_ref = up ? mx : m_run;
      const float alpha = up ? ex2(m_run - m_ref) : 1.f;

      // P row (64 tokens, packed in pairs), computed while P.V(it-1) may
      // still be running, and written over S(it) (this thread's TMEM lane)
      uint32_t pw[kUmmaTokens / 2];
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};  // partial sums (as the max: no long chain)
      auto expo = [&](int j) { return ex2(fmaf(s[j], p.scale_log2, -m_ref)); };
      if (full) {
#pragma unroll
        for (int j = 0; j < kUmmaTokens; j += 2) {
          const float p0 = expo(j);
          const float p1 = expo(j + 1);
          sum4[(j >> 1) & 3] += p0 + p1;
          pw[j / 2] = pack2<BF16>(p0, p1);
        }
      } else {
#pragma unroll
        for (int j = 0; j < kUmmaTokens; j += 2) {
          const float p0 = j < nvalid ? expo(j) : 0.f;
          const float p1 = j + 1 < nvalid ? expo(j + 1) : 0.f;
          sum4[(j >> 1) & 3] += p0 + p1;
          pw[j / 2] = pack2<BF16>(p0, p1);
        }
      }
      const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      l_run = l_run * alpha + sum;
      m_run = m_ref;
      static_assert(kUmmaTokens / 2 == 32, "one 32-column store of P");
      tmem_st32u(tS + (it & 1) * kUmmaTokens, pw);

      if (it > 0) {  // P.V(it-1) done: O is free
        ok = __all_sync(0xffffffffu,
                        mbar_wait_or_abort(bar_pv, static_cast<uint32_t>((it - 1) & 1), abort));
        if (!ok) {
          tmem_st_wait();  // (P's store) before the CTA drains
          break;
        }
        tc_fence_after();
        // rows whose reference max moved rescale their O row
        if (__any_sync(0xffffffffu, up)) {
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            float o[32];
            tmem_ld32(tO + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(tO + c, o);
          }
        }
      }
      tmem_st_wait();  // P (and a rescaled O) in tensor memory
      tc_fence_before();
      mbar_arrive(bar_pfull);
    }
    if (ok) {  // the last P.V
      ok = __all_sync(0xffffffffu,
                      mbar_wait_or_abort(bar_pv, static_cast<uint32_t>((nsteps - 1) & 1), abort));
      tc_fence_after();
    }

    // ---- one partial per query row -------------------------------------------
    // Rows are staged in shared memory (free now: every MMA has completed)
    // as D/32 quarters of 128-byte rows with the 128-byte swizzle (conflict
    // free), then one thread per tile stores the tile with D/32 TMA stores
    // into ws_o viewed as [batch][Hq][partition][D] (rows past the batch or
    // the tile's sequences are clipped by the map / the box).
    const int si = my_row / p.group;
    const int bq = (rt * NT + tile) * ug.seqs_per_tile + si;
    const bool write = ok && si < ug.seqs_per_tile && bq < p.batch;
    const int64_t bh =
        static_cast<int64_t>(bq) * p.num_q_heads + hk * p.group + (my_row - si * p.group);
    const float inv = 1.f / l_run;
    constexpr int kQuarter = kUmmaRows * 128;  // 32 channels of 128 rows
    const uint32_t stage = base + tile * (D / 32) * kQuarter;
    if (ok) {
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float o[32];
        tmem_ld32(tO + c, o);
        tmem_ld_wait();
        const uint32_t row = stage + (c / 32) * kQuarter + my_row * 128;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"r"(
                           row + ((e ^ (my_row & 7)) << 4)),
                       "f"(o[4 * e] * inv), "f"(o[4 * e + 1] * inv), "f"(o[4 * e + 2] * inv),
                       "f"(o[4 * e + 3] * inv)
                       : "memory");
      }
    }
    fence_async_smem();
    if (bar_and(1 + tile, kUmmaRows, ok) && my_row == 0) {
#pragma unroll
      for (int q = 0; q < D / 32; ++q)
        tma_store_4d(&tm_o, stage + q * kQuarter, 32 * q, chunk, hk * p.group,
                     (rt * NT + tile) * ug.seqs_per_tile);
      bulk_commit_and_wait();
    }
    if (write) p.ws_ml[bh * p.num_partitions + chunk] = make_float2(m_run, l_run);
  }

  tc_fence_before();
  __syncthreads();
  uint32_t aborted;
  asm volatile("ld.volatile.shared.u32 %0, [%1];\n" : "=r"(aborted) : "r"(abort));
  if (aborted && tid == 0) flag_error(PA_DEVERR_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace pa
