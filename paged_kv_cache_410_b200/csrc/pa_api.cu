// Host side of the C ABI declared in include/pa_api.h: argument checks,
// split-K planning, template dispatch and launches. All kernels of the
// library live in this one translation unit (they share the device error
// word).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <type_traits>
#include <mutex>
#include <unordered_map>
#include <unordered_set>
#include <utility>

#include "pa_api.h"
#include "pa_append_copy.cuh"
#include "pa_common.cuh"
#include "pa_decode.cuh"
#include "pa_prefix.cuh"
#include "pa_prefix_umma.cuh"

namespace {

// Build-time tuning of the decode CTA (warps, and cp.async stages per warp).
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 2
#endif

constexpr int kNumSMs = 148;         // B200
constexpr int kDecodeWarps = PA_DECODE_WARPS;
constexpr int kDecodeStages = PA_DECODE_STAGES;
constexpr int kPartitionRowBytes = 128 * 1024;  // K bytes of one KV head per partition
constexpr int kMinAutoPartition = 64;

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool pow2_log(int v, int* lg) {
  if (v <= 0 || (v & (v - 1)) != 0) return false;
  int l = 0;
  while ((1 << l) < v) ++l;
  *lg = l;
  return true;
}

pa_status check_cache(const pa_cache_desc* cd, int* bs_log2) {
  if (!cd) return PA_ERR_INVALID_ARG;
  if (cd->num_blocks <= 0 || cd->num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
  if (!pow2_log(cd->block_size, bs_log2) || cd->block_size > 256) return PA_ERR_INVALID_ARG;
  if (cd->cache_dtype != PA_F16 && cd->cache_dtype != PA_BF16 && cd->cache_dtype != PA_E4M3)
    return PA_ERR_INVALID_ARG;
  if (cd->head_dim != 64 && cd->head_dim != 128) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

int64_t elem_bytes(int dtype) { return dtype == PA_E4M3 ? 1 : 2; }

// Partition length used when the caller passes 0: the tokens whose K rows of
// one KV head take 128 KB (512 at fp16/bf16 and head_dim 128, 1024 for E4M3
// or head_dim 64), halved (down to 64) while the launch would have fewer
// than two CTAs per SM. When the sequences alone are fewer than one wave of
// CTAs (batch x KV heads below kWaveCtas, so the split is what fills the
// GPU: long contexts at small batch), the partition is then lengthened so
// that the CTAs make whole waves: of equal CTAs, a last partial wave costs
// as long as a full one. Several sequences (a work-list launch, whose plan
// may lengthen the partitions further) take the shortest such length; a
// single sequence (a grid launch) takes the fewest waves whose partitions
// stay within kMaxWavePartition tokens -- one wave where it can: measured
// on the 131072-token context at batch 1, one wave of 440 CTAs read 0.834
// of the copy bandwidth, two waves 0.814, four waves 0.792.
constexpr int kDecodeCtasPerSm = 3;  // decode CTAs resident per SM at head_dim 128
constexpr int64_t kWaveCtas = int64_t{kDecodeCtasPerSm} * kNumSMs;
constexpr int64_t kMaxWavePartition = 8192;

int auto_partition(int64_t batch, int64_t max_context, const pa_cache_desc* cd) {
  int pt = kPartitionRowBytes / static_cast<int>(cd->head_dim * elem_bytes(cd->cache_dtype));
  auto ctas = [&](int64_t p) { return batch * cd->num_kv_heads * ((max_context + p - 1) / p); };
  while (pt > kMinAutoPartition && ctas(pt) < 2 * kNumSMs) pt >>= 1;
  const int64_t rows = batch * cd->num_kv_heads;  // (sequence, KV head) pairs
  if (cd->head_dim == 128 && rows > 0 && rows < kWaveCtas) {
    const int64_t waves = ctas(pt) / kWaveCtas;
    if (waves >= 1 && ctas(pt) % kWaveCtas != 0) {
      for (int64_t w = batch == 1 ? 1 : waves; w <= waves; ++w) {
        const int64_t parts = w * kWaveCtas / rows;  // partitions per row in w whole waves
        const int64_t pt2 = ((max_context + parts - 1) / parts + 15) / 16 * 16;
        if (w < waves && pt2 > kMaxWavePartition) continue;
        if (pt2 <= (int64_t{1} << 20) && ctas(pt2) <= w * kWaveCtas) pt = static_cast<int>(pt2);
        break;
      }
    }
  }
  return pt;
}

struct Plan {
  int partition_tokens;
  int num_partitions;
  size_t ws_o_bytes;     // partial outputs, then (max, sum) pairs
  size_t ws_list_offset;  // work-list counter (256 bytes), then the items
  size_t ws_bytes;
  bool fits;  // false: the workspace would not be addressable (sizes refused)
};

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// The split-K workspace holds head_dim + 2 floats per (row, partition); plans
// whose workspace would pass 2^60 bytes are refused rather than let the size
// wrap around.
bool workspace_fits(int64_t rows, int64_t parts, int64_t head_dim) {
  const int64_t lim = (int64_t{1} << 60) / ((head_dim + 2) * 4);
  return rows <= lim && parts <= lim / std::max<int64_t>(rows, 1);
}

Plan make_plan(int64_t batch, int64_t num_q_heads, int64_t max_context, int partition_tokens,
               const pa_cache_desc* cd, int window = 0) {
  // with a sliding window a sequence spans at most window + 15 tokens from
  // its first (16-aligned) partition start
  if (window > 0) max_context = std::min<int64_t>(max_context, window + 15);
  Plan pl{};
  pl.partition_tokens = partition_tokens > 0
                            ? partition_tokens
                            : auto_partition(batch, max_context, cd);
  const int64_t np = (max_context + pl.partition_tokens - 1) / pl.partition_tokens;
  pl.num_partitions = static_cast<int>(std::max<int64_t>(np, 1));
  pl.fits = workspace_fits(batch * num_q_heads, pl.num_partitions, cd->head_dim);
  if (pl.num_partitions > 1 && pl.fits) {
    pl.ws_o_bytes = round_up(static_cast<size_t>(batch * num_q_heads) * pl.num_partitions *
                                 cd->head_dim * sizeof(float),
                             256);
    pl.ws_list_offset = pl.ws_o_bytes + round_up(static_cast<size_t>(batch * num_q_heads) *
                                                     pl.num_partitions * sizeof(float2),
                                                 256);
    // the work list: a counter section, then one (sequence, partition) item
    // per partition a sequence can have
    pl.ws_bytes = pl.ws_list_offset + 256 +
                  round_up(static_cast<size_t>(batch) * pl.num_partitions * sizeof(int2), 256);
  }
  return pl;
}

// Partials and (plain decode) work list of a split plan in `ws`.
void bind_workspace(pa::DecodeParams& p, const Plan& pl, void* ws) {
  if (!pl.ws_bytes) return;
  char* base = static_cast<char*>(ws);
  p.ws_o = reinterpret_cast<float*>(base);
  p.ws_ml = reinterpret_cast<float2*>(base + pl.ws_o_bytes);
  p.work_count = reinterpret_cast<int*>(base + pl.ws_list_offset);
  p.work_items = reinterpret_cast<int2*>(base + pl.ws_list_offset + 256);
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device),
// raised to the largest size requested so far. Every kernel that comes here
// also prefers the largest shared-memory carveout (228 KB per SM), so that
// CTAs of the shared-prefix and suffix-decode kernels, which run side by
// side, find the same split of each SM and fit next to each other.
cudaError_t ensure_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::unordered_map<const void*, std::array<int, 64>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find(kernel);
  if (it == done.end()) it = done.emplace(kernel, std::array<int, 64>{}).first;
  int& have = it->second[dev & 63];
  if (have >= bytes) return cudaSuccess;
  if (have == 0) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

// Launch `kern` as the programmatic dependent of the kernel before it in
// `st`: it may start once every CTA of that kernel has started (or exited),
// and waits (griddepcontrol.wait) before reading that kernel's results.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Split-K merge, the decode kernel's programmatic dependent: 1, 2, 4, 8, 16
// or 32 warps per (sequence, query head) row by the number of partials per
// row (a row of 16 or 32 warps is a CTA of its own).
template <typename TQ, int D, bool PARTIAL>
pa_status launch_reduce_t(const pa::DecodeParams& p, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(p.batch) * p.num_q_heads;
  const int n = p.num_partitions;
  auto go = [&](auto kern, int warps, int rows_per_cta) {
    const int64_t ctas = (rows + rows_per_cta - 1) / rows_per_cta;
    return launch_dependent(kern, dim3(static_cast<unsigned>(ctas)), dim3(warps * 32), 0, st, p) ==
                   cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
  };
  // one warp per row: 32 rows per CTA, so that a large batch's merge is a few
  // hundred CTAs that all start at once
  if (n <= 8) return go(pa::pa_decode_reduce_kernel<TQ, D, 1, 8, 32, PARTIAL>, 32, 32);
  if (n <= 16) return go(pa::pa_decode_reduce_kernel<TQ, D, 1, 16, 32, PARTIAL>, 32, 32);
  // several warps per row: at most 8 partials a warp up to 128 partials, 16
  // up to 256; beyond, 32 warps take batches of 8 each (1024 threads leave a
  // thread 64 registers)
  if (n <= 32) return go(pa::pa_decode_reduce_kernel<TQ, D, 4, 8, 16, PARTIAL>, 16, 4);
  if (n <= 64) return go(pa::pa_decode_reduce_kernel<TQ, D, 8, 8, 16, PARTIAL>, 16, 2);
  if (n <= 128) return go(pa::pa_decode_reduce_kernel<TQ, D, 16, 8, 16, PARTIAL>, 16, 1);
  if (n <= 256) return go(pa::pa_decode_reduce_kernel<TQ, D, 16, 16, 16, PARTIAL>, 16, 1);
  return go(pa::pa_decode_reduce_kernel<TQ, D, 32, 8, 32, PARTIAL>, 32, 1);
}

// (partial mode writes fp32 pieces instead of `out`: its own instantiations)
template <typename TQ, int D>
pa_status launch_reduce(const pa::DecodeParams& p, cudaStream_t st) {
  return p.cp_o ? launch_reduce_t<TQ, D, true>(p, st) : launch_reduce_t<TQ, D, false>(p, st);
}

// Work-list mode (plain, fused and sliding-window decodes of a batch split
// into partitions): the workspace holds the list, and the units (items x KV
// head groups) stay below 2^31. The plan kernel may lengthen the partitions
// by up to 2^kListGrowLog2 (fewer units and partials when the batch's
// tokens allow; the workspace, sized for the host's length, holds fewer):
// up to 4 times by doubling, up to 8 times to hold every sequence whole.
// The suffix decode of a cascade keeps its grid (its sequences have one
// partition or few, visited longest first).
constexpr int kListGrowLog2 = 3;

bool use_work_list(const pa::DecodeParams& p, bool dependent) {
  return !dependent && p.prefix_blocks == 0 && p.work_items && !p.cp_o && p.batch > 1 &&
         p.num_partitions > 1 &&
         static_cast<int64_t>(p.batch) * p.num_partitions * p.num_kv_heads * p.head_groups <
             (int64_t{1} << 31);
}

// Steal mode (a single sequence's split decode over a 16-bit cache with
// blocks of 16 tokens or more and partitions of kStealMinPartition tokens or
// more, unless the caller asked for reproducible results): the CTAs of each
// KV head group share the sequence's tiles through a counter per group, so
// that CTAs on slower SMs take fewer tiles instead of setting the launch's
// end. Shorter partitions keep their fixed split: the claims' latency would
// cost more than the balance gains. The counters sit in the work list's
// section of the workspace (256 bytes, then 8 per partition; 8 bytes a
// counter), and a counter's claimed-tile field (kStealCountBits wide) must
// hold the tiles plus one overshooting chunk per warp.
constexpr int kStealMinPartition = 1024;
std::atomic<int> g_deterministic{0};
std::atomic<int> g_withhold_steal_counts{0};  // pa_testing_withhold_steal_counts

bool use_steal(const pa::DecodeParams& p, int grid_x, bool dependent) {
  const int64_t hb = static_cast<int64_t>(p.num_kv_heads) * p.head_groups;
  const int64_t list_bytes = 256 + (static_cast<int64_t>(p.num_partitions) * 8 + 255) / 256 * 256;
  const int64_t most_claimed = static_cast<int64_t>(p.max_context) / 16 + 1 +
                               static_cast<int64_t>(p.num_partitions) * kDecodeWarps *
                                   pa::kStealChunk + pa::kStealChunk;
  return g_deterministic.load(std::memory_order_relaxed) == 0 && !dependent && !p.cp_o &&
         p.prefix_blocks == 0 && !p.k_new && p.work_count && p.batch == 1 &&
         p.num_partitions > 1 && p.partition_tokens >= kStealMinPartition &&
         grid_x == p.num_partitions && p.part_offset == 0 &&
         !p.force_partials && p.bs_log2 >= 4 && hb * 8 <= list_bytes &&
         most_claimed < (int64_t{1} << pa::kStealCountBits);
}

// A fresh steal epoch per launch (bit 62 set, the call count above the
// claimed-tile field).
unsigned long long next_steal_epoch() {
  static std::atomic<unsigned long long> calls{0};
  const unsigned long long n = (calls.fetch_add(1, std::memory_order_relaxed) + 1) &
                               ((1ull << (62 - pa::kStealCountBits)) - 1);
  return (1ull << 62) | (n << pa::kStealCountBits);
}

// CTAs of `kern` resident per SM at this block and shared-memory size, and
// the device's SM count (cached per kernel, size and device).
cudaError_t resident_ctas(const void* kern, int threads, int smem, int* per_sm, int* sms) {
  struct Key {
    const void* kern;
    int threads, smem, dev;
    bool operator==(const Key& o) const {
      return kern == o.kern && threads == o.threads && smem == o.smem && dev == o.dev;
    }
  };
  struct KeyHash {
    size_t operator()(const Key& k) const {
      return std::hash<const void*>()(k.kern) ^
             (static_cast<size_t>(k.smem) * 131 + static_cast<size_t>(k.threads) * 7 +
              static_cast<size_t>(k.dev));
    }
  };
  static std::mutex mu;
  static std::unordered_map<Key, std::pair<int, int>, KeyHash> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const Key key{kern, threads, smem, dev};
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it == cache.end()) {
    int n = 0, m = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&m, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    it = cache.emplace(key, std::make_pair(n, m)).first;
  }
  *per_sm = it->second.first;
  *sms = it->second.second;
  return cudaSuccess;
}

// Decode kernel over `grid_x` partition columns (or, in work-list mode, the
// plan kernel and a persistent grid), then the split-K merge when the plan
// has more than one partial per sequence (or always, in cascade mode).
template <typename TQ, int CK, int D, int NH>
pa_status launch_decode_t(const pa::DecodeParams& p_in, int grid_x, cudaStream_t st,
                          bool with_reduce = true, bool dependent = false) {
  using S = pa::DecodeSmem<CK, D, kDecodeWarps, kDecodeStages>;
  auto kern = p_in.k_new
                  ? pa::pa_decode_kernel<TQ, CK, D, kDecodeWarps, kDecodeStages, NH, true>
                  : pa::pa_decode_kernel<TQ, CK, D, kDecodeWarps, kDecodeStages, NH, false>;
  if constexpr (CK == pa::kE4M3 && NH == 1)
    kern = p_in.k_new ? pa::pa_decode_e4m3_kernel<TQ, D, kDecodeWarps, kDecodeStages, true>
                      : pa::pa_decode_e4m3_kernel<TQ, D, kDecodeWarps, kDecodeStages, false>;
  pa::DecodeParams p = p_in;
  const bool list = use_work_list(p, dependent);
  p.steal_ctr = nullptr;
  p.steal_epoch = 0;
  p.steal_merge = 0;
  p.steal_withhold = 0;
  if constexpr (CK != pa::kE4M3) {
    if (!list && use_steal(p, grid_x, dependent)) {
      kern = pa::pa_decode_kernel<TQ, CK, D, kDecodeWarps, kDecodeStages, NH, false, true>;
      p.steal_ctr = reinterpret_cast<unsigned long long*>(p.work_count);
      p.steal_epoch = next_steal_epoch();
    }
  }
  if (list) {
    // the plan kernel may lengthen the partitions up to this
    p.max_partition_tokens = static_cast<int>(
        std::min<int64_t>(int64_t{p.partition_tokens} << kListGrowLog2, int64_t{1} << 20));
  } else {
    p.work_items = nullptr;
    p.work_count = nullptr;
    p.max_partition_tokens = 0;
  }
  const int bt_entries = pa::staged_block_ids(p);
  const int smem = (p.k_new && CK == pa::kE4M3)
                       ? S::new_rows_offset(bt_entries) + S::kNewRowBytes
                       : S::kMainBytes + bt_entries * 4;
  if (smem > 227 * 1024) return PA_ERR_UNSUPPORTED;
  if (ensure_smem(reinterpret_cast<const void*>(kern), smem) != cudaSuccess) return PA_ERR_CUDA;
  if (list) {
    // the plan kernel, then a persistent grid (one CTA per resident slot, at
    // most one per unit) as its programmatic dependent
    int per_sm = 0, sms = 0;
    if (resident_ctas(reinterpret_cast<const void*>(kern), kDecodeWarps * 32, smem, &per_sm,
                      &sms) != cudaSuccess)
      return PA_ERR_CUDA;
    const int64_t hb = static_cast<int64_t>(p.num_kv_heads) * p.head_groups;
    const int64_t units = static_cast<int64_t>(p.batch) * p.num_partitions * hb;
    const int64_t ctas = std::min<int64_t>(std::max(per_sm, 1) * int64_t{sms}, units);
    p.list_slots = static_cast<int>(ctas);
    pa::pa_decode_plan_kernel<<<1, pa::kPlanThreads, 0, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
    if (launch_dependent(kern, dim3(static_cast<unsigned>(ctas)), dim3(kDecodeWarps * 32), smem,
                         st, p) != cudaSuccess)
      return PA_ERR_CUDA;
    return with_reduce ? launch_reduce<TQ, D>(p, st) : PA_OK;
  }
  dim3 grid(grid_x, p.num_kv_heads * p.head_groups, p.batch);
  if (p.steal_ctr) {
    // Steal mode: when the whole grid fits on the GPU at once and the
    // workspace section holds three counters per head group, the rows merge
    // their own partials in the launch (a cooperative launch, so that the
    // CTAs a row's merge waits for are resident) and no merge kernel follows
    int per_sm = 0, sms = 0;
    if (resident_ctas(reinterpret_cast<const void*>(kern), kDecodeWarps * 32, smem, &per_sm,
                      &sms) != cudaSuccess)
      return PA_ERR_CUDA;
    const int64_t hb = static_cast<int64_t>(p.num_kv_heads) * p.head_groups;
    const int64_t list_bytes =
        256 + (static_cast<int64_t>(p.num_partitions) * 8 + 255) / 256 * 256;
    const int64_t ctas = static_cast<int64_t>(grid_x) * hb * p.batch;
    if (ctas <= static_cast<int64_t>(per_sm) * sms && 3 * hb * p.batch * 8 <= list_bytes) {
      pa::DecodeParams pm = p;
      pm.steal_merge = 1;
      pm.steal_withhold = g_withhold_steal_counts.load(std::memory_order_relaxed);
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = grid;
      cfg.blockDim = dim3(kDecodeWarps * 32);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeCooperative;
      attr[0].val.cooperative = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      return cudaLaunchKernelEx(&cfg, kern, pm) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
    }
  }
  if (dependent) {
    if (launch_dependent(kern, grid, dim3(kDecodeWarps * 32), smem, st, p) != cudaSuccess)
      return PA_ERR_CUDA;
  } else {
    kern<<<grid, kDecodeWarps * 32, smem, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  if (with_reduce && (p.num_partitions > 1 || p.force_partials)) {
    const pa_status rs = launch_reduce<TQ, D>(p, st);
    if (rs != PA_OK) return rs;
  }
  return PA_OK;
}

template <typename TQ, int CK>
pa_status launch_decode_d(const pa::DecodeParams& p, int head_dim, int grid_x,
                          cudaStream_t st, bool with_reduce = true, bool dependent = false) {
  // query heads per CTA: the whole group up to 16; 8-head column blocks
  const bool two = std::min(p.group, 16) > 8;
  if (head_dim == 64)
    return two ? launch_decode_t<TQ, CK, 64, 2>(p, grid_x, st, with_reduce, dependent)
               : launch_decode_t<TQ, CK, 64, 1>(p, grid_x, st, with_reduce, dependent);
  return two ? launch_decode_t<TQ, CK, 128, 2>(p, grid_x, st, with_reduce, dependent)
             : launch_decode_t<TQ, CK, 128, 1>(p, grid_x, st, with_reduce, dependent);
}

pa_status launch_decode(const pa::DecodeParams& p, int q_dtype, const pa_cache_desc* cache,
                        cudaStream_t s, int grid_x = -1) {
  if (grid_x < 0) grid_x = p.num_partitions;
  switch (cache->cache_dtype) {
    case PA_F16: return launch_decode_d<__half, pa::kF16>(p, cache->head_dim, grid_x, s);
    case PA_BF16: return launch_decode_d<__nv_bfloat16, pa::kBF16>(p, cache->head_dim, grid_x, s);
    default:
      return q_dtype == PA_F16
                 ? launch_decode_d<__half, pa::kE4M3>(p, cache->head_dim, grid_x, s)
                 : launch_decode_d<__nv_bfloat16, pa::kE4M3>(p, cache->head_dim, grid_x, s);
  }
}

// Host-side checks shared by the decode entry points. *nothing is set when
// the call is valid but has no work (batch == 0).
pa_status check_decode_args(const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads,
                            const void* k_cache, const void* v_cache, const pa_cache_desc* cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* context_lens, int32_t max_context, float scale,
                            void* out, int32_t partition_tokens, int* bs_log2, bool* nothing) {
  *nothing = false;
  pa_status st = check_cache(cache, bs_log2);
  if (st != PA_OK) return st;
  if (batch < 0 || num_q_heads <= 0 || max_context < 0 || max_blocks_per_seq <= 0)
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (q_dtype != PA_F16 && q_dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (cache->cache_dtype != PA_E4M3 && cache->cache_dtype != q_dtype) return PA_ERR_UNSUPPORTED;
  if (partition_tokens != 0 &&
      (partition_tokens < 16 || partition_tokens > (1 << 20) || partition_tokens % 16 != 0))
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (batch == 0) {
    *nothing = true;
    return PA_OK;
  }
  if (batch > 65535) return PA_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return PA_ERR_INVALID_ARG;
  if (cache->cache_dtype == PA_E4M3 && (!cache->k_scale || !cache->v_scale ||
                                         !aligned16(cache->k_scale) || !aligned16(cache->v_scale)))
    return PA_ERR_INVALID_ARG;
  const int group = num_q_heads / cache->num_kv_heads;
  if (static_cast<int64_t>(cache->num_kv_heads) * ((group + 15) / 16) > 65535)
    return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

pa::DecodeParams decode_params(const void* q, int32_t batch, int32_t num_q_heads,
                               const void* k_cache, const void* v_cache,
                               const pa_cache_desc* cache, const int32_t* block_tables,
                               int32_t max_blocks_per_seq, const int32_t* context_lens,
                               int32_t max_context, float scale, void* out, int bs_log2) {
  pa::DecodeParams p{};
  p.q = q;
  p.out = out;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.k_scale = cache->k_scale;
  p.v_scale = cache->v_scale;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.num_blocks = cache->num_blocks;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = cache->num_kv_heads;
  p.group = num_q_heads / cache->num_kv_heads;
  p.head_groups = (p.group + 15) / 16;
  p.bs_log2 = bs_log2;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_context = max_context;
  p.scale_log2 = scale * 1.4426950408889634f;
  return p;
}

// ---- shared-prefix (cascade) decode -----------------------------------------
constexpr int kPrefixWarps = 4;   // 16 query columns per warp
constexpr int kPrefixStages = 2;  // CTA-wide cp.async stages of one 32/64-token block
#ifndef PA_PREFIX_CHUNK_MAX
#define PA_PREFIX_CHUNK_MAX 512
#endif
constexpr int kPrefixChunkMax = PA_PREFIX_CHUNK_MAX;  // a multiple of 64

struct CascadePlan {
  int prefix_len;
  int chunk_tokens;
  int num_chunks;
  int suffix_partition_tokens;
  int suffix_partitions;
  int num_partitions;  // chunks + suffix partitions
  size_t ws_o_bytes;
  size_t ws_bytes;
  bool longest_first;  // the suffix decode visits the sequences longest first
  bool fits;           // as Plan::fits
};

// 16-bit caches with blocks of >= 8 tokens (whole 1024-byte swizzle atoms
// per TMA box) and groups of <= 128 query heads run the prefix on the
// tcgen05 kernel (pa_prefix_umma.cuh); the rest on the mma.sync prefix CTAs
// of pa_cascade_kernel.
bool cascade_uses_umma(const pa_cache_desc* cd, int64_t group) {
  return cd->cache_dtype != PA_E4M3 && cd->block_size >= 8 && group <= pa::kUmmaRows &&
         cd->num_blocks * cd->block_size < (int64_t{1} << 31);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the CUDA driver library).
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// A tiled map with 128-byte swizzle, zeros out of range (loads) and
// clipping (stores). Strides in bytes for dimensions 1 .. rank-1.
template <int R>
bool make_map(CUtensorMap* m, CUtensorMapDataType type, const void* base,
              const uint64_t (&dims)[R], const uint64_t (&strides)[R - 1],
              const uint32_t (&box)[R]) {
  const EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint64_t d[R], st[R - 1];
  cuuint32_t b[R], es[R];
  for (int i = 0; i < R; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i < R - 1) st[i] = strides[i];
  }
  return fn(m, type, R, const_cast<void*>(base), d, st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool make_map_3d(CUtensorMap* m, bool bf16, const void* base, const uint64_t (&dims)[3],
                 const uint64_t (&strides)[2], const uint32_t (&box)[3]) {
  return make_map<3>(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                     base, dims, strides, box);
}

constexpr int kUmmaMaxChunks = 64;
// Row tiles of 128 query rows per prefix CTA, and K / V stages.
#ifndef PA_UMMA_TILES
#define PA_UMMA_TILES 2
#endif
#ifndef PA_UMMA_STAGES
#define PA_UMMA_STAGES 2
#endif
constexpr int kUmmaTiles = PA_UMMA_TILES;
constexpr int kUmmaStages = PA_UMMA_STAGES;
#ifndef PA_UMMA_TARGET_CTAS
#define PA_UMMA_TARGET_CTAS (148 * (kUmmaTiles == 1 ? 2 : 1))
#endif
constexpr int kUmmaTargetCtas = PA_UMMA_TARGET_CTAS;  // prefix CTAs the chunk plan aims at

CascadePlan make_cascade_plan(int64_t batch, int64_t num_q_heads, int64_t max_context,
                              int prefix_blocks, int partition_tokens, const pa_cache_desc* cd) {
  CascadePlan pl{};
  pl.prefix_len = prefix_blocks * cd->block_size;
  const int64_t group = num_q_heads / cd->num_kv_heads;
  if (cascade_uses_umma(cd, group)) {
    // row blocks (kUmmaTiles x 128 / group sequences each) x KV heads x
    // chunks of 64-token steps, about kUmmaTargetCtas CTAs (the kernel's
    // occupancy on 148 SMs)
    const int64_t seqs = kUmmaTiles * (pa::kUmmaRows / group);  // sequences per CTA
    const int64_t tiles = (batch + seqs - 1) / seqs * cd->num_kv_heads;
    const int64_t steps = (pl.prefix_len + pa::kUmmaTokens - 1) / pa::kUmmaTokens;
    const int64_t want = std::max<int64_t>(1, kUmmaTargetCtas / tiles);
    const int64_t chunks = std::min<int64_t>(std::min<int64_t>(want, steps), kUmmaMaxChunks);
    pl.chunk_tokens = static_cast<int>((steps + chunks - 1) / chunks) * pa::kUmmaTokens;
  } else {
    // prefix tokens per prefix CTA: the whole prefix up to kPrefixChunkMax
    pl.chunk_tokens = std::min((pl.prefix_len + 15) / 16 * 16, kPrefixChunkMax);
  }
  pl.num_chunks = (pl.prefix_len + pl.chunk_tokens - 1) / pl.chunk_tokens;
  const int64_t suffix_max = std::max<int64_t>(max_context - pl.prefix_len, 0);
  pl.suffix_partition_tokens =
      partition_tokens > 0 ? partition_tokens : auto_partition(batch, suffix_max, cd);
  if (partition_tokens == 0 && cascade_uses_umma(cd, group)) {
    // every row already merges the prefix partials: take up to four times
    // the plain decode's partition while that still leaves two CTAs per SM
    for (int i = 0; i < 2; ++i) {
      const int64_t pt2 = 2 * static_cast<int64_t>(pl.suffix_partition_tokens);
      if (batch * cd->num_kv_heads * ((suffix_max + pt2 - 1) / pt2) < 2 * kNumSMs) break;
      pl.suffix_partition_tokens = static_cast<int>(pt2);
    }
  }
  pl.suffix_partitions =
      static_cast<int>((suffix_max + pl.suffix_partition_tokens - 1) / pl.suffix_partition_tokens);
  pl.num_partitions = pl.num_chunks + pl.suffix_partitions;
  pl.fits = workspace_fits(batch * num_q_heads, pl.num_partitions, cd->head_dim);
  if (!pl.fits) return pl;
  pl.ws_o_bytes = round_up(static_cast<size_t>(batch * num_q_heads) * pl.num_partitions *
                               cd->head_dim * sizeof(float),
                           256);
  pl.ws_bytes = pl.ws_o_bytes + round_up(static_cast<size_t>(batch * num_q_heads) *
                                             pl.num_partitions * sizeof(float2),
                                         256);
  // the tensor-core path's suffix decode takes long partitions (up to four
  // times the plain rule), so it visits the sequences longest first
  pl.longest_first = cascade_uses_umma(cd, group) && batch > 1 && batch <= pa::kOrderMaxBatch;
  return pl;
}

// Prefix CTAs and suffix CTAs in one launch (so they overlap), then the merge.
template <typename TQ, int CK, int D, int NH>
pa_status launch_cascade_t(const pa::DecodeParams& p, const CascadePlan& pl, cudaStream_t st) {
  using SD = pa::DecodeSmem<CK, D, kDecodeWarps, kDecodeStages>;
  using SP = pa::PrefixSmem<CK, D, kPrefixStages, pa::prefix_subtiles<CK>()>;
  auto kern = pa::pa_cascade_kernel<TQ, CK, D, kDecodeWarps, kDecodeStages, NH, kPrefixWarps,
                                    kPrefixStages>;
  const int bt_d = std::min((p.partition_tokens >> p.bs_log2) + 2, pa::kBlockIdsInSmem);
  const int bt_p = std::min((p.prefix_chunk_tokens >> p.bs_log2) + 2, pa::kBlockIdsInSmem);
  const int smem = std::max(SD::kMainBytes + bt_d * 4, SP::kPipeBytes + bt_p * 4);
  if (smem > 227 * 1024) return PA_ERR_UNSUPPORTED;
  if (ensure_smem(reinterpret_cast<const void*>(kern), smem) != cudaSuccess) return PA_ERR_CUDA;
  pa::CascadeGrid cg{};
  cg.n_chunks = pl.num_chunks;
  const int64_t rows = static_cast<int64_t>(p.batch) * p.group;
  cg.n_rowblocks = static_cast<int>((rows + 16 * kPrefixWarps - 1) / (16 * kPrefixWarps));
  const int64_t n_prefix = static_cast<int64_t>(cg.n_chunks) * cg.n_rowblocks * p.num_kv_heads;
  cg.n_suffix_parts = std::max(pl.suffix_partitions, 1);
  const int64_t n_suffix =
      static_cast<int64_t>(cg.n_suffix_parts) * p.num_kv_heads * p.head_groups * p.batch;
  const int64_t total = n_prefix + n_suffix;
  if (total > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  cg.n_prefix = static_cast<int>(n_prefix);
  cg.n_suffix = static_cast<int>(n_suffix);
  cg.ratio = static_cast<int>(n_suffix / std::max<int64_t>(n_prefix, 1));
  kern<<<static_cast<unsigned>(total), kDecodeWarps * 32, smem, st>>>(p, cg);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  return launch_reduce<TQ, D>(p, st);
}

std::mutex g_hook_mu;
int g_withhold_prefix_scores = 0;  // pa_testing_withhold_prefix_scores

// 16-bit caches: the tcgen05 prefix kernel, then the suffix decode (cascade
// mode) as its programmatic dependent, so that the two run side by side
// (every prefix CTA lets it start at once; the suffix grid finishes only
// after the prefix grid), then the merge as the suffix decode's dependent.
template <typename TQ, int CK, int D>
pa_status launch_cascade_umma_t(const pa::DecodeParams& p, const CascadePlan& pl,
                                cudaStream_t st) {
  using C = pa::UmmaCfg<D, kUmmaTiles, kUmmaStages>;
  constexpr bool kBF16 = std::is_same<TQ, __nv_bfloat16>::value;
  auto kern = pa::pa_prefix_umma_kernel<TQ, D, kUmmaTiles, kUmmaStages>;
  if (ensure_smem(reinterpret_cast<const void*>(kern), C::kRequest) != cudaSuccess)
    return PA_ERR_CUDA;
  pa::UmmaGrid ug{};
  ug.n_chunks = pl.num_chunks;
  ug.seqs_per_tile = pa::kUmmaRows / p.group;
  const int seqs_per_cta = kUmmaTiles * ug.seqs_per_tile;
  ug.n_rowtiles = (p.batch + seqs_per_cta - 1) / seqs_per_cta;
  const int bs = 1 << p.bs_log2;
  ug.unit_tokens = std::min(bs, pa::kUmmaTokens);
  ug.num_slots = static_cast<int>(p.num_blocks * bs);
  // q [batch][Hq][D]: box of 64 channels x the group's heads x the tile's
  // sequences; caches [slot][Hkv][D]: box of 64 channels x 1 head x a unit
  CUtensorMap tq, tk, tv;
  const uint64_t row = static_cast<uint64_t>(D) * 2;
  if (!make_map_3d(&tq, kBF16, p.q,
                   {static_cast<uint64_t>(D), static_cast<uint64_t>(p.num_q_heads),
                    static_cast<uint64_t>(p.batch)},
                   {row, row * p.num_q_heads},
                   {64u, static_cast<uint32_t>(p.group), static_cast<uint32_t>(ug.seqs_per_tile)}) ||
      !make_map_3d(&tk, kBF16, p.k_cache,
                   {static_cast<uint64_t>(D), static_cast<uint64_t>(p.num_kv_heads),
                    static_cast<uint64_t>(ug.num_slots)},
                   {row, row * p.num_kv_heads}, {64u, 1u, static_cast<uint32_t>(ug.unit_tokens)}) ||
      !make_map_3d(&tv, kBF16, p.v_cache,
                   {static_cast<uint64_t>(D), static_cast<uint64_t>(p.num_kv_heads),
                    static_cast<uint64_t>(ug.num_slots)},
                   {row, row * p.num_kv_heads}, {64u, 1u, static_cast<uint32_t>(ug.unit_tokens)}))
    return PA_ERR_CUDA;
  // partial outputs ws_o [batch][Hq][partition][D] f32: box of 32 channels x
  // 1 partition x the group's heads x the tile's sequences
  CUtensorMap to;
  const uint64_t prow = static_cast<uint64_t>(D) * 4;
  const uint64_t np = static_cast<uint64_t>(p.num_partitions);
  if (!make_map<4>(&to, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.ws_o,
                   {static_cast<uint64_t>(D), np, static_cast<uint64_t>(p.num_q_heads),
                    static_cast<uint64_t>(p.batch)},
                   {prow, prow * np, prow * np * p.num_q_heads},
                   {32u, 1u, static_cast<uint32_t>(p.group),
                    static_cast<uint32_t>(ug.seqs_per_tile)}))
    return PA_ERR_CUDA;
  const int64_t ctas = static_cast<int64_t>(ug.n_chunks) * ug.n_rowtiles * p.num_kv_heads;
  if (ctas > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  {
    std::lock_guard<std::mutex> lock(g_hook_mu);
    ug.withhold_scores = g_withhold_prefix_scores;
  }
  kern<<<static_cast<unsigned>(ctas), C::kThreads, C::kRequest, st>>>(p, ug, tq, tk, tv, to);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  pa::DecodeParams ps = p;  // the suffix decode, longest sequences first
  ps.longest_first = pl.longest_first ? 1 : 0;
  const pa_status rs = launch_decode_d<TQ, CK>(ps, D, std::max(pl.suffix_partitions, 1), st,
                                               /*with_reduce=*/false, /*dependent=*/true);
  if (rs != PA_OK) return rs;
  return launch_reduce<TQ, D>(p, st);
}

template <typename TQ, int CK>
pa_status launch_cascade_d(const pa::DecodeParams& p, const CascadePlan& pl,
                           const pa_cache_desc* cd, cudaStream_t st) {
  const int head_dim = cd->head_dim;
  if constexpr (CK != pa::kE4M3) {
    if (cascade_uses_umma(cd, p.group))
      return head_dim == 64 ? launch_cascade_umma_t<TQ, CK, 64>(p, pl, st)
                            : launch_cascade_umma_t<TQ, CK, 128>(p, pl, st);
  }
  {
    const bool two = std::min(p.group, 16) > 8;
    if (head_dim == 64)
      return two ? launch_cascade_t<TQ, CK, 64, 2>(p, pl, st)
                 : launch_cascade_t<TQ, CK, 64, 1>(p, pl, st);
    return two ? launch_cascade_t<TQ, CK, 128, 2>(p, pl, st)
               : launch_cascade_t<TQ, CK, 128, 1>(p, pl, st);
  }
}

}  // namespace

extern "C" {

const char* pa_status_string(int32_t s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported dtype or shape";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_DEVICE_BOUNDS: return "a kernel saw an out-of-range slot, block id or length";
    default: return "unknown status";
  }
}

int32_t pa_version(void) { return 100; }

pa_status pa_decode_partial(const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads,
                            const void* k_cache, const void* v_cache, const pa_cache_desc* cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* context_lens, int32_t max_context, float scale,
                            float* part_o, float* part_ml, int32_t partition_tokens,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!part_o || !part_ml || !aligned16(part_ml)) return PA_ERR_INVALID_ARG;
  int bs_log2 = 0;
  bool nothing = false;
  // (part_o stands in for `out` in the shared checks: same rows, never read)
  pa_status st = check_decode_args(q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache,
                                   block_tables, max_blocks_per_seq, context_lens, max_context,
                                   scale, part_o, partition_tokens, &bs_log2, &nothing);
  if (st != PA_OK || nothing) return st;
  const Plan pl = make_plan(batch, num_q_heads, max_context, partition_tokens, cache);
  if (!pl.fits) return PA_ERR_UNSUPPORTED;
  if (pl.ws_bytes > 0) {
    if (!workspace || workspace_bytes < pl.ws_bytes) return PA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PA_ERR_WORKSPACE;
  }
  pa::DecodeParams p = decode_params(q, batch, num_q_heads, k_cache, v_cache, cache,
                                     block_tables, max_blocks_per_seq, context_lens, max_context,
                                     scale, part_o, bs_log2);
  bind_workspace(p, pl, workspace);
  p.partition_tokens = pl.partition_tokens;
  p.num_partitions = pl.num_partitions;
  p.cp_o = part_o;
  p.cp_ml = reinterpret_cast<float2*>(part_ml);
  return launch_decode(p, q_dtype, cache, as_stream(stream));
}

pa_status pa_merge_partials(const float* part_o, const float* part_ml, int32_t num_parts,
                            int64_t rows, int32_t head_dim, void* out, int32_t out_dtype,
                            void* stream) {
  if (num_parts < 1 || rows < 0 || (head_dim != 64 && head_dim != 128)) return PA_ERR_INVALID_ARG;
  if (out_dtype != PA_F16 && out_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (rows == 0) return PA_OK;
  if (!part_o || !part_ml || !out || !aligned16(part_o) || !aligned16(part_ml) ||
      !aligned16(out))
    return PA_ERR_INVALID_ARG;
  if (rows > (int64_t{1} << 40) / num_parts) return PA_ERR_UNSUPPORTED;
  const int64_t ctas = (rows + 7) / 8;
  if (ctas > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  const cudaStream_t st = as_stream(stream);
  const float2* ml = reinterpret_cast<const float2*>(part_ml);
  const dim3 grid(static_cast<unsigned>(ctas));
  if (out_dtype == PA_F16) {
    if (head_dim == 64)
      pa::pa_merge_partials_kernel<__half, 64><<<grid, 256, 0, st>>>(part_o, ml, num_parts, rows,
                                                                   static_cast<__half*>(out));
    else
      pa::pa_merge_partials_kernel<__half, 128><<<grid, 256, 0, st>>>(
          part_o, ml, num_parts, rows, static_cast<__half*>(out));
  } else {
    if (head_dim == 64)
      pa::pa_merge_partials_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(
          part_o, ml, num_parts, rows, static_cast<__nv_bfloat16*>(out));
    else
      pa::pa_merge_partials_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(
          part_o, ml, num_parts, rows, static_cast<__nv_bfloat16*>(out));
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

void pa_testing_withhold_steal_counts(int32_t on) {
  g_withhold_steal_counts.store(on != 0 ? 1 : 0, std::memory_order_relaxed);
}

int32_t pa_set_deterministic(int32_t on) {
  return g_deterministic.exchange(on != 0 ? 1 : 0);
}

void pa_testing_withhold_prefix_scores(int32_t on) {
  std::lock_guard<std::mutex> lock(g_hook_mu);
  g_withhold_prefix_scores = on != 0;
}

pa_status pa_append_kv(const void* k, const void* v, int32_t in_dtype, int64_t num_tokens,
                       const int64_t* slot_mapping, void* k_cache, void* v_cache,
                       const pa_cache_desc* cache, void* stream) {
  int bs_log2 = 0;
  pa_status st = check_cache(cache, &bs_log2);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (in_dtype != PA_F16 && in_dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (cache->cache_dtype != PA_E4M3 && cache->cache_dtype != in_dtype) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  if (num_tokens > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  pa::AppendParams p{};
  p.k = k;
  p.v = v;
  p.slots = slot_mapping;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.num_slots = cache->num_blocks * cache->block_size;
  p.row_elems = cache->num_kv_heads * cache->head_dim;
  const cudaStream_t s = as_stream(stream);
  const dim3 grid(static_cast<unsigned>(num_tokens));
  if (cache->cache_dtype == PA_E4M3) {
    if (!cache->k_inv_scale || !cache->v_inv_scale) return PA_ERR_INVALID_ARG;
    if (!aligned16(cache->k_inv_scale) || !aligned16(cache->v_inv_scale))
      return PA_ERR_INVALID_ARG;
    p.k_inv_scale = cache->k_inv_scale;
    p.v_inv_scale = cache->v_inv_scale;
    if (in_dtype == PA_F16)
      pa::pa_append_kernel<1><<<grid, 128, 0, s>>>(p);
    else
      pa::pa_append_kernel<2><<<grid, 128, 0, s>>>(p);
  } else {
    pa::pa_append_kernel<0><<<grid, 128, 0, s>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t max_context,
                                int32_t partition_tokens, const pa_cache_desc* cache) {
  int bs_log2 = 0;
  if (check_cache(cache, &bs_log2) != PA_OK || batch <= 0 || num_q_heads <= 0 ||
      max_context < 0 || partition_tokens < 0)
    return 0;
  return make_plan(batch, num_q_heads, max_context, partition_tokens, cache).ws_bytes;
}

int32_t pa_decode_partition_tokens(int32_t batch, int32_t max_context,
                                   const pa_cache_desc* cache) {
  int bs_log2 = 0;
  if (check_cache(cache, &bs_log2) != PA_OK || batch <= 0 || max_context < 0) return 0;
  return auto_partition(batch, max_context, cache);
}

pa_status pa_decode(const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads,
                    const void* k_cache, const void* v_cache, const pa_cache_desc* cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t max_context, float scale, void* out,
                    int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                    void* stream) {
  int bs_log2 = 0;
  bool nothing = false;
  pa_status st = check_decode_args(q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache,
                                   block_tables, max_blocks_per_seq, context_lens, max_context,
                                   scale, out, partition_tokens, &bs_log2, &nothing);
  if (st != PA_OK || nothing) return st;
  const Plan pl = make_plan(batch, num_q_heads, max_context, partition_tokens, cache);
  if (!pl.fits) return PA_ERR_UNSUPPORTED;
  if (pl.ws_bytes > 0) {
    if (!workspace || workspace_bytes < pl.ws_bytes) return PA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PA_ERR_WORKSPACE;
  }
  pa::DecodeParams p = decode_params(q, batch, num_q_heads, k_cache, v_cache, cache,
                                     block_tables, max_blocks_per_seq, context_lens, max_context,
                                     scale, out, bs_log2);
  bind_workspace(p, pl, workspace);
  p.partition_tokens = pl.partition_tokens;
  p.num_partitions = pl.num_partitions;
  return launch_decode(p, q_dtype, cache, as_stream(stream));
}

pa_status pa_append_decode(const void* q, const void* k, const void* v, int32_t dtype,
                           int32_t batch, int32_t num_q_heads, const int64_t* slot_mapping,
                           void* k_cache, void* v_cache, const pa_cache_desc* cache,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, int32_t max_context, float scale,
                           void* out, int32_t partition_tokens, void* workspace,
                           size_t workspace_bytes, void* stream) {
  int bs_log2 = 0;
  bool nothing = false;
  pa_status st = check_decode_args(q, dtype, batch, num_q_heads, k_cache, v_cache, cache,
                                   block_tables, max_blocks_per_seq, context_lens, max_context,
                                   scale, out, partition_tokens, &bs_log2, &nothing);
  if (st != PA_OK || nothing) return st;
  if (!k || !v || !slot_mapping || !aligned16(k) || !aligned16(v)) return PA_ERR_INVALID_ARG;
  if (cache->cache_dtype == PA_E4M3 &&
      (!cache->k_inv_scale || !cache->v_inv_scale || !aligned16(cache->k_inv_scale) ||
       !aligned16(cache->v_inv_scale)))
    return PA_ERR_INVALID_ARG;
  const Plan pl = make_plan(batch, num_q_heads, max_context, partition_tokens, cache);
  if (!pl.fits) return PA_ERR_UNSUPPORTED;
  if (pl.ws_bytes > 0) {
    if (!workspace || workspace_bytes < pl.ws_bytes) return PA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PA_ERR_WORKSPACE;
  }
  pa::DecodeParams p = decode_params(q, batch, num_q_heads, k_cache, v_cache, cache,
                                     block_tables, max_blocks_per_seq, context_lens, max_context,
                                     scale, out, bs_log2);
  bind_workspace(p, pl, workspace);
  p.partition_tokens = pl.partition_tokens;
  p.num_partitions = pl.num_partitions;
  p.k_new = k;
  p.v_new = v;
  p.slot_mapping = slot_mapping;
  p.k_inv_scale = cache->k_inv_scale;
  p.v_inv_scale = cache->v_inv_scale;
  return launch_decode(p, dtype, cache, as_stream(stream));
}

size_t pa_decode_sliding_window_workspace_size(int32_t batch, int32_t num_q_heads,
                                               int32_t max_context, int32_t window,
                                               int32_t partition_tokens,
                                               const pa_cache_desc* cache) {
  int bs_log2 = 0;
  if (check_cache(cache, &bs_log2) != PA_OK || batch <= 0 || num_q_heads <= 0 ||
      max_context < 0 || partition_tokens < 0 || window <= 0)
    return 0;
  return make_plan(batch, num_q_heads, max_context, partition_tokens, cache, window).ws_bytes;
}

pa_status pa_decode_sliding_window(const void* q, int32_t q_dtype, int32_t batch,
                                   int32_t num_q_heads, const void* k_cache, const void* v_cache,
                                   const pa_cache_desc* cache, const int32_t* block_tables,
                                   int32_t max_blocks_per_seq, const int32_t* context_lens,
                                   int32_t max_context, int32_t window, float scale, void* out,
                                   int32_t partition_tokens, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  int bs_log2 = 0;
  bool nothing = false;
  pa_status st = check_decode_args(q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache,
                                   block_tables, max_blocks_per_seq, context_lens, max_context,
                                   scale, out, partition_tokens, &bs_log2, &nothing);
  if (st != PA_OK) return st;
  if (window <= 0) return PA_ERR_INVALID_ARG;
  if (nothing) return PA_OK;
  const Plan pl = make_plan(batch, num_q_heads, max_context, partition_tokens, cache, window);
  if (!pl.fits) return PA_ERR_UNSUPPORTED;
  if (pl.ws_bytes > 0) {
    if (!workspace || workspace_bytes < pl.ws_bytes) return PA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PA_ERR_WORKSPACE;
  }
  pa::DecodeParams p = decode_params(q, batch, num_q_heads, k_cache, v_cache, cache,
                                     block_tables, max_blocks_per_seq, context_lens, max_context,
                                     scale, out, bs_log2);
  bind_workspace(p, pl, workspace);
  p.partition_tokens = pl.partition_tokens;
  p.num_partitions = pl.num_partitions;
  p.window = window;
  return launch_decode(p, q_dtype, cache, as_stream(stream));
}

int32_t pa_decode_shared_prefix_partition_tokens(int32_t batch, int32_t num_q_heads,
                                                 int32_t max_context, int32_t prefix_blocks,
                                                 const pa_cache_desc* cache) {
  int bs_log2 = 0;
  if (check_cache(cache, &bs_log2) != PA_OK || batch <= 0 || num_q_heads <= 0 ||
      max_context < 0 || prefix_blocks < 0 || num_q_heads % cache->num_kv_heads != 0)
    return 0;
  if (prefix_blocks == 0) return auto_partition(batch, max_context, cache);
  return make_cascade_plan(batch, num_q_heads, max_context, prefix_blocks, 0, cache)
      .suffix_partition_tokens;
}

size_t pa_decode_shared_prefix_workspace_size(int32_t batch, int32_t num_q_heads,
                                              int32_t max_context, int32_t prefix_blocks,
                                              int32_t partition_tokens,
                                              const pa_cache_desc* cache) {
  int bs_log2 = 0;
  if (check_cache(cache, &bs_log2) != PA_OK || batch <= 0 || num_q_heads <= 0 ||
      max_context < 0 || partition_tokens < 0 || prefix_blocks < 0)
    return 0;
  if (prefix_blocks == 0)
    return make_plan(batch, num_q_heads, max_context, partition_tokens, cache).ws_bytes;
  return make_cascade_plan(batch, num_q_heads, max_context, prefix_blocks, partition_tokens,
                           cache)
      .ws_bytes;
}

pa_status pa_decode_shared_prefix(const void* q, int32_t q_dtype, int32_t batch,
                                  int32_t num_q_heads, const void* k_cache, const void* v_cache,
                                  const pa_cache_desc* cache, const int32_t* block_tables,
                                  int32_t max_blocks_per_seq, const int32_t* context_lens,
                                  int32_t max_context, int32_t prefix_blocks, float scale,
                                  void* out, int32_t partition_tokens, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  int bs_log2 = 0;
  bool nothing = false;
  pa_status st = check_decode_args(q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache,
                                   block_tables, max_blocks_per_seq, context_lens, max_context,
                                   scale, out, partition_tokens, &bs_log2, &nothing);
  if (st != PA_OK) return st;
  if (prefix_blocks < 0 || prefix_blocks > max_blocks_per_seq ||
      static_cast<int64_t>(prefix_blocks) * cache->block_size > max_context)
    return PA_ERR_INVALID_ARG;
  if (nothing) return PA_OK;
  if (prefix_blocks == 0)
    return pa_decode(q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache, block_tables,
                     max_blocks_per_seq, context_lens, max_context, scale, out, partition_tokens,
                     workspace, workspace_bytes, stream);
  const CascadePlan pl = make_cascade_plan(batch, num_q_heads, max_context, prefix_blocks,
                                           partition_tokens, cache);
  if (!pl.fits) return PA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < pl.ws_bytes) return PA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PA_ERR_WORKSPACE;

  pa::DecodeParams p = decode_params(q, batch, num_q_heads, k_cache, v_cache, cache,
                                     block_tables, max_blocks_per_seq, context_lens, max_context,
                                     scale, out, bs_log2);
  p.ws_o = reinterpret_cast<float*>(workspace);
  p.ws_ml = reinterpret_cast<float2*>(reinterpret_cast<char*>(workspace) + pl.ws_o_bytes);
  p.partition_tokens = pl.suffix_partition_tokens;
  p.num_partitions = pl.num_partitions;
  p.prefix_blocks = prefix_blocks;
  p.token_start = pl.prefix_len;
  p.part_offset = pl.num_chunks;
  p.force_partials = 1;
  p.prefix_chunk_tokens = pl.chunk_tokens;

  // One launch: the shared prefix once per block of query rows, and every
  // sequence's own suffix (at least one partition column, so that each
  // sequence's table is checked against the shared prefix); then the merge.
  const cudaStream_t s = as_stream(stream);
  switch (cache->cache_dtype) {
    case PA_F16: return launch_cascade_d<__half, pa::kF16>(p, pl, cache, s);
    case PA_BF16: return launch_cascade_d<__nv_bfloat16, pa::kBF16>(p, pl, cache, s);
    default:
      return q_dtype == PA_F16 ? launch_cascade_d<__half, pa::kE4M3>(p, pl, cache, s)
                               : launch_cascade_d<__nv_bfloat16, pa::kE4M3>(p, pl, cache, s);
  }
}

pa_status pa_copy_blocks_layers(const int32_t* pairs_host, int32_t num_pairs,
                                void* const* k_caches, void* const* v_caches, int32_t num_layers,
                                const pa_cache_desc* cache, void* stream) {
  int bs_log2 = 0;
  pa_status st = check_cache(cache, &bs_log2);
  if (st != PA_OK) return st;
  if (num_pairs < 0 || num_layers < 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0 || num_layers == 0) return PA_OK;
  if (!pairs_host || !k_caches || !v_caches) return PA_ERR_INVALID_ARG;
  for (int32_t l = 0; l < num_layers; ++l)
    if (!k_caches[l] || !v_caches[l] || !aligned16(k_caches[l]) || !aligned16(v_caches[l]))
      return PA_ERR_INVALID_ARG;
  std::unordered_set<int32_t> srcs, dsts;
  for (int32_t i = 0; i < num_pairs; ++i) {
    const int32_t s = pairs_host[2 * i], d = pairs_host[2 * i + 1];
    if (s < 0 || d < 0 || s >= cache->num_blocks || d >= cache->num_blocks)
      return PA_ERR_INVALID_ARG;
    if (!dsts.insert(d).second) return PA_ERR_INVALID_ARG;
    srcs.insert(s);
  }
  for (int32_t d : dsts)
    if (srcs.count(d)) return PA_ERR_INVALID_ARG;

  const int64_t block_bytes = static_cast<int64_t>(cache->block_size) * cache->num_kv_heads *
                              cache->head_dim * elem_bytes(cache->cache_dtype);
  pa::CopyParams p{};
  p.block_vec16 = block_bytes / 16;
  const int64_t slices = std::min<int64_t>(std::max<int64_t>(p.block_vec16 / (256 * 4), 1), 64);
  const cudaStream_t s = as_stream(stream);
  for (int32_t l0 = 0; l0 < num_layers; l0 += pa::kCopyLayersPerLaunch) {
    const int nl = std::min(num_layers - l0, pa::kCopyLayersPerLaunch);
    for (int l = 0; l < nl; ++l) {
      p.k_cache[l] = k_caches[l0 + l];
      p.v_cache[l] = v_caches[l0 + l];
    }
    for (int32_t base = 0; base < num_pairs; base += pa::kCopyPairsPerLaunch) {
      const int n = std::min(num_pairs - base, pa::kCopyPairsPerLaunch);
      p.num_pairs = n;
      for (int i = 0; i < n; ++i)
        p.pairs[i] = make_int2(pairs_host[2 * (base + i)], pairs_host[2 * (base + i) + 1]);
      pa::pa_copy_blocks_kernel<<<dim3(n, static_cast<unsigned>(slices), nl), 256, 0, s>>>(p);
      if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
    }
  }
  return PA_OK;
}

pa_status pa_copy_blocks(const int32_t* pairs_host, int32_t num_pairs, void* k_cache,
                         void* v_cache, const pa_cache_desc* cache, void* stream) {
  return pa_copy_blocks_layers(pairs_host, num_pairs, &k_cache, &v_cache, 1, cache, stream);
}

pa_status pa_get_device_error(void* stream, uint32_t* flags) {
  if (!flags) return PA_ERR_INVALID_ARG;
  *flags = 0;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return PA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_pa_error_word, sizeof(v)) != cudaSuccess) return PA_ERR_CUDA;
  if (v) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(pa::g_pa_error_word, &zero, sizeof(zero)) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  *flags = v;
  return v ? PA_ERR_DEVICE_BOUNDS : PA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without any device allocation, for callers that cannot call
// cudaMalloc: the split-K workspace lives in a fixed array in the library's
// own device memory instead of a caller-provided buffer.
namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(32) << 20;  // 32 MiB per device

// Reserved in every device context that loads this library, until exit.
static __device__ __align__(256) unsigned char g_pa_static_workspace[kStaticWorkspaceBytes];

// Device address of g_pa_static_workspace in the current CUDA context. In
// host code the array's name is only a host-side handle; the device address
// belongs to a context (each device's primary context, or one the caller made
// current), so it is looked up with cudaGetSymbolAddress on the first call in
// each context and kept under that context's process-unique id (cuCtxGetId),
// which a context created after a device reset does not share.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(f);
}

// Id of the context current on this thread (0 when none is current yet).
bool current_context_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  *id = 0;
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  return ctx == nullptr || get_id(ctx, id) == CUDA_SUCCESS;
}

pa_status static_workspace_address(void** out) {
  static std::mutex mu;
  static std::unordered_map<unsigned long long, void*> addr;  // context id -> address
  unsigned long long id = 0;
  if (!current_context_id(&id)) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (id != 0) {
    const auto it = addr.find(id);
    if (it != addr.end()) {
      *out = it->second;
      return PA_OK;
    }
  }
  // first call in this context (or no context yet: the lookup makes the
  // current device's primary context current)
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_pa_static_workspace) != cudaSuccess || !p) return PA_ERR_CUDA;
  if (id == 0 && (!current_context_id(&id) || id == 0)) return PA_ERR_CUDA;
  addr[id] = p;
  *out = p;
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_static_workspace(
    const void* q, int32_t q_dtype, int32_t batch, int32_t num_q_heads, const void* k_cache,
    const void* v_cache, const pa_cache_desc* cache, const int32_t* block_tables,
    int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t max_context, float scale,
    void* out, int32_t partition_tokens, void* stream) {
  // the argument checks of pa_decode come first, so that an invalid call
  // gets the same status from both entry points
  int bs_log2 = 0;
  bool nothing = false;
  pa_status st = check_decode_args(q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache,
                                   block_tables, max_blocks_per_seq, context_lens, max_context,
                                   scale, out, partition_tokens, &bs_log2, &nothing);
  if (st != PA_OK || nothing) return st;
  const Plan pl = make_plan(batch, num_q_heads, max_context, partition_tokens, cache);
  if (!pl.fits) return PA_ERR_UNSUPPORTED;
  const size_t need = pl.ws_bytes;
  if (need > kStaticWorkspaceBytes) return PA_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    st = static_workspace_address(&ws);
    if (st != PA_OK) return st;
  }
  // The split-K partials need no initial value: every partial the reduce
  // kernel reads is written earlier in the same call.
  return pa_decode(q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache, block_tables,
                   max_blocks_per_seq, context_lens, max_context, scale, out, partition_tokens,
                   ws, need > 0 ? kStaticWorkspaceBytes : 0, stream);
}
