// KV append and copy-on-write block copy (sm_100a).
//
// Append: each decode step computes only the new token's k_t, v_t and
// stores them in the cache (page "AI 陪读顶会论文（三）：KV Cache 显存占用计算与
// PagedAttention 原理拆解", section "为什么自回归解码必须使用 KV Cache？"); with
// paging, token slot s is row s % block_size of block s / block_size. In
// the [num_blocks][block_size][num_kv_heads][head_dim] layout all heads of
// one slot are contiguous, so a token is one contiguous row of
// num_kv_heads * head_dim elements on both sides: one CTA per token moves it
// with 16-byte vectors. An E4M3 cache stores e4m3_rn_satfinite(x * inv_scale)
// per (head, channel) (KV cache article, section "再往后：压 KV 的三条路线":
// FP8 K/V with per-channel scaling factors).
//
// Block copy: branches that share prompt blocks copy a block only where
// they diverge (KV cache article, section "PagedAttention：把操作系统的老智慧
// 搬进推理引擎"; page 3, section "PagedAttention 的破局哲学", third
// innovation). A block of K (and of V) is contiguous: block_size *
// num_kv_heads * head_dim elements.
#pragma once

#include "pa_common.cuh"

namespace pa {

struct AppendParams {
  const void* k;
  const void* v;
  const int64_t* slots;
  void* k_cache;
  void* v_cache;
  const float* k_inv_scale;
  const float* v_inv_scale;
  int64_t num_slots;  // num_blocks * block_size
  int row_elems;      // num_kv_heads * head_dim
};

// MODE 0: 16-bit copy; 1: f16 -> E4M3; 2: bf16 -> E4M3.
template <int MODE>
__global__ void __launch_bounds__(128) pa_append_kernel(const AppendParams p) {
  const int64_t tok = blockIdx.x;
  const int64_t s = p.slots[tok];
  if (s < 0) return;
  if (s >= p.num_slots) {
    if (threadIdx.x == 0) flag_error(PA_DEVERR_SLOT);
    return;
  }
  const int n8 = p.row_elems / 8;  // 8-element groups per token row
  if constexpr (MODE == 0) {
    const uint4* ks = reinterpret_cast<const uint4*>(p.k) + tok * n8;
    const uint4* vs = reinterpret_cast<const uint4*>(p.v) + tok * n8;
    uint4* kd = reinterpret_cast<uint4*>(p.k_cache) + s * n8;
    uint4* vd = reinterpret_cast<uint4*>(p.v_cache) + s * n8;
    for (int i = threadIdx.x; i < n8; i += blockDim.x) {
      const uint4 a = __ldg(ks + i);
      const uint4 c = __ldg(vs + i);
      kd[i] = a;
      vd[i] = c;
    }
  } else {
    using TIn = typename std::conditional<MODE == 1, __half, __nv_bfloat16>::type;
    const uint4* ks = reinterpret_cast<const uint4*>(p.k) + tok * n8;
    const uint4* vs = reinterpret_cast<const uint4*>(p.v) + tok * n8;
    uint2* kd = reinterpret_cast<uint2*>(p.k_cache) + s * n8;
    uint2* vd = reinterpret_cast<uint2*>(p.v_cache) + s * n8;
    const float4* kinv = reinterpret_cast<const float4*>(p.k_inv_scale);
    const float4* vinv = reinterpret_cast<const float4*>(p.v_inv_scale);
    auto quant8 = [](uint4 x, float4 s0, float4 s1) -> uint2 {
      const TIn* e = reinterpret_cast<const TIn*>(&x);
      const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      float y[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] = __fmul_rn(to_f32<TIn>(e[j]), sc[j]);
      uint2 r;
      r.x = f32x2_to_e4m3x2(y[0], y[1]) | (f32x2_to_e4m3x2(y[2], y[3]) << 16);
      r.y = f32x2_to_e4m3x2(y[4], y[5]) | (f32x2_to_e4m3x2(y[6], y[7]) << 16);
      return r;
    };
    for (int i = threadIdx.x; i < n8; i += blockDim.x) {
      kd[i] = quant8(__ldg(ks + i), __ldg(kinv + 2 * i), __ldg(kinv + 2 * i + 1));
      vd[i] = quant8(__ldg(vs + i), __ldg(vinv + 2 * i), __ldg(vinv + 2 * i + 1));
    }
  }
}

constexpr int kCopyPairsPerLaunch = 256;
constexpr int kCopyLayersPerLaunch = 32;

struct CopyParams {
  void* k_cache[kCopyLayersPerLaunch];  // one K and one V cache per layer of this launch
  void* v_cache[kCopyLayersPerLaunch];
  int64_t block_vec16;  // 16-byte vectors per block
  int num_pairs;
  int2 pairs[kCopyPairsPerLaunch];  // (src, dst), checked on the host
};

// grid.x = pair, grid.y = slices of the block, grid.z = layer; each thread
// moves 16 B of K and 16 B of V at a time.
__global__ void __launch_bounds__(256) pa_copy_blocks_kernel(const CopyParams p) {
  const int2 pr = p.pairs[blockIdx.x];
  const int layer = blockIdx.z;
  const uint4* ks = reinterpret_cast<const uint4*>(p.k_cache[layer]) + pr.x * p.block_vec16;
  const uint4* vs = reinterpret_cast<const uint4*>(p.v_cache[layer]) + pr.x * p.block_vec16;
  uint4* kd = reinterpret_cast<uint4*>(p.k_cache[layer]) + pr.y * p.block_vec16;
  uint4* vd = reinterpret_cast<uint4*>(p.v_cache[layer]) + pr.y * p.block_vec16;
  const int64_t stride = static_cast<int64_t>(gridDim.y) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x; i < p.block_vec16;
       i += stride) {
    const uint4 a = ks[i];
    const uint4 c = vs[i];
    kd[i] = a;
    vd[i] = c;
  }
}

}  // namespace pa
