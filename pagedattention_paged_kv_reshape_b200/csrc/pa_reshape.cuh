// reshape_and_cache: scatter this step's new K/V rows into the paged cache.
//
// "vLLM 架构源码解析 | 第 1 篇" §3.3.3: the attention layer calls
// reshape_and_cache(k, v, kv_cache, slot_mapping) before paged_attention;
// §3.3.2 builds slot_mapping per token.  Slot s names physical block
// s / block_size, offset s % block_size; a negative slot marks a padding token.
//
// One warp per (token, KV head).  The K row and the V row of that pair are
// head_dim * elem bytes each (256 B for bf16 x 128); lanes move them as
// 16-byte vectors, so a warp writes both rows in one coalesced pass.  The
// copy is pure data movement: the bytes land unchanged.
#pragma once

#include "pa_common.cuh"

namespace pa {

__global__ void __launch_bounds__(256)
    reshape_and_cache_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                             uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                             const int* __restrict__ slot_mapping, int num_tokens,
                             int num_kv_heads, int row_vecs, int block_size,
                             long long num_slots) {
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(num_tokens) * num_kv_heads) return;
  const int t = static_cast<int>(gw / num_kv_heads);
  const int h = static_cast<int>(gw % num_kv_heads);
  const int slot = __ldg(slot_mapping + t);
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (lane == 0) report_error(PA_ERR_DEVICE_BOUNDS, kWhereReshapeSlot, t, slot);
    return;
  }
  const long long blk = slot / block_size, off = slot % block_size;
  const long long src = (static_cast<long long>(t) * num_kv_heads + h) * row_vecs;
  const long long dst = ((blk * num_kv_heads + h) * block_size + off) * row_vecs;
  // lanes [0, row_vecs) copy K, the next row_vecs lanes copy V, and so on
  for (int c = lane; c < 2 * row_vecs; c += 32) {
    if (c < row_vecs)
      k_cache[dst + c] = __ldg(k + src + c);
    else
      v_cache[dst + c - row_vecs] = __ldg(v + src + c - row_vecs);
  }
}

// The quantising write into an FP8 (e4m3) cache: element x of KV head h is
// stored as the e4m3 code of float(x) / scale[h] -- one correctly rounded fp32
// division, then round to nearest even, saturating at +-448 (the reading of
// the engine's calibrated FP8 KV cache, "vLLM 深度拆解" §10.1).  One warp per
// (token, KV head); lane l converts element pairs 2l, 2l + 64, ...
template <typename T>
__global__ void __launch_bounds__(256)
    reshape_and_cache_fp8_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                 uint8_t* __restrict__ k_cache, uint8_t* __restrict__ v_cache,
                                 const int* __restrict__ slot_mapping,
                                 const float* __restrict__ k_scale,
                                 const float* __restrict__ v_scale, int num_tokens,
                                 int num_kv_heads, int head_dim, int block_size,
                                 long long num_slots) {
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(num_tokens) * num_kv_heads) return;
  const int t = static_cast<int>(gw / num_kv_heads);
  const int h = static_cast<int>(gw % num_kv_heads);
  const int slot = __ldg(slot_mapping + t);
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (lane == 0) report_error(PA_ERR_DEVICE_BOUNDS, kWhereReshapeSlot, t, slot);
    return;
  }
  const long long blk = slot / block_size, off = slot % block_size;
  const long long src = (static_cast<long long>(t) * num_kv_heads + h) * head_dim;
  const long long dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
  const float ks = __ldg(k_scale + h), vs = __ldg(v_scale + h);
  for (int e = 2 * lane; e < head_dim; e += 64) {
    const float2 kx = make_float2(__fdiv_rn(to_f32<T>(k[src + e]), ks),
                                  __fdiv_rn(to_f32<T>(k[src + e + 1]), ks));
    const float2 vx = make_float2(__fdiv_rn(to_f32<T>(v[src + e]), vs),
                                  __fdiv_rn(to_f32<T>(v[src + e + 1]), vs));
    *reinterpret_cast<uint16_t*>(k_cache + dst + e) =
        __nv_cvt_float2_to_fp8x2(kx, __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint16_t*>(v_cache + dst + e) =
        __nv_cvt_float2_to_fp8x2(vx, __NV_SATFINITE, __NV_E4M3);
  }
}

}  // namespace pa
