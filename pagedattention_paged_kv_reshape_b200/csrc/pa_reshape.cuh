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

// Rotary position embedding fused with the cache write ("vLLM 深度拆解" §6.1:
// fold elementwise work into the neighbouring kernel so activations cross
// HBM once).  The rotation is RoFormer's: the first rot_dim dims of a head
// form rot_dim/2 pairs -- (2i, 2i+1), or (i, i + rot_dim/2) with `neox` --
// and the pair (x1, x2) of a token at position p becomes
// (x1 c - x2 s, x2 c + x1 s) with c, s = cos_sin[p][i], cos_sin[p][R/2 + i].
// One warp per (token, head): a query head is rotated in place; a KV head
// writes its rotated k row and its v row into the cache at the token's slot
// (padding tokens, slot < 0, rotate q only).  Each result is computed in fp32
// and rounded once to the storage type.
template <typename T>
__global__ void __launch_bounds__(256)
    rope_reshape_and_cache_kernel(T* __restrict__ q, const T* __restrict__ k,
                                  const T* __restrict__ v, T* __restrict__ k_cache,
                                  T* __restrict__ v_cache, const int* __restrict__ slot_mapping,
                                  const int* __restrict__ positions,
                                  const float* __restrict__ cos_sin, int max_position,
                                  int rot_dim, bool neox, int num_tokens, int num_q_heads,
                                  int num_kv_heads, int head_dim, int block_size,
                                  long long num_slots) {
  const int heads = num_q_heads + num_kv_heads;
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(num_tokens) * heads) return;
  const int t = static_cast<int>(gw / heads), h = static_cast<int>(gw % heads);
  const int pos = __ldg(positions + t);
  if (pos < 0 || pos >= max_position) {
    if (lane == 0 && h == 0) report_error(PA_ERR_DEVICE_BOUNDS, kWhereRopePos, t, pos);
    return;
  }
  const float* cs = cos_sin + static_cast<size_t>(pos) * rot_dim;
  const int half = rot_dim / 2;
  auto pair = [&](int i, int& i1, int& i2) {
    i1 = neox ? i : 2 * i;
    i2 = neox ? i + half : 2 * i + 1;
  };
  if (h < num_q_heads) {
    T* x = q + (static_cast<size_t>(t) * num_q_heads + h) * head_dim;
    for (int i = lane; i < half; i += 32) {
      int i1, i2;
      pair(i, i1, i2);
      const float c = __ldg(cs + i), sn = __ldg(cs + half + i);
      const float x1 = to_f32<T>(x[i1]), x2 = to_f32<T>(x[i2]);
      x[i1] = from_f32<T>(fmaf(x1, c, -x2 * sn));
      x[i2] = from_f32<T>(fmaf(x2, c, x1 * sn));
    }
    return;
  }
  const int kh = h - num_q_heads;
  const int slot = __ldg(slot_mapping + t);
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (lane == 0) report_error(PA_ERR_DEVICE_BOUNDS, kWhereReshapeSlot, t, slot);
    return;
  }
  const long long blk = slot / block_size, off = slot % block_size;
  const size_t src = (static_cast<size_t>(t) * num_kv_heads + kh) * head_dim;
  const size_t dst = ((blk * num_kv_heads + kh) * block_size + off) * head_dim;
  for (int i = lane; i < half; i += 32) {
    int i1, i2;
    pair(i, i1, i2);
    const float c = __ldg(cs + i), sn = __ldg(cs + half + i);
    const float x1 = to_f32<T>(k[src + i1]), x2 = to_f32<T>(k[src + i2]);
    k_cache[dst + i1] = from_f32<T>(fmaf(x1, c, -x2 * sn));
    k_cache[dst + i2] = from_f32<T>(fmaf(x2, c, x1 * sn));
  }
  for (int e = rot_dim + lane; e < head_dim; e += 32) k_cache[dst + e] = k[src + e];
  for (int e = lane; e < head_dim; e += 32) v_cache[dst + e] = v[src + e];
}

}  // namespace pa
