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
  // launched with programmatic dependent launch: let the next kernel be
  // scheduled, and touch memory only once the previous grid is done
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
  // launched with programmatic dependent launch: let the next kernel be
  // scheduled, and touch memory only once the previous grid is done
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
  // launched with programmatic dependent launch: let the next kernel be
  // scheduled, and touch memory only once the previous grid is done
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
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


// Four consecutive elements of T as one load: 8 bytes for 16-bit types, 16 for
// fp32, with the conversions to and from fp32 (one RNE rounding on the way out).
template <typename T>
struct Quad {
  using Raw = std::conditional_t<sizeof(T) == 2, uint2, float4>;
  static __device__ __forceinline__ Raw load(const T* p) {
    return *reinterpret_cast<const Raw*>(p);
  }
  static __device__ __forceinline__ void store(T* p, const Raw& r) {
    *reinterpret_cast<Raw*>(p) = r;
  }
  static __device__ __forceinline__ void to_f32(const Raw& r, float (&f)[4]) {
    if constexpr (sizeof(T) == 2) {
      const float2 a = unpack2<T>(r.x), b = unpack2<T>(r.y);
      f[0] = a.x, f[1] = a.y, f[2] = b.x, f[3] = b.y;
    } else {
      f[0] = r.x, f[1] = r.y, f[2] = r.z, f[3] = r.w;
    }
  }
  static __device__ __forceinline__ Raw from_f32(const float (&f)[4]) {
    if constexpr (sizeof(T) == 2)
      return make_uint2(pack2<T>(f[0], f[1]), pack2<T>(f[2], f[3]));
    else
      return make_float4(f[0], f[1], f[2], f[3]);
  }
};

// The same operation with vector accesses, for rot_dim a multiple of 8 and a
// 16-byte aligned cos_sin table (the host picks it then).  Work is split in
// four-element quads: with NeoX pairs a rotation unit is the quad at 4u and
// its partner quad at rot_dim/2 + 4u (cos/sin of pairs 4u..4u+3 as two float4
// loads); with (2i, 2i+1) pairs a unit is the single quad at 4u, holding
// pairs 2u and 2u+1.  One warp per (token, part): a part is up to kHeads
// query heads, rotated in place, or up to kHeads KV heads, whose rotated k
// rows, pass-through dims and v rows go to the token's cache slot.  Each lane
// loads kBatch units before it computes and stores any.  Measured on B200
// (16384 tokens, 32/8 heads, D=128, bf16): 16 heads per warp with batches of
// 4 beats 8 (fewer, longer-lived warps) and batches of 8 (registers cut the
// warps per SM).  Arithmetic per element is the scalar kernel's.
#ifndef PA_ROPE_HEADS
#define PA_ROPE_HEADS 16
#endif
#ifndef PA_ROPE_BATCH
#define PA_ROPE_BATCH 4
#endif
constexpr int kRopeHeads = PA_ROPE_HEADS;  // heads per warp

template <typename T>
__global__ void __launch_bounds__(256)
    rope_reshape_and_cache_vec_kernel(T* __restrict__ q, const T* __restrict__ k,
                                      const T* __restrict__ v, T* __restrict__ k_cache,
                                      T* __restrict__ v_cache, const int* __restrict__ slot_mapping,
                                      const int* __restrict__ positions,
                                      const float* __restrict__ cos_sin, int max_position,
                                      int rot_dim, bool neox, int num_tokens, int num_q_heads,
                                      int num_kv_heads, int head_dim, int block_size,
                                      long long num_slots) {
  // launched with programmatic dependent launch: let the next kernel be
  // scheduled, and touch memory only once the previous grid is done
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  using Q = Quad<T>;
  using Raw = typename Q::Raw;
  constexpr int kHeads = kRopeHeads, kBatch = PA_ROPE_BATCH;
  const int qparts = (num_q_heads + kHeads - 1) / kHeads;
  const int parts = qparts + (num_kv_heads + kHeads - 1) / kHeads;
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(num_tokens) * parts) return;
  const int t = static_cast<int>(gw / parts), part = static_cast<int>(gw % parts);
  const int pos = __ldg(positions + t);
  if (pos < 0 || pos >= max_position) {
    if (lane == 0 && part == 0) report_error(PA_ERR_DEVICE_BOUNDS, kWhereRopePos, t, pos);
    return;
  }
  const float* cs = cos_sin + static_cast<size_t>(pos) * rot_dim;
  const int half = rot_dim / 2;
  const int ru = neox ? rot_dim / 8 : rot_dim / 4;  // rotation units per row
  const int pu = (head_dim - rot_dim) / 4;           // pass-through quads per row

  // Rotate `nh` rows (src -> dst, row strides in elements); with `pass`, also
  // copy each row's dims from rot_dim on.
  auto rotate_rows = [&](const T* src, long long src_stride, T* dst, long long dst_stride,
                         int nh, bool pass) {
    const int upr = ru + (pass ? pu : 0);
    const int n = nh * upr;
    for (int base = lane; base < n; base += 32 * kBatch) {
      Raw xa[kBatch], xb[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int idx = base + 32 * j;
        if (idx >= n) break;
        const int r = idx / upr, u = idx - r * upr;
        const T* x = src + r * src_stride;
        if (u >= ru) {
          xa[j] = Q::load(x + rot_dim + 4 * (u - ru));
        } else {
          xa[j] = Q::load(x + 4 * u);
          if (neox) xb[j] = Q::load(x + half + 4 * u);
        }
      }
      // the table row is shared by every warp of the token: cached after the
      // first touch, so its loads wait here rather than holding registers above
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int idx = base + 32 * j;
        if (idx >= n) break;
        const int r = idx / upr, u = idx - r * upr;
        T* y = dst + r * dst_stride;
        if (u >= ru) {
          Q::store(y + rot_dim + 4 * (u - ru), xa[j]);
          continue;
        }
        float cc[4], ss[4];
        if (neox) {
          const float4 c4 = __ldg(reinterpret_cast<const float4*>(cs + 4 * u));
          const float4 s4 = __ldg(reinterpret_cast<const float4*>(cs + half + 4 * u));
          cc[0] = c4.x, cc[1] = c4.y, cc[2] = c4.z, cc[3] = c4.w;
          ss[0] = s4.x, ss[1] = s4.y, ss[2] = s4.z, ss[3] = s4.w;
        } else {
          const float2 c2 = __ldg(reinterpret_cast<const float2*>(cs + 2 * u));
          const float2 s2 = __ldg(reinterpret_cast<const float2*>(cs + half + 2 * u));
          cc[0] = cc[1] = c2.x, cc[2] = cc[3] = c2.y;
          ss[0] = ss[1] = s2.x, ss[2] = ss[3] = s2.y;
        }
        float a[4], oa[4];
        Q::to_f32(xa[j], a);
        if (neox) {
          float b[4], ob[4];
          Q::to_f32(xb[j], b);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            oa[e] = fmaf(a[e], cc[e], -b[e] * ss[e]);
            ob[e] = fmaf(b[e], cc[e], a[e] * ss[e]);
          }
          Q::store(y + 4 * u, Q::from_f32(oa));
          Q::store(y + half + 4 * u, Q::from_f32(ob));
        } else {
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            oa[e] = fmaf(a[e], cc[e], -a[e + 1] * ss[e]);
            oa[e + 1] = fmaf(a[e + 1], cc[e], a[e] * ss[e]);
          }
          Q::store(y + 4 * u, Q::from_f32(oa));
        }
      }
    }
  };

  if (part < qparts) {
    const int h0 = part * kHeads;
    const int nh = min(kHeads, num_q_heads - h0);
    T* x = q + (static_cast<size_t>(t) * num_q_heads + h0) * head_dim;
    rotate_rows(x, head_dim, x, head_dim, nh, false);
    return;
  }
  const int h0 = (part - qparts) * kHeads;
  const int nh = min(kHeads, num_kv_heads - h0);
  const int slot = __ldg(slot_mapping + t);
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (lane == 0 && h0 == 0) report_error(PA_ERR_DEVICE_BOUNDS, kWhereReshapeSlot, t, slot);
    return;
  }
  const long long blk = slot / block_size, off = slot % block_size;
  const size_t src = (static_cast<size_t>(t) * num_kv_heads + h0) * head_dim;
  const size_t dst = ((blk * num_kv_heads + h0) * block_size + off) * head_dim;
  const long long cache_stride = static_cast<long long>(block_size) * head_dim;
  rotate_rows(k + src, head_dim, k_cache + dst, cache_stride, nh, true);
  // v rows: 16-byte copies, all loads of a batch before its stores
  const int vpr = head_dim * static_cast<int>(sizeof(T)) / 16;
  const int n = nh * vpr;
  const uint4* vs = reinterpret_cast<const uint4*>(v + src);
  uint4* vd = reinterpret_cast<uint4*>(v_cache + dst);
  const long long vd_stride = cache_stride * static_cast<long long>(sizeof(T)) / 16;
  for (int base = lane; base < n; base += 32 * kBatch) {
    uint4 w[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (base + 32 * j < n) w[j] = __ldg(vs + base + 32 * j);
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int idx = base + 32 * j;
      if (idx < n) vd[(idx / vpr) * vd_stride + idx % vpr] = w[j];
    }
  }
}

}  // namespace pa
