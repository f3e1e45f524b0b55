// CUDA-core paged attention: the fp32 path, and a fallback for 16-bit types.
//
// Same work units as the tensor-core kernel (pa_sched.cuh), processed by a
// persistent grid of 4-warp CTAs.  Inside a unit, warp w takes the unit's
// 16-key tiles w, w+4, ... ; each tile's rows are found through the request's
// block-table row ("vLLM 深度拆解" §3.3; one 16-row run of a 16- or 32-token
// block, or two 8-token blocks) and read with plain vector loads.
// Each warp keeps an online softmax (running max m, sum l, unnormalised o)
// per tile row in the log2 domain; the epilogue merges the four warps.
//
// Lane layout for one block: for scores, lane = 2 * token + half, each lane
// dots half of head_dim (loaded 32 elements at a time, so head_dim 256 needs
// no more registers than 64) and a shuffle joins the halves; for P.V, lane
// owns head dims lane, lane + 32, ...  The query tile and the merge buffer
// live in dynamic shared memory (simt_smem_bytes).
//
// KV8: the cache holds FP8 e4m3 codes with one fp32 scale per KV head for K
// and for V; codes are decoded to fp32 as they are loaded, the K scale folds
// into the softmax scale and the V scale multiplies the accumulator.
#pragma once

#include "pa_sched.cuh"

namespace pa {

// N consecutive elements of a cache row, converted to fp32.
template <typename T, int N>
__device__ __forceinline__ void load_row_piece(const T* __restrict__ src, float (&dst)[N]) {
  constexpr int kBytes = N * sizeof(T);
  static_assert(kBytes % 16 == 0, "row pieces must be 16-byte vectors");
  const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int c = 0; c < kBytes / 16; ++c) {
    const uint4 w = __ldg(p + c);
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
    if constexpr (sizeof(T) == 4) {
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[c * 4 + e] = __uint_as_float(wv[e]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack2<T>(wv[e]);
        dst[c * 8 + 2 * e] = f.x;
        dst[c * 8 + 2 * e + 1] = f.y;
      }
    }
  }
}

template <int N>
__device__ __forceinline__ void load_row_piece(const uint8_t* __restrict__ src,
                                               float (&dst)[N]) {
  static_assert(N % 16 == 0, "row pieces must be 16-byte vectors");
  const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int c = 0; c < N / 16; ++c) {
    const uint4 w = __ldg(p + c);
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((wv[e >> 1] >> (16 * (e & 1))) & 0xffffu), __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
      dst[c * 16 + 2 * e] = f.x;
      dst[c * 16 + 2 * e + 1] = f.y;
    }
  }
}

__device__ __forceinline__ float fp8_to_f32(uint8_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
  return __half2float(*reinterpret_cast<const __half*>(&h));
}

// Dynamic shared memory of attn_simt_kernel<.., D, ..>: the query tile
// [kRows][D] and the four warps' merge buffer [4][kRows][D + 8], fp32.
template <int D>
constexpr int simt_smem_bytes() {
  return (kRows * D + 4 * kRows * (D + 8)) * 4;
}

template <typename T, int D, bool KV8 = false>
__global__ void __launch_bounds__(128, 1)
    attn_simt_kernel(Shape s, T* __restrict__ out, const T* __restrict__ q,
                     const typename std::conditional<KV8, uint8_t, T>::type* __restrict__ k_cache,
                     const typename std::conditional<KV8, uint8_t, T>::type* __restrict__ v_cache,
                     const int* __restrict__ block_tables, const int* __restrict__ qsl,
                     const int* __restrict__ seq_lens, Work w, float scale_log2,
                     const float* __restrict__ k_scale, const float* __restrict__ v_scale) {
  constexpr int NW = 4;
  constexpr int HALF = D / 2;
  constexpr int PIECE = 32;  // K elements a lane holds at a time
  constexpr int PER = D / 32;
  extern __shared__ __align__(16) float simt_smem[];
  auto q_s = reinterpret_cast<float (*)[D]>(simt_smem);                        // [kRows][D]
  auto co = reinterpret_cast<float (*)[kRows][D + 8]>(simt_smem + kRows * D);  // [NW][kRows][D+8]
  __shared__ float cm[NW * kRows];
  __shared__ float cl[NW * kRows];
  __shared__ Unit u_s;

  asm volatile("griddepcontrol.wait;" ::: "memory");  // the prep kernel's results
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int total_a = __ldcg(&w.sched->total_a);
  const int total = total_a + __ldcg(&w.sched->total_b);
  const int tok = lane >> 1, half = lane & 1;
  while (true) {
    if (tid == 0) {
      const int unit = atomicAdd(&w.sched->next, 1);
      if (unit < total) {
        int local, cls;
        const int row = locate_unit_thread(s, w, total_a, unit, local, cls);
        const RowInfo ri = load_row(s, qsl, seq_lens, row);
        u_s = decode_unit(s, ri, row, local, cls);
      } else {
        u_s.row = -1;
      }
    }
    __syncthreads();
    const Unit u = u_s;
    if (u.row < 0) break;
    if (u.kv_begin >= u.kv_end) {  // tile rows see no key of this partition
      __syncthreads();
      continue;
    }
    const int nrows = u.nq * s.gs;
    for (int idx = tid; idx < kRows * D; idx += NW * 32) {
      const int r = idx / D, d = idx % D, i = r / s.gs, g = r % s.gs;
      float val = 0.f;
      if (i < u.nq && g < u.rows)
        val = to_f32<T>(q[(static_cast<size_t>(u.token0 + i) * s.num_q_heads + u.head0 + g) * D + d]);
      q_s[r][d] = val;
    }
    __syncthreads();

    float m[kRows], l[kRows], o[kRows][PER], pr[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      m[r] = -INFINITY;
      l[r] = 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) o[r][e] = 0.f;
    }

    const int nblk = ceil_div(u.kv_end - u.kv_begin, kBlock);
    const int* table = block_tables + static_cast<size_t>(u.row) * s.table_stride;
    const float sl = KV8 ? scale_log2 * __ldg(k_scale + u.kvh) : scale_log2;
    for (int j = warp; j < nblk; j += NW) {
      const int blk_start = u.kv_begin + j * kBlock;
      // cache rows of keys 0-7 and 8-15 of this tile (two 8-token blocks, or
      // one run of 16 rows of a 16- or 32-token block)
      const int y0 = key_row(table, blk_start, s.block_size, s.num_kv_heads, u.kvh,
                             s.num_blocks, u.row);
      const int y1 = s.block_size >= kBlock ? y0 + 8
                     : blk_start + 8 < u.kv_end
                         ? key_row(table, blk_start + 8, s.block_size, s.num_kv_heads, u.kvh,
                                   s.num_blocks, u.row)
                         : y0;
      auto row_of = [&](int t) { return static_cast<size_t>(t < 8 ? y0 + t : y1 + t - 8); };
      // this lane's half of the dot products, one 32-element piece of the key
      // row at a time (each sum in the order of the head dims)
      float dot[kRows];
#pragma unroll
      for (int r = 0; r < kRows; ++r) dot[r] = 0.f;
#pragma unroll
      for (int pc = 0; pc < HALF / PIECE; ++pc) {
        float kr[PIECE];
        const size_t at = row_of(tok) * D + half * HALF + pc * PIECE;
        if constexpr (KV8)
          load_row_piece<PIECE>(k_cache + at, kr);
        else
          load_row_piece<T, PIECE>(k_cache + at, kr);
#pragma unroll
        for (int r = 0; r < kRows; ++r)
          if (r < nrows)
#pragma unroll
            for (int e = 0; e < PIECE; ++e)
              dot[r] = fmaf(q_s[r][half * HALF + pc * PIECE + e], kr[e], dot[r]);
      }
      const int kidx = blk_start + tok;
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        if (r < nrows) {
          float sc = dot[r];
          sc += __shfl_xor_sync(0xffffffffu, sc, 1);
          const int lim = u.lim0 + r / s.gs;
          const float x = kidx < lim ? sc * sl : -INFINITY;
          float bm = x;
#pragma unroll
          for (int off = 2; off < 32; off <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
          const float mn = fmaxf(m[r], bm);
          const float mu = mn == -INFINITY ? 0.f : mn;
          const float alpha = exp2f(m[r] - mu);
          const float p = exp2f(x - mu);
          float ps = half == 0 ? p : 0.f;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
          l[r] = l[r] * alpha + ps;
          m[r] = mn;
#pragma unroll
          for (int e = 0; e < PER; ++e) o[r][e] *= alpha;
          pr[r] = p;
        }
      }
      const int nvalid = u.kv_end - blk_start;  // V rows at or past this are padding
#pragma unroll 4
      for (int t2 = 0; t2 < kBlock; ++t2) {
        const auto* vt = v_cache + row_of(t2) * D;
        float vv[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          if constexpr (KV8)
            vv[e] = t2 < nvalid ? fp8_to_f32(vt[lane + 32 * e]) : 0.f;
          else
            vv[e] = t2 < nvalid ? to_f32<T>(vt[lane + 32 * e]) : 0.f;
        }
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          if (r < nrows) {
            const float pp = __shfl_sync(0xffffffffu, pr[r], 2 * t2);
#pragma unroll
            for (int e = 0; e < PER; ++e) o[r][e] = fmaf(pp, vv[e], o[r][e]);
          }
        }
      }
    }

    if constexpr (KV8) {  // the V scale of this KV head
      const float vsc = __ldg(v_scale + u.kvh);
#pragma unroll
      for (int r = 0; r < kRows; ++r)
#pragma unroll
        for (int e = 0; e < PER; ++e) o[r][e] *= vsc;
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      if (lane == 0) {
        cm[warp * kRows + r] = m[r];
        cl[warp * kRows + r] = l[r];
      }
#pragma unroll
      for (int e = 0; e < PER; ++e) co[warp][r][lane + 32 * e] = o[r][e];
    }
    __syncthreads();
    epilogue<T, D, NW>(s, u, cm, cl, co, out, w, tid, NW * 32);
    __syncthreads();
  }
}

}  // namespace pa
