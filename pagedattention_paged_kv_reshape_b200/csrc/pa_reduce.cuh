// Split-K reduce: merge the partial states of queries whose keys span more
// than one 512-key partition, by log-sum-exp:
//   M = max_p lse_p,  w_p = 2^(lse_p - M),  out = sum_p w_p o_p / sum_p w_p
// (lse_p in log2 units, o_p already normalised by its partition's sum).
//
// One CTA per (request, slice of kReduceTokens query tokens, group of eight
// query heads; CTAs stride over the slices of longer rows): it reads the
// request's metadata once; each warp merges one head for the slice's tokens,
// each lane owning D/32 dims.  The
// loop over partitions is unrolled so that eight partitions' loads are in
// flight at once (32K-token contexts have 64 partitions).  Rows handled by the
// tcgen05 chunk kernel are skipped: that kernel writes them directly.
//
// With many partitions per row (long contexts) that layout leaves too few
// CTAs and a long chain of dependent load batches per warp, so
// reduce_wide_kernel takes one query head per CTA instead: its eight warps
// split the partitions of each token (warp w merges partitions w, w+8, ...
// against the common maximum) and add their sums through shared memory.
//
// Both kernels are launched behind the attention kernels with programmatic
// dependent launch (their CTAs may be scheduled as attention CTAs retire) and
// wait for those grids to complete before reading the partials.
#pragma once

#include "pa_sched.cuh"

namespace pa {

constexpr int kReduceTokens = 16;

template <typename T, int D>
__global__ void __launch_bounds__(256) reduce_kernel(Shape s, const int* __restrict__ qsl,
                                                     const int* __restrict__ seq_lens, Work w,
                                                     T* __restrict__ out) {
  // the next kernel on the stream may be scheduled now; it waits for this grid
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int kPer = D / 32;  // dims per lane
  constexpr int kUnroll = 8;
  const int row = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const RowInfo ri = load_row(s, qsl, seq_lens, row);
  if (!ri.ok || ri.q_len == 0 || is_chunk_row(s, ri)) return;
  const int head = blockIdx.z * 8 + warp;
  if (head >= s.num_q_heads) return;
  for (int t0 = blockIdx.y * kReduceTokens; t0 < ri.q_len; t0 += gridDim.y * kReduceTokens) {
    const int nt = min(kReduceTokens, ri.q_len - t0);
    for (int ti = t0; ti < t0 + nt; ++ti) {
      const int parts = parts_for(ri.seq_len - ri.q_len + ti + 1);
      if (parts <= 1) continue;  // written directly by the attention kernel
      const int token = ri.token0 + ti;
      const size_t base = (static_cast<size_t>(token) * s.num_q_heads + head) * s.p_stride;
      const float* lse = w.part_lse + base;
      float mx = -INFINITY;
      for (int p = lane; p < parts; p += 32) mx = fmaxf(mx, lse[p]);
  #pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float acc[kPer];
  #pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
      float wsum = 0.f;
      const float* po = w.part_o + base * D + lane * kPer;
      for (int p0 = 0; p0 < parts; p0 += 32) {
        const int n = min(32, parts - p0);
        const float wl = lane < n ? exp2f(lse[p0 + lane] - mx) : 0.f;  // weight of partition p0+lane
        for (int j0 = 0; j0 < n; j0 += kUnroll) {
          float v[kUnroll][kPer];
  #pragma unroll
          for (int j = 0; j < kUnroll; ++j) {  // issue every load first
            const int jj = min(j0 + j, n - 1);
            const float* src = po + static_cast<size_t>(p0 + jj) * D;
            if constexpr (kPer == 8) {
              const float4 a = *reinterpret_cast<const float4*>(src);
              const float4 b = *reinterpret_cast<const float4*>(src + 4);
              v[j][0] = a.x; v[j][1] = a.y; v[j][2] = a.z; v[j][3] = a.w;
              v[j][4] = b.x; v[j][5] = b.y; v[j][6] = b.z; v[j][7] = b.w;
            } else if constexpr (kPer == 4) {
              const float4 a = *reinterpret_cast<const float4*>(src);
              v[j][0] = a.x; v[j][1] = a.y; v[j][2] = a.z; v[j][3] = a.w;
            } else {
              const float2 a = *reinterpret_cast<const float2*>(src);
              v[j][0] = a.x; v[j][1] = a.y;
            }
          }
  #pragma unroll
          for (int j = 0; j < kUnroll; ++j) {
            const float wj = __shfl_sync(0xffffffffu, wl, (j0 + j) & 31);
            if (j0 + j < n) {
              wsum += wj;
  #pragma unroll
              for (int e = 0; e < kPer; ++e) acc[e] = fmaf(wj, v[j][e], acc[e]);
            }
          }
        }
      }
      const float inv = 1.f / wsum;
      T* o = out + (static_cast<size_t>(token) * s.num_q_heads + head) * D + lane * kPer;
  #pragma unroll
      for (int e = 0; e < kPer; ++e) o[e] = from_f32<T>(acc[e] * inv);
    }
  }
}

// Loads of `kPer` floats of one partition's normalised o.
template <int kPer>
__device__ __forceinline__ void load_part(const float* src, float (&v)[kPer]) {
  if constexpr (kPer == 8) {
    const float4 a = *reinterpret_cast<const float4*>(src);
    const float4 b = *reinterpret_cast<const float4*>(src + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else if constexpr (kPer == 4) {
    const float4 a = *reinterpret_cast<const float4*>(src);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else {
    const float2 a = *reinterpret_cast<const float2*>(src);
    v[0] = a.x; v[1] = a.y;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) reduce_wide_kernel(Shape s, const int* __restrict__ qsl,
                                                          const int* __restrict__ seq_lens,
                                                          Work w, T* __restrict__ out) {
  // the next kernel on the stream may be scheduled now; it waits for this grid
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int kPer = D / 32;  // dims per lane
  constexpr int kWarps = 8, kUnroll = 8;
  __shared__ float red_o[kWarps][D];
  __shared__ float red_w[kWarps];
  const int row = blockIdx.x, head = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const RowInfo ri = load_row(s, qsl, seq_lens, row);
  if (!ri.ok || ri.q_len == 0 || is_chunk_row(s, ri) || head >= s.num_q_heads) return;
  for (int t0 = blockIdx.y * kReduceTokens; t0 < ri.q_len; t0 += gridDim.y * kReduceTokens) {
    const int nt = min(kReduceTokens, ri.q_len - t0);
    for (int ti = t0; ti < t0 + nt; ++ti) {
      const int parts = parts_for(ri.seq_len - ri.q_len + ti + 1);
      if (parts <= 1) continue;  // written directly by the attention kernel
      const int token = ri.token0 + ti;
      const size_t base = (static_cast<size_t>(token) * s.num_q_heads + head) * s.p_stride;
      const float* lse = w.part_lse + base;
      // every warp finds the same maximum over all partitions
      float mx = -INFINITY;
      for (int p = lane; p < parts; p += 32) mx = fmaxf(mx, lse[p]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float acc[kPer];
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
      float wsum = 0.f;
      const float* po = w.part_o + base * D + lane * kPer;
      // this warp's partitions: warp, warp + 8, ...; kUnroll of them in flight
      for (int p0 = warp; p0 < parts; p0 += kWarps * kUnroll) {
        float v[kUnroll][kPer];
        float wt[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
          const int p = p0 + j * kWarps;
          if (p < parts) {
            load_part<kPer>(po + static_cast<size_t>(p) * D, v[j]);
            wt[j] = lse[p];
          }
        }
#pragma unroll
        for (int j = 0; j < kUnroll; ++j) {
          if (p0 + j * kWarps < parts) {
            const float f = exp2f(wt[j] - mx);
            wsum += f;
#pragma unroll
            for (int e = 0; e < kPer; ++e) acc[e] = fmaf(f, v[j][e], acc[e]);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < kPer; ++e) red_o[warp][lane * kPer + e] = acc[e];
      if (lane == 0) red_w[warp] = wsum;
      __syncthreads();
      if (threadIdx.x < D) {
        float o = 0.f, ws = 0.f;
#pragma unroll
        for (int q = 0; q < kWarps; ++q) {
          o += red_o[q][threadIdx.x];
          ws += red_w[q];
        }
        out[(static_cast<size_t>(token) * s.num_q_heads + head) * D + threadIdx.x] =
            from_f32<T>(o / ws);
      }
      __syncthreads();  // red_o is written again for the next token
    }
  }
}

}  // namespace pa
