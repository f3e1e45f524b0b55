// Work decomposition shared by the attention kernels, the split-K reduce and
// the epilogue that merges per-warp online-softmax states.
//
// A batch is a list of rows (requests).  Row r has q_len query tokens (1 for
// a decode row) at positions seq_len - q_len + i ("vLLM 架构源码解析" §3.3.2:
// positions run from num_computed_tokens) and reads keys 0 .. position.
//
// Work unit = (row, query tile, KV head slice, partition):
//   * query tile   : up to `qpt` consecutive query tokens of the row;
//   * head slice   : up to 16 query heads of one KV head (all of a GQA group
//                    when it has <= 16 heads), so each KV block is streamed
//                    once per KV head and tile;
//   * partition    : keys [p*512, (p+1)*512) -- the split-K unit.
// Tile rows are (query token, head) pairs, row = i * gs + g, at most 16.
//
// A one-CTA prep kernel writes row_start[r] = number of units before row r,
// so a persistent attention CTA maps a unit index to its row with a short
// forward scan and decodes the rest by division.
#pragma once

#include "pa_common.cuh"

namespace pa {

struct Shape {
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int group;        // num_q_heads / num_kv_heads
  int gs;           // heads per slice = min(group, 16)
  int ns;           // slices per KV head = ceil(group / 16)
  int qpt;          // query tokens per tile (1 for pa_decode)
  int head_dim;
  int table_stride;
  int num_blocks;
  int max_seq_len;  // host bound on seq_lens / context_lens
  int max_query_len;
  int total_q;
  int p_stride;     // partitions per (token, head) in the workspace
};

// Per-row metadata.  `qsl` is null for decode batches (row r owns token r).
struct RowInfo {
  int seq_len;
  int q_len;
  int token0;
  bool ok;
};

__device__ __forceinline__ RowInfo load_row(const Shape& s, const int* __restrict__ qsl,
                                            const int* __restrict__ seq_lens, int row) {
  RowInfo ri;
  ri.seq_len = seq_lens[row];
  if (qsl) {
    ri.token0 = qsl[row];
    ri.q_len = qsl[row + 1] - ri.token0;
  } else {
    ri.token0 = row;
    ri.q_len = ri.seq_len > 0 ? 1 : 0;  // an empty decode context: a zero output row
  }
  ri.ok = ri.seq_len >= 0 && ri.seq_len <= s.max_seq_len &&
          ri.seq_len <= s.table_stride * kBlock && ri.q_len >= 0 &&
          ri.q_len <= ri.seq_len && ri.token0 >= 0 && ri.token0 + ri.q_len <= s.total_q &&
          (qsl == nullptr || ri.q_len <= s.max_query_len);
  return ri;
}

__device__ __forceinline__ int row_units(const Shape& s, const RowInfo& ri) {
  if (!ri.ok || ri.q_len == 0) return 0;
  const int items = ceil_div(ri.q_len, s.qpt);
  const int parts = ceil_div(ri.seq_len, kPart);
  return items * parts * s.num_kv_heads * s.ns;
}

struct Unit {
  int row;
  int token0;    // first query token of the tile (index into q / out)
  int nq;        // query tokens in the tile
  int kvh;       // KV head
  int head0;     // first query head of the slice
  int rows;      // valid heads in the slice (<= gs)
  int p;         // partition
  int kv_begin;  // first key of the partition
  int kv_end;    // one past the last key any tile row may see in this partition
  int lim0;      // keys visible to tile row 0 (its position + 1); row i*gs+g sees lim0 + i
};

// Decode the unit at offset `local` inside row `row`.  Unit order inside a row:
// query tile fastest, then partition, then head slice -- consecutive units of
// a prefill chunk read the same KV blocks, which stay in L2.
__device__ __forceinline__ Unit decode_unit(const Shape& s, const RowInfo& ri, int row,
                                            int local) {
  Unit u;
  const int items = ceil_div(ri.q_len, s.qpt);
  const int parts = ceil_div(ri.seq_len, kPart);
  const int item = local % items;
  const int rest = local / items;
  u.p = rest % parts;
  const int hu = rest / parts;
  u.kvh = hu / s.ns;
  const int slice = hu % s.ns;
  u.head0 = u.kvh * s.group + slice * kRows;
  u.rows = min(s.gs, s.group - slice * kRows);
  u.row = row;
  const int q0 = item * s.qpt;
  u.nq = min(s.qpt, ri.q_len - q0);
  u.token0 = ri.token0 + q0;
  u.lim0 = ri.seq_len - ri.q_len + q0 + 1;
  u.kv_begin = u.p * kPart;
  u.kv_end = min(u.lim0 + u.nq - 1, u.kv_begin + kPart);
  return u;
}

// Number of partitions whose partial state a query at `limit` visible keys
// has (1 = written directly as output, no reduce).
__device__ __forceinline__ int parts_for(int limit) { return ceil_div(limit, kPart); }

// ---------------------------------------------------------------------------
// Prep kernel: validate rows, write row_start (exclusive prefix of units),
// zero the output rows of empty decode requests.  One CTA of 1024 threads.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(1024) schedule_kernel(Shape s, const int* __restrict__ qsl,
                                                        const int* __restrict__ seq_lens,
                                                        int* __restrict__ row_start,
                                                        T* __restrict__ out) {
  __shared__ int warp_tot[32];
  __shared__ int carry_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry_s = 0;
    if (qsl && (qsl[0] != 0 || qsl[s.num_seqs] != s.total_q))
      report_error(PA_ERR_DEVICE_BOUNDS, kWhereRowMeta, -1, qsl[s.num_seqs]);
  }
  __syncthreads();
  for (int base = 0; base < s.num_seqs; base += 1024) {
    const int r = base + tid;
    int v = 0;
    if (r < s.num_seqs) {
      const RowInfo ri = load_row(s, qsl, seq_lens, r);
      if (!ri.ok) report_error(PA_ERR_DEVICE_BOUNDS, kWhereRowMeta, r, ri.seq_len);
      v = row_units(s, ri);
      if (ri.ok && qsl == nullptr && ri.seq_len == 0) {
        // attention over an empty context: a zero row
        T* o = out + static_cast<size_t>(r) * s.num_q_heads * s.head_dim;
        for (int i = 0; i < s.num_q_heads * s.head_dim; ++i) o[i] = from_f32<T>(0.f);
      }
    }
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;
    }
    __syncthreads();
    const int excl = carry_s + x - v + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (r < s.num_seqs) row_start[r] = excl;
    __syncthreads();
    if (tid == 1023) carry_s = excl + v;
    __syncthreads();
  }
  if (tid == 0) row_start[s.num_seqs] = carry_s;
}

// Largest r with row_start[r] <= u, scanning forward from `cursor` one warp
// (32 rows) at a time.  All lanes of the warp call it; returns the row and
// its row_start in `start`.  Requires u < row_start[num_seqs].
__device__ __forceinline__ int find_row_warp(const int* __restrict__ row_start, int num_seqs,
                                             int u, int cursor, int& start) {
  const int lane = threadIdx.x & 31;
  while (true) {
    const int idx = cursor + lane;
    const int v = idx <= num_seqs ? row_start[idx] : 0x7fffffff;
    const unsigned m = __ballot_sync(0xffffffffu, v <= u);
    const int cnt = __popc(m);
    if (cnt < 32) {
      start = __shfl_sync(0xffffffffu, v, cnt - 1);
      return cursor + cnt - 1;
    }
    cursor += 31;
  }
}

// Binary search version for a single thread.
__device__ __forceinline__ int find_row_thread(const int* __restrict__ row_start, int num_seqs,
                                               int u) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (row_start[mid] <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------
// Epilogue: merge NW warps' online-softmax states for the tile's rows and
// write either the final output (row's keys all in partition 0) or this
// partition's partial (normalised o and log2-sum-exp) for the reduce.
//
// Shared layout: cm[NW][16], cl[NW][16] (running max in log2 units and sum),
// co[NW][16][D + 8] (unnormalised accumulators).
// ---------------------------------------------------------------------------
template <typename T, int D, int NW>
__device__ __forceinline__ void combine_and_store(const Shape& s, const Unit& u, float* cm,
                                                  float* cl, float (*co)[kRows][D + 8],
                                                  T* __restrict__ out, float* __restrict__ part_o,
                                                  float* __restrict__ part_lse, int tid) {
  constexpr int kChunks = D / 8;
  for (int task = tid; task < kRows * kChunks; task += NW * 32) {
    const int r = task / kChunks, c = task % kChunks;
    const int i = r / s.gs, g = r % s.gs;
    if (i >= u.nq || g >= u.rows) continue;
    const int limit = u.lim0 + i;
    const int parts = parts_for(limit);
    if (u.p >= parts) continue;  // no key of this partition is visible to the row
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) mx = fmaxf(mx, cm[w * kRows + r]);
    float L = 0.f;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = exp2f(cm[w * kRows + r] - mx);
      L += f * cl[w * kRows + r];
      const float4 a = *reinterpret_cast<const float4*>(&co[w][r][c * 8]);
      const float4 b = *reinterpret_cast<const float4*>(&co[w][r][c * 8 + 4]);
      acc[0] += f * a.x; acc[1] += f * a.y; acc[2] += f * a.z; acc[3] += f * a.w;
      acc[4] += f * b.x; acc[5] += f * b.y; acc[6] += f * b.z; acc[7] += f * b.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int token = u.token0 + i;
    const int head = u.head0 + g;
    if (parts == 1) {
      T* o = out + (static_cast<size_t>(token) * s.num_q_heads + head) * D + c * 8;
      if constexpr (sizeof(T) == 2) {
        uint4 v;
        v.x = pack2<T>(acc[0] * inv, acc[1] * inv);
        v.y = pack2<T>(acc[2] * inv, acc[3] * inv);
        v.z = pack2<T>(acc[4] * inv, acc[5] * inv);
        v.w = pack2<T>(acc[6] * inv, acc[7] * inv);
        *reinterpret_cast<uint4*>(o) = v;
      } else {
        *reinterpret_cast<float4*>(o) =
            make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<float4*>(o + 4) =
            make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      }
    } else {
      const size_t slot = (static_cast<size_t>(token) * s.num_q_heads + head) * s.p_stride + u.p;
      float* po = part_o + slot * D + c * 8;
      *reinterpret_cast<float4*>(po) =
          make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      *reinterpret_cast<float4*>(po + 4) =
          make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      if (c == 0) part_lse[slot] = L > 0.f ? mx + log2f(L) : -INFINITY;
    }
  }
}

// ---------------------------------------------------------------------------
// Split-K reduce: for every (query token, head) whose keys span more than one
// partition, merge the partials by log-sum-exp:
//   M = max_p lse_p,  w_p = 2^(lse_p - M),  out = sum_p w_p o_p / sum_p w_p.
// One warp per (token, head).
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) reduce_kernel(Shape s, const int* __restrict__ qsl,
                                                     const int* __restrict__ seq_lens,
                                                     const float* __restrict__ part_o,
                                                     const float* __restrict__ part_lse,
                                                     T* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int token = static_cast<int>(gw / s.num_q_heads);
  const int head = static_cast<int>(gw % s.num_q_heads);
  if (token >= s.total_q) return;
  int row = token;
  if (qsl) {  // the request owning this token
    int lo = 0, hi = s.num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (qsl[mid] <= token)
        lo = mid;
      else
        hi = mid - 1;
    }
    row = lo;
  }
  const RowInfo ri = load_row(s, qsl, seq_lens, row);
  if (!ri.ok || ri.q_len == 0) return;
  const int limit = ri.seq_len - ri.q_len + (token - ri.token0) + 1;
  const int parts = parts_for(limit);
  if (parts <= 1) return;
  const size_t base = (static_cast<size_t>(token) * s.num_q_heads + head) * s.p_stride;
  float mx = -INFINITY;
  for (int p = lane; p < parts; p += 32) mx = fmaxf(mx, part_lse[base + p]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  constexpr int kPer = D / 32;  // dims per lane
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  for (int p0 = 0; p0 < parts; p0 += 32) {
    const int p = p0 + lane;
    const float w = p < parts ? exp2f(part_lse[base + p] - mx) : 0.f;
    const int n = min(32, parts - p0);
    for (int j = 0; j < n; ++j) {
      const float wj = __shfl_sync(0xffffffffu, w, j);
      wsum += wj;
      const float* po = part_o + (base + p0 + j) * D + lane * kPer;
      if constexpr (kPer == 4) {
        const float4 a = *reinterpret_cast<const float4*>(po);
        acc[0] += wj * a.x; acc[1] += wj * a.y; acc[2] += wj * a.z; acc[3] += wj * a.w;
      } else {
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] += wj * po[e];
      }
    }
  }
  const float inv = 1.f / wsum;
  T* o = out + (static_cast<size_t>(token) * s.num_q_heads + head) * D + lane * kPer;
#pragma unroll
  for (int e = 0; e < kPer; ++e) o[e] = from_f32<T>(acc[e] * inv);
}

}  // namespace pa
