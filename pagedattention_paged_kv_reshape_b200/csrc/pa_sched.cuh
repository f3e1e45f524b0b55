// Work decomposition shared by the attention kernels, and the epilogue that
// merges online-softmax states (across warps, then across split-K partitions).
//
// A batch is a list of rows (requests).  Row r has q_len query tokens (1 for
// a decode row) at positions seq_len - q_len + i ("vLLM 架构源码解析" §3.3.2:
// positions run from num_computed_tokens); query i reads keys 0 .. position.
//
// Work unit = (row, query tile, KV head slice, partition):
//   * query tile  : up to `qpt` consecutive query tokens of the row;
//   * head slice  : up to 16 query heads of one KV head (a whole GQA group
//                   when it has <= 16 heads), so each KV block is streamed
//                   once per KV head and tile;
//   * partition   : keys [p*512, (p+1)*512), the split-K unit.
// Tile rows are (query token, head) pairs, row = i * gs + g, at most 16.
//
// Units come in two classes so the longest go first: class A holds every
// partition but a row's last (always 512 keys), class B the last partitions.
// A one-CTA prep kernel validates the rows and writes prefix sums of both
// classes; CTAs of the attention kernel claim unit indices from an atomic
// counter, so the short tail units are spread over whichever CTAs free up.
//
// When a tile's keys span several partitions, each unit writes its rows'
// partial state (normalised o and log2-sum-exp) to the workspace and
// reduce_kernel merges them by log-sum-exp.  (Merging inside the attention
// kernel, by the last unit of each tile, was measured slower: the merge
// stalls that CTA's consumer warps while the stage ring drains.)
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
  int block_size;   // tokens per physical block: 8, 16 or 32
  int num_blocks;
  int max_seq_len;  // host bound on seq_lens / context_lens
  int max_query_len;
  int total_q;
  int p_stride;     // partitions per (token, head) in the workspace
  int chunk_qt;     // > 0: rows with q_len >= chunk_qt go to the tcgen05 chunk kernel
                    // as tiles of chunk_qt query tokens (128 / gs)
  int chunk_cap;    // capacity of the chunk-tile list
  int chunk_span;   // query tokens per chunk-list entry: chunk_qt, or 2 chunk_qt when
                    // the chunk kernel takes two tiles per item
};

// Schedule block at the start of the workspace.
struct Sched {
  int next;         // next unit index to claim
  int total_a;      // class-A units
  int total_b;      // class-B units
  int chunk_count;  // entries of the chunk-tile list
};

// Pointers into the workspace.
struct Work {
  Sched* sched;
  int* row_a;       // [num_seqs + 1] prefix of class-A units
  int* row_b;       // [num_seqs + 1] prefix of class-B units
  int2* chunk_list; // (row, first query) of every tcgen05 chunk tile
  float* part_lse;  // [total_q][Hq][p_stride]
  float* part_o;    // [total_q][Hq][p_stride][D]
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
          ri.seq_len <= s.table_stride * s.block_size && ri.q_len >= 0 &&
          ri.q_len <= ri.seq_len && ri.token0 >= 0 && ri.token0 + ri.q_len <= s.total_q &&
          (qsl == nullptr || ri.q_len <= s.max_query_len);
  return ri;
}

__device__ __forceinline__ int head_units(const Shape& s) { return s.num_kv_heads * s.ns; }

// Units of each class in a row.
__device__ __forceinline__ bool is_chunk_row(const Shape& s, const RowInfo& ri) {
  return s.chunk_qt > 0 && ri.q_len >= s.chunk_qt;
}

__device__ __forceinline__ void row_units(const Shape& s, const RowInfo& ri, int& a, int& b) {
  a = b = 0;
  if (!ri.ok || ri.q_len == 0 || is_chunk_row(s, ri)) return;
  const int items = ceil_div(ri.q_len, s.qpt);
  const int parts = ceil_div(ri.seq_len, kPart);
  b = items * head_units(s);
  a = b * (parts - 1);
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

// Decode the unit at offset `local` of class `cls` inside row `row`.  Inside a
// row the query tile varies fastest, so consecutive units of a prefill chunk
// read the same KV blocks while they are in L2.
__device__ __forceinline__ Unit decode_unit(const Shape& s, const RowInfo& ri, int row,
                                            int local, int cls) {
  Unit u;
  const int items = ceil_div(ri.q_len, s.qpt);
  const int parts = ceil_div(ri.seq_len, kPart);
  const int item = local % items;
  const int rest = local / items;
  int hu;
  if (cls == 0) {
    u.p = rest % (parts - 1);
    hu = rest / (parts - 1);
  } else {
    u.p = parts - 1;
    hu = rest;
  }
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

// Number of partitions holding keys visible to a query that sees `limit` keys
// (1 = its output is written directly, without partials).
__device__ __forceinline__ int parts_for(int limit) { return ceil_div(limit, kPart); }

// Largest r with row_start[r] <= u, scanning forward from `cursor` one warp
// (32 rows) at a time.  All lanes of the warp call it; returns the row and its
// row_start.  Requires row_start non-decreasing and u < row_start[num_seqs].
__device__ __forceinline__ int find_row_warp(const int* __restrict__ row_start, int num_seqs,
                                             int u, int cursor, int& start) {
  const int lane = threadIdx.x & 31;
  while (true) {
    const int idx = cursor + lane;
    const int v = idx <= num_seqs ? __ldcg(row_start + idx) : 0x7fffffff;
    const unsigned m = __ballot_sync(0xffffffffu, v <= u);
    const int cnt = __popc(m);
    if (cnt < 32) {
      start = __shfl_sync(0xffffffffu, v, cnt - 1);
      return cursor + cnt - 1;
    }
    cursor += 31;
  }
}

// Same, binary search, one thread.
__device__ __forceinline__ int find_row_thread(const int* __restrict__ row_start, int num_seqs,
                                               int u) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldcg(row_start + mid) <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// Map a claimed unit index to (row, local offset, class); class-A units come
// first.  Warp form: forward scans from the caller's cursors.
__device__ __forceinline__ int locate_unit_warp(const Shape& s, const Work& w, int total_a, int u,
                                                int& cur_a, int& cur_b, int& local, int& cls) {
  int start;
  int row;
  if (u < total_a) {
    cls = 0;
    row = find_row_warp(w.row_a, s.num_seqs, u, cur_a, start);
    cur_a = row;
    local = u - start;
  } else {
    cls = 1;
    const int ub = u - total_a;
    row = find_row_warp(w.row_b, s.num_seqs, ub, cur_b, start);
    cur_b = row;
    local = ub - start;
  }
  return row;
}

// Thread form: binary search.
__device__ __forceinline__ int locate_unit_thread(const Shape& s, const Work& w, int total_a,
                                                  int u, int& local, int& cls) {
  int row;
  if (u < total_a) {
    cls = 0;
    row = find_row_thread(w.row_a, s.num_seqs, u);
    local = u - __ldcg(w.row_a + row);
  } else {
    cls = 1;
    const int ub = u - total_a;
    row = find_row_thread(w.row_b, s.num_seqs, ub);
    local = ub - __ldcg(w.row_b + row);
  }
  return row;
}

// ---------------------------------------------------------------------------
// Prep kernel: validate rows, write the two prefix sums and the totals, zero
// the claim counter, list the tiles of chunk rows for the tcgen05 kernel,
// zero the output rows of empty decode requests.  One CTA of 1024 threads.  It lets the attention kernel
// launch at once (programmatic dependent launch); that kernel waits for this
// grid to complete before it reads any of the above.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(1024) schedule_kernel(Shape s, const int* __restrict__ qsl,
                                                        const int* __restrict__ seq_lens,
                                                        Work w, T* __restrict__ out) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // launched behind the cache write with programmatic dependent launch: the
  // workspace and the rows are touched only after the previous grid is done
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ int warp_tot[2][32];
  __shared__ int carry_s[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry_s[0] = carry_s[1] = 0;
    w.sched->chunk_count = 0;
    if (qsl && (qsl[0] != 0 || qsl[s.num_seqs] != s.total_q))
      report_error(PA_ERR_DEVICE_BOUNDS, kWhereRowMeta, -1, qsl[s.num_seqs]);
  }
  __syncthreads();
  for (int base = 0; base < s.num_seqs; base += 1024) {
    const int r = base + tid;
    int va = 0, vb = 0;
    if (r < s.num_seqs) {
      const RowInfo ri = load_row(s, qsl, seq_lens, r);
      if (!ri.ok) report_error(PA_ERR_DEVICE_BOUNDS, kWhereRowMeta, r, ri.seq_len);
      row_units(s, ri, va, vb);
      if (ri.ok && is_chunk_row(s, ri)) {
        const int n = ceil_div(ri.q_len, s.chunk_span);
        const int at = atomicAdd(&w.sched->chunk_count, n);
        if (at + n <= s.chunk_cap) {
          for (int j = 0; j < n; ++j) w.chunk_list[at + j] = make_int2(r, j * s.chunk_span);
        } else {  // rows overlap in query_start_loc: more tiles than tokens allow
          report_error(PA_ERR_DEVICE_BOUNDS, kWhereRowMeta, r, at + n);
        }
      }
      if (ri.ok && qsl == nullptr && ri.seq_len == 0) {
        T* o = out + static_cast<size_t>(r) * s.num_q_heads * s.head_dim;
        for (int i = 0; i < s.num_q_heads * s.head_dim; ++i) o[i] = from_f32<T>(0.f);
      }
    }
    int xa = va, xb = vb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, xa, o);
      const int yb = __shfl_up_sync(0xffffffffu, xb, o);
      if (lane >= o) {
        xa += ya;
        xb += yb;
      }
    }
    if (lane == 31) {
      warp_tot[0][warp] = xa;
      warp_tot[1][warp] = xb;
    }
    __syncthreads();
    if (warp < 2) {
      int t = warp_tot[warp][lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_tot[warp][lane] = t;
    }
    __syncthreads();
    const int ea = carry_s[0] + xa - va + (warp > 0 ? warp_tot[0][warp - 1] : 0);
    const int eb = carry_s[1] + xb - vb + (warp > 0 ? warp_tot[1][warp - 1] : 0);
    if (r < s.num_seqs) {
      w.row_a[r] = ea;
      w.row_b[r] = eb;
    }
    __syncthreads();
    if (tid == 1023) {
      carry_s[0] = ea + va;
      carry_s[1] = eb + vb;
    }
    __syncthreads();
  }
  if (tid == 0) {
    w.row_a[s.num_seqs] = carry_s[0];
    w.row_b[s.num_seqs] = carry_s[1];
    w.sched->next = 0;
    w.sched->total_a = carry_s[0];
    w.sched->total_b = carry_s[1];
  }
  __syncthreads();
  if (tid == 0 && w.sched->chunk_count > s.chunk_cap) w.sched->chunk_count = s.chunk_cap;
}

// ---------------------------------------------------------------------------
// Epilogue of one unit, run by the `nthreads` consumer threads of a CTA: merge
// NW warps' states per tile row (cm/cl: running max in log2 units and sum; co:
// unnormalised accumulators) and write the output row directly if its keys fit
// one partition, else this partition's partial (normalised o, log2-sum-exp).
// ---------------------------------------------------------------------------
template <typename T, int D>
__device__ __forceinline__ void store_row8(const Shape& s, T* __restrict__ out, int token,
                                           int head, int c, const float (&acc)[8], float inv) {
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
}

// Float offset, inside a merge-buffer row, of the 4-float chunk `ch` (dims
// 4ch .. 4ch+3) in the swizzled layout: within each run of 8 chunks (32 dims)
// the chunk index is XORed with 0, 4, 1, 5 for runs 0..3.  A warp whose lanes
// (g, q) hold dims 32q .. 32q+31 of rows g and g+8 then stores its run
// conflict-free with float4 stores at a row stride of D + 8 floats.
__device__ __forceinline__ int co_swizzled(int ch) {
  const int run = ch >> 3;
  const int x = ((run & 1) << 2) | ((run >> 1) & 1);
  return 4 * ((ch & ~7) | ((ch & 7) ^ x));
}

template <typename T, int D, int NW, bool kSwizzledCo = false, int CR = kRows>
__device__ __forceinline__ void epilogue(const Shape& s, const Unit& u, const float* cm,
                                         const float* cl, const float (*co)[CR][D + 8],
                                         T* __restrict__ out, const Work& w, int tid,
                                         int nthreads) {
  static_assert(!kSwizzledCo || D <= 128, "the swizzle covers four runs of 32 dims");
  constexpr int kChunks = D / 8;
  for (int task = tid; task < CR * kChunks; task += nthreads) {
    const int r = task / kChunks, c = task % kChunks;
    const int i = r / s.gs, g = r % s.gs;
    if (i >= u.nq || g >= u.rows) continue;
    const int parts = parts_for(u.lim0 + i);
    if (u.p >= parts) continue;  // no key of this partition is visible to the row
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < NW; ++q) mx = fmaxf(mx, cm[q * CR + r]);
    float L = 0.f;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int q = 0; q < NW; ++q) {
      const float f = exp2f(cm[q * CR + r] - mx);
      L += f * cl[q * CR + r];
      const int oa = kSwizzledCo ? co_swizzled(2 * c) : c * 8;
      const int ob = kSwizzledCo ? co_swizzled(2 * c + 1) : c * 8 + 4;
      const float4 a = *reinterpret_cast<const float4*>(&co[q][r][oa]);
      const float4 b = *reinterpret_cast<const float4*>(&co[q][r][ob]);
      acc[0] += f * a.x; acc[1] += f * a.y; acc[2] += f * a.z; acc[3] += f * a.w;
      acc[4] += f * b.x; acc[5] += f * b.y; acc[6] += f * b.z; acc[7] += f * b.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int token = u.token0 + i;
    const int head = u.head0 + g;
    if (parts == 1) {
      store_row8<T, D>(s, out, token, head, c, acc, inv);
    } else {
      const size_t slot = (static_cast<size_t>(token) * s.num_q_heads + head) * s.p_stride + u.p;
      float* po = w.part_o + slot * D + c * 8;
      *reinterpret_cast<float4*>(po) =
          make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      *reinterpret_cast<float4*>(po + 4) =
          make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      if (c == 0) w.part_lse[slot] = L > 0.f ? mx + log2f(L) : -INFINITY;
    }
  }
}

}  // namespace pa
