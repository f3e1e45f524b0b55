// Causal prefill-chunk attention on tcgen05 tensor cores with TMEM accumulators.
//
// A chunk row of a mixed batch ("vLLM 深度拆解" §4.3 chunked prefill;
// "vLLM 架构源码解析" §3.2 / §3.3.2) has q_len query tokens at positions
// seq_len - q_len + i over a cached context.  Its QK^T and PV are dense
// contractions, so they run here on 128-row tiles instead of the decode
// kernel's 16-row tiles:
//
// * work item = (chunk row, tile of 128/gs query tokens x gs query heads =
//   128 tile rows, KV head slice); a persistent grid walks the items listed
//   by the prep kernel;
// * Q (one 3-D TMA box) and K/V (eight 16-token TMA boxes per 128-key tile,
//   a two-stage ring) land in shared memory with 128-byte swizzling, which is
//   exactly the canonical K-major layout (Q, K, P) and MN-major layout (V) the
//   tcgen05 shared-memory descriptors describe;
// * one thread issues S = Q K^T (M=128, N=128, K=16 steps) into TMEM;
// * four softmax warps read S with tcgen05.ld, one tile row per thread, apply
//   the causal mask (key <= position) and the online softmax in the log2
//   domain, and write P (rounded to the input type) to shared memory;
// * the same thread issues O_tile = P V into a second TMEM region; the
//   softmax threads fold it into their fp32 row accumulators with the
//   running rescale, and write the output row at the end.
//
// Every wait is bounded.  TMEM (256 columns) is freed on every path, after a
// final commit has drained the MMAs this CTA issued.  The kernel is launched
// behind the decode kernel with programmatic dependent launch so that it
// fills that kernel's tail; it reads nothing the decode kernel writes, and it
// waits for that grid before exiting so that a later kernel waiting for this
// grid has both complete.
#pragma once

#include <type_traits>

#include "pa_sched.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

constexpr int kTcRows = 128;  // tile rows = TMEM lanes
constexpr int kTcKeys = 128;  // keys per KV tile = 8 blocks
constexpr int kTcStages = 2;

template <int D>
struct TcLayout {
  static constexpr int kHalves = D / 64;           // 128-byte swizzle rows per token row
  static constexpr int kHalfBytes = 128 * 128;     // 128 rows x 128 B
  static constexpr int kQBytes = kHalves * kHalfBytes;
  static constexpr int kKVBytes = kHalves * kHalfBytes;
  static constexpr int kPBytes = 2 * kHalfBytes;   // 128 rows x 128 keys x 2 B
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kTcStages * kKVBytes;
  static constexpr int kOffP = kOffV + kTcStages * kKVBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  // qfull, qfree, kvfull[2], kvempty[2], sfull, pfull, pvfull, drain
  static constexpr int kNumBars = 10;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kBytes = kOffAbort + 12;
  static constexpr int kSmem = kBytes + 1024;
  static constexpr int kThreads = 160;             // 4 softmax warps + 1 TMA/MMA warp
  static constexpr uint32_t kTmemCols = 256;       // S in [0,128), O in [128, 128 + D)
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0, "1 KB alignment");
};

template <typename T, int D>
__global__ void __launch_bounds__(160, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, Shape s, T* __restrict__ out,
                    const int* __restrict__ block_tables, const int* __restrict__ qsl,
                    const int* __restrict__ seq_lens, Work w, float scale_log2) {
  using L = TcLayout<D>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescS = instr_desc_f16(kBf16, false, false, kTcRows, kTcKeys);
  constexpr uint32_t kIdescPV = instr_desc_f16(kBf16, false, true, kTcRows, D);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kOffBar;
  const uint32_t qfull = bar0, qfree = bar0 + 8;
  auto kvfull = [&](int st) { return bar0 + 16u + 8u * st; };
  auto kvempty = [&](int st) { return bar0 + 32u + 8u * st; };
  const uint32_t sfull = bar0 + 48, pfull = bar0 + 56, pvfull = bar0 + 64, drain = bar0 + 72;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  const uint32_t q_smem = sbase + L::kOffQ;
  const uint32_t p_smem = sbase + L::kOffP;
  auto k_smem = [&](int st) { return sbase + L::kOffK + st * L::kKVBytes; };
  auto v_smem = [&](int st) { return sbase + L::kOffV + st * L::kKVBytes; };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    mbar_init(qfull, 1);
    mbar_init(qfree, 1);
    for (int st = 0; st < kTcStages; ++st) {
      mbar_init(kvfull(st), 1);
      mbar_init(kvempty(st), 1);
    }
    mbar_init(sfull, 1);
    mbar_init(pfull, 4);
    mbar_init(pvfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(sbase + L::kOffTmem, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_s = tbase;
  const uint32_t t_o = tbase + kTcKeys;

  const int count = __ldcg(&w.sched->chunk_count);
  const int hun = head_units(s);
  const int items = count * hun;
  const int qt = kTcRows / s.gs;

  // Everything about one item, computed identically by every thread.
  struct Item {
    int row, token0, nq, kvh, head0, rows, pos0, kv_end, nkt;
  };
  auto load_item = [&](int item) {
    Item it;
    const int e = item % count;
    const int hu = item / count;
    const int2 ent = __ldcg(w.chunk_list + e);
    const RowInfo ri = load_row(s, qsl, seq_lens, ent.x);
    it.row = ent.x;
    it.kvh = hu / s.ns;
    const int slice = hu % s.ns;
    it.head0 = it.kvh * s.group + slice * 16;
    it.rows = min(s.gs, s.group - slice * 16);
    it.nq = min(qt, ri.q_len - ent.y);
    it.token0 = ri.token0 + ent.y;
    it.pos0 = ri.seq_len - ri.q_len + ent.y;
    it.kv_end = it.pos0 + it.nq;
    it.nkt = ceil_div(it.kv_end, kTcKeys);
    return it;
  };

  if (warp == 4) {
    // ------------------------------------------------ TMA loads + MMA issue
    int g = 0;  // KV tiles issued so far by this CTA (stage ring position)
    int k = 0;  // items so far
    bool ok = true;
    // K/V tile t of `it` into stage (g + t) % 2: eight 16-token blocks.
    auto issue_kv = [&](const Item& it, int t) -> bool {
      bool r = true;
      if (lane == 0) {
        const int gt = g + t;
        const int st = gt % kTcStages;
        r = mbar_wait(kvempty(st), ((gt / kTcStages) & 1) ^ 1, kWhereWaitEmpty, abort_flag);
        if (r) {
          const int first = t * (kTcKeys / kBlock);
          const int nb = min(kTcKeys / kBlock, ceil_div(it.kv_end, kBlock) - first);
          mbar_arrive_expect_tx(kvfull(st), static_cast<uint32_t>(nb * 2 * L::kHalves * 2048));
          const int* table = block_tables + static_cast<size_t>(it.row) * s.table_stride + first;
          for (int b = 0; b < nb; ++b) {
            int pb = __ldg(table + b);
            if (pb < 0 || pb >= s.num_blocks) {
              report_error(PA_ERR_DEVICE_BOUNDS, kWhereBlockId, it.row, pb);
              pb = 0;
            }
            const int y = (pb * s.num_kv_heads + it.kvh) * kBlock;
#pragma unroll
            for (int h = 0; h < L::kHalves; ++h) {
              tma_load_2d(k_smem(st) + h * L::kHalfBytes + b * 2048, &tm_k, kvfull(st), h * 64, y);
              tma_load_2d(v_smem(st) + h * L::kHalfBytes + b * 2048, &tm_v, kvfull(st), h * 64, y);
            }
          }
        }
      }
      return __shfl_sync(0xffffffffu, r, 0);
    };
    // Wait for tile t, zero V rows past the item's last key, issue S = Q K^T.
    auto issue_s = [&](const Item& it, int t) -> bool {
      const int gt = g + t;
      const int st = gt % kTcStages;
      bool r = true;
      if (lane == 0) r = mbar_wait(kvfull(st), (gt / kTcStages) & 1, kWhereWaitFull, abort_flag);
      r = __shfl_sync(0xffffffffu, r, 0);
      if (!r) return false;
      const int valid = it.kv_end - t * kTcKeys;  // keys of this tile that exist
      if (valid < kTcKeys) {
        // padding rows may hold anything (NaN included), and 0 * NaN is NaN
        const int nchunks = (kTcKeys - valid) * L::kHalves * 8;
        for (int c = lane; c < nchunks; c += 32) {
          const int row = valid + c / (L::kHalves * 8);
          const int h = (c / 8) % L::kHalves;
          const int ch = c % 8;
          *reinterpret_cast<uint4*>(smem + L::kOffV + st * L::kKVBytes + h * L::kHalfBytes +
                                    row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kHalfBytes + (kk & 3) * 32;
          umma_ss(t_s, smem_desc_sw128(q_smem + off, 16, 1024),
                  smem_desc_sw128(k_smem(st) + off, 16, 1024), kIdescS, kk > 0);
        }
        umma_commit(sfull);
        if (t == it.nkt - 1) umma_commit(qfree);
      }
      return true;
    };
    for (int item = blockIdx.x; item < items && ok; item += gridDim.x, ++k) {
      const Item it = load_item(item);
      if (lane == 0) {
        if (k > 0) ok = mbar_wait(qfree, (k - 1) & 1, kWhereWaitQ, abort_flag);
        if (ok) {
          mbar_arrive_expect_tx(qfull, static_cast<uint32_t>(L::kQBytes));
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_3d(q_smem + h * L::kHalfBytes, &tm_q, qfull, h * 64, it.head0, it.token0);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int t = 0; t < min(kTcStages, it.nkt) && ok; ++t) ok = issue_kv(it, t);
      if (ok && lane == 0) ok = mbar_wait(qfull, k & 1, kWhereWaitQ, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) ok = issue_s(it, 0);
      for (int t = 0; t < it.nkt && ok; ++t) {
        const int st = (g + t) % kTcStages;
        if (lane == 0) {
          ok = mbar_wait(pfull, (g + t) & 1, kWhereWaitMma, abort_flag);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kTcKeys / 16; ++kk) {
              umma_ss(t_o,
                      smem_desc_sw128(p_smem + (kk >> 2) * L::kHalfBytes + (kk & 3) * 32, 16, 1024),
                      smem_desc_sw128(v_smem(st) + kk * 2048, L::kHalfBytes, 1024), kIdescPV,
                      kk > 0);
            }
            umma_commit(pvfull);
            umma_commit(kvempty(st));
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok && t + 1 < it.nkt) ok = issue_s(it, t + 1);
        if (ok && t + kTcStages < it.nkt) ok = issue_kv(it, t + kTcStages);
      }
      g += it.nkt;
    }
    if (lane == 0) {  // no MMA of this CTA may still run when TMEM is freed
      umma_commit(drain);
      volatile int own_flag = 0;
      mbar_wait(drain, 0, kWhereWaitMma, &own_flag);
    }
  } else {
    // ------------------------------------------------------- softmax warps
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int r = tid;  // tile row = TMEM lane
    int g = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
      const Item it = load_item(item);
      const int i = r / s.gs, gi = r % s.gs;
      const bool valid = i < it.nq && gi < it.rows;
      const int lim = it.pos0 + i + 1;  // keys visible to this row
      float o[D];
#pragma unroll
      for (int d = 0; d < D; ++d) o[d] = 0.f;
      float m = -INFINITY, l = 0.f, alpha_prev = 1.f;
      for (int t = 0; t < it.nkt && ok; ++t) {
        ok = __all_sync(0xffffffffu, mbar_wait(sfull, (g + t) & 1, kWhereWaitMma, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int key0 = t * kTcKeys;
        float v[32];
        // pass 1: the row maximum of this tile
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < kTcKeys / 32; ++c) {
          tmem_ld32(t_s + lane_base + c * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            mx = fmaxf(mx, key0 + c * 32 + j < lim ? v[j] * scale_log2 : -INFINITY);
        }
        const float mn = fmaxf(m, mx);
        const float mu = mn == -INFINITY ? 0.f : mn;
        const float alpha = exp2f(m - mu);
        // the previous tile's P V: fold it in, which also frees P and O
        if (t > 0) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(pvfull, (g + t - 1) & 1, kWhereWaitMma, abort_flag));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(t_o + lane_base + c * 32, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) o[c * 32 + j] = fmaf(o[c * 32 + j], alpha_prev, v[j]);
          }
        }
        // pass 2: P = 2^(x - m), rounded to the input type, into shared memory
        float psum = 0.f;
#pragma unroll 1
        for (int c = 0; c < kTcKeys / 32; ++c) {
          tmem_ld32(t_s + lane_base + c * 32, v);
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int key = key0 + c * 32 + 2 * j;
            const float x0 = key < lim ? v[2 * j] * scale_log2 : -INFINITY;
            const float x1 = key + 1 < lim ? v[2 * j + 1] * scale_log2 : -INFINITY;
            pk[j] = pack2<T>(exp2f(x0 - mu), exp2f(x1 - mu));
            const float2 f = unpack2<T>(pk[j]);
            psum += f.x + f.y;
          }
          const int half = c >> 1;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int ch = (c & 1) * 4 + q4;  // 16-byte chunk within the 128-byte row
            *reinterpret_cast<uint4*>(smem + L::kOffP + half * L::kHalfBytes + r * 128 +
                                      ((ch ^ (r & 7)) << 4)) =
                make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull);
        l = l * alpha + psum;
        m = mn;
        alpha_prev = alpha;
      }
      if (ok && it.nkt > 0) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(pvfull, (g + it.nkt - 1) & 1, kWhereWaitMma, abort_flag));
        if (ok) {
          tc_fence_after();
          float v[32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(t_o + lane_base + c * 32, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) o[c * 32 + j] = fmaf(o[c * 32 + j], alpha_prev, v[j]);
          }
          if (valid) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
              float a[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) a[e] = o[c * 8 + e];
              store_row8<T, D>(s, out, it.token0 + i, it.head0 + gi, c, a, inv);
            }
          }
        }
      }
      g += it.nkt;
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, L::kTmemCols);
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace pa
