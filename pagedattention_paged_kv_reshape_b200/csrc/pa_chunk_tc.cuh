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
// * Q (one 3-D TMA box) and K, V (eight 16-token TMA boxes per 128-key tile;
//   a three-stage K ring and a two-stage V ring) land in shared memory with
//   128-byte swizzling, which is exactly the canonical K-major layout (Q, K,
//   P) and MN-major layout (V) the tcgen05 shared-memory descriptors describe;
// * one thread issues S = Q K^T (M=128, N=128, K=16 steps) into one of two
//   TMEM score buffers, two tiles ahead of the softmax, so the tensor core
//   computes the next scores while the softmax warps work;
// * four softmax warps read S with tcgen05.ld, one tile row per thread, apply
//   the causal mask (key <= position) and the online softmax in the log2
//   domain, and write P (rounded to the input type) to shared memory;
// * the same thread issues O_tile = P V into a second TMEM region; the
//   softmax threads fold it into their fp32 row accumulators with the
//   running rescale, and write the output row at the end.
//
// Every wait is bounded.  TMEM (512 columns) is freed on every path, after a
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

constexpr int kTcRows = 128;   // tile rows = TMEM lanes
constexpr int kTcKeys = 128;   // keys per KV tile = 8 blocks
constexpr int kTcKStages = 3;  // K ring: a K tile is free once its QK^T has run
constexpr int kTcVStages = 2;  // V ring: a V tile is free once its PV has run

template <int D>
struct TcLayout {
  static constexpr int kHalves = D / 64;           // 128-byte swizzle rows per token row
  static constexpr int kHalfBytes = 128 * 128;     // 128 rows x 128 B
  static constexpr int kQBytes = kHalves * kHalfBytes;
  static constexpr int kKVBytes = kHalves * kHalfBytes;  // one K or V tile
  static constexpr int kPBytes = 2 * kHalfBytes;   // 128 rows x 128 keys x 2 B
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kTcKStages * kKVBytes;
  static constexpr int kOffP = kOffV + kTcVStages * kKVBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  // qfull, qfree, kfull[3], kempty[3], vfull[2], vempty[2], sfull[2], pfull, pvfull, drain
  static constexpr int kNumBars = 2 + 2 * kTcKStages + 2 * kTcVStages + 2 + 3;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kBytes = kOffAbort + 12;
  // at least ~114 KB, so that a single CTA fits per SM and its TMEM
  // allocation can never wait for another CTA's
  static constexpr int kSmem = (kBytes + 1024) > 116 * 1024 ? (kBytes + 1024) : 116 * 1024;
  static constexpr int kThreads = 160;             // 4 softmax warps + 1 TMA/MMA warp
  static constexpr uint32_t kTmemCols = 512;       // S0 [0,128), S1 [128,256), O [256, 256 + D)
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0, "1 KB alignment");
  static_assert(kBytes + 1024 <= 232448, "shared memory budget");
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
  auto kfull = [&](int st) { return bar0 + 16u + 8u * st; };
  auto kempty = [&](int st) { return bar0 + 16u + 8u * (kTcKStages + st); };
  auto vfull = [&](int st) { return bar0 + 16u + 8u * (2 * kTcKStages + st); };
  auto vempty = [&](int st) { return bar0 + 16u + 8u * (2 * kTcKStages + kTcVStages + st); };
  auto sfull = [&](int b) { return bar0 + 16u + 8u * (2 * kTcKStages + 2 * kTcVStages + b); };
  const uint32_t pfull = bar0 + 16u + 8u * (2 * kTcKStages + 2 * kTcVStages + 2);
  const uint32_t pvfull = pfull + 8, drain = pfull + 16;
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
    for (int st = 0; st < kTcKStages; ++st) {
      mbar_init(kfull(st), 1);
      mbar_init(kempty(st), 1);
    }
    for (int st = 0; st < kTcVStages; ++st) {
      mbar_init(vfull(st), 1);
      mbar_init(vempty(st), 1);
    }
    mbar_init(sfull(0), 1);
    mbar_init(sfull(1), 1);
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
  auto t_s = [&](int b) { return tbase + static_cast<uint32_t>(b * kTcKeys); };  // S0, S1
  const uint32_t t_o = tbase + 2 * kTcKeys;

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
    // Tile t of the current item is this CTA's tile g + t: its K lands in K
    // stage (g+t) % 3, its V in V stage (g+t) % 2, its scores in S buffer
    // (g+t) % 2.  Steady state, per tile t: wait for P(t), issue PV(t), then
    // S(t+2) (its S buffer was freed by P(t)), then refill K and V stages.
    int g = 0;  // tiles of earlier items
    int k = 0;  // items so far
    bool ok = true;
    // One lane per 16-token block issues that block's TMA boxes, so the eight
    // blocks of a tile (16 boxes for K or V) go out in parallel instead of
    // one after another from a single thread.
    auto load_blocks = [&](const Item& it, int t, uint32_t dst, const CUtensorMap* map,
                           uint32_t bar) {
      const int first = t * (kTcKeys / kBlock);
      const int nb = min(kTcKeys / kBlock, ceil_div(it.kv_end, kBlock) - first);
      if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nb * L::kHalves * 2048));
      __syncwarp();
      if (lane < nb) {
        int pb = __ldg(block_tables + static_cast<size_t>(it.row) * s.table_stride + first + lane);
        if (pb < 0 || pb >= s.num_blocks) {
          report_error(PA_ERR_DEVICE_BOUNDS, kWhereBlockId, it.row, pb);
          pb = 0;
        }
        const int y = (pb * s.num_kv_heads + it.kvh) * kBlock;
#pragma unroll
        for (int h = 0; h < L::kHalves; ++h)
          tma_load_2d(dst + h * L::kHalfBytes + lane * 2048, map, bar, h * 64, y);
      }
      __syncwarp();
    };
    auto issue_k = [&](const Item& it, int t) -> bool {
      const int gt = g + t, st = gt % kTcKStages;
      bool r = true;
      if (lane == 0)
        r = mbar_wait(kempty(st), ((gt / kTcKStages) & 1) ^ 1, kWhereWaitEmpty, abort_flag);
      r = __shfl_sync(0xffffffffu, r, 0);
      if (r) load_blocks(it, t, k_smem(st), &tm_k, kfull(st));
      return r;
    };
    auto issue_v = [&](const Item& it, int t) -> bool {
      const int gt = g + t, st = gt % kTcVStages;
      bool r = true;
      if (lane == 0)
        r = mbar_wait(vempty(st), ((gt / kTcVStages) & 1) ^ 1, kWhereWaitEmpty, abort_flag);
      r = __shfl_sync(0xffffffffu, r, 0);
      if (r) load_blocks(it, t, v_smem(st), &tm_v, vfull(st));
      return r;
    };
    // S(t) = Q K(t)^T into S buffer (g+t) % 2.
    auto issue_s = [&](const Item& it, int t) -> bool {
      bool r = true;
      if (lane == 0) {
        const int gt = g + t, st = gt % kTcKStages;
        r = mbar_wait(kfull(st), (gt / kTcKStages) & 1, kWhereWaitFull, abort_flag);
        if (r) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kHalfBytes + (kk & 3) * 32;
            umma_ss(t_s(gt & 1), smem_desc_sw128(q_smem + off, 16, 1024),
                    smem_desc_sw128(k_smem(st) + off, 16, 1024), kIdescS, kk > 0);
          }
          umma_commit(sfull(gt & 1));
          umma_commit(kempty(st));
          if (t == it.nkt - 1) umma_commit(qfree);
        }
      }
      return __shfl_sync(0xffffffffu, r, 0);
    };
    // O_tile = P(t) V(t), once the softmax warps have written P(t).
    auto issue_pv = [&](const Item& it, int t) -> bool {
      const int gt = g + t, st = gt % kTcVStages;
      bool r = true;
      if (lane == 0) {
        r = mbar_wait(pfull, gt & 1, kWhereWaitMma, abort_flag) &&
            mbar_wait(vfull(st), (gt / kTcVStages) & 1, kWhereWaitFull, abort_flag);
      }
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
        for (int kk = 0; kk < kTcKeys / 16; ++kk) {
          umma_ss(t_o,
                  smem_desc_sw128(p_smem + (kk >> 2) * L::kHalfBytes + (kk & 3) * 32, 16, 1024),
                  smem_desc_sw128(v_smem(st) + kk * 2048, L::kHalfBytes, 1024), kIdescPV, kk > 0);
        }
        umma_commit(pvfull);
        umma_commit(vempty(st));
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
      for (int t = 0; t < min(kTcKStages, it.nkt) && ok; ++t) ok = issue_k(it, t);
      for (int t = 0; t < min(kTcVStages, it.nkt) && ok; ++t) ok = issue_v(it, t);
      if (ok && lane == 0) ok = mbar_wait(qfull, k & 1, kWhereWaitQ, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int t = 0; t < min(2, it.nkt) && ok; ++t) ok = issue_s(it, t);
      for (int t = 0; t < it.nkt && ok; ++t) {
        // K stage of tile t was freed by S(t), issued two steps ago: refill it
        // first so the load has the most time to land before S(t+3) needs it
        if (t + kTcKStages < it.nkt) ok = issue_k(it, t + kTcKStages);
        if (ok) ok = issue_pv(it, t);
        if (ok && t + 2 < it.nkt) ok = issue_s(it, t + 2);
        if (ok && t + kTcVStages < it.nkt) ok = issue_v(it, t + kTcVStages);
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
        const int gt = g + t;
        const uint32_t sb = t_s(gt & 1) + lane_base;  // this tile's S buffer, this warp's lanes
        ok = __all_sync(0xffffffffu,
                        mbar_wait(sfull(gt & 1), (gt >> 1) & 1, kWhereWaitMma, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int key0 = t * kTcKeys;
        float v[32];
        // pass 1: the row maximum of this tile (4 independent chains; the
        // causal mask is applied only to chunks that cross this row's limit)
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
        for (int c = 0; c < kTcKeys / 32; ++c) {
          tmem_ld32(sb + c * 32, v);
          const int kb = key0 + c * 32;
          if (kb + 32 <= lim) {
#pragma unroll
            for (int j = 0; j < 32; ++j) m4[j & 3] = fmaxf(m4[j & 3], v[j] * scale_log2);
          } else if (kb < lim) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (kb + j < lim) m4[j & 3] = fmaxf(m4[j & 3], v[j] * scale_log2);
          }
        }
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
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
        float ps4[4] = {0.f, 0.f, 0.f, 0.f};
        const float nmu = -mu;
#pragma unroll 1
        for (int c = 0; c < kTcKeys / 32; ++c) {
          tmem_ld32(sb + c * 32, v);
          const int kb = key0 + c * 32;
          uint32_t pk[16];
          if (kb + 32 <= lim) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[j] = pack2<T>(exp2f(fmaf(v[2 * j], scale_log2, nmu)),
                               exp2f(fmaf(v[2 * j + 1], scale_log2, nmu)));
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float p0 = kb + 2 * j < lim ? exp2f(fmaf(v[2 * j], scale_log2, nmu)) : 0.f;
              const float p1 =
                  kb + 2 * j + 1 < lim ? exp2f(fmaf(v[2 * j + 1], scale_log2, nmu)) : 0.f;
              pk[j] = pack2<T>(p0, p1);
            }
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {  // sum the same rounded weights P.V uses
            const float2 f = unpack2<T>(pk[j]);
            ps4[j & 3] += f.x + f.y;
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
        const float psum = (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
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
