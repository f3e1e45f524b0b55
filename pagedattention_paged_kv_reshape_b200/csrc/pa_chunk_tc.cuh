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
// * Q (one 3-D TMA box) and K, V (eight 16-token TMA boxes per 128-key tile,
//   in K and V rings) land in shared memory with 128-byte swizzling, which is
//   exactly the canonical K-major layout (Q, K, P) and MN-major layout (V) the
//   tcgen05 shared-memory descriptors describe;
// * one thread issues S = Q K^T (M=128, N=128, K=16 steps) into one of two
//   TMEM score buffers, two tiles ahead of the softmax, so the tensor core
//   computes the next scores while the softmax warps work;
// * four softmax warps read a tile's scores with one round of tcgen05.ld (a
//   whole 128-key row per thread), apply the causal mask (key <= position)
//   and the online softmax in the log2 domain, and write P (rounded to the
//   input type) into one of two shared-memory P buffers;
// * the same thread issues O += P V into a TMEM accumulator that lives for
//   the whole work item.  The running maximum that P is taken against is
//   raised only when a row's maximum grows by more than 2^8 (P then stays
//   below 256); only then is the row's O brought to the new reference point,
//   through TMEM, between two PV steps.  The epilogue reads O once and
//   divides by the row sum.
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

constexpr int kTcRows = 128;        // tile rows = TMEM lanes
constexpr int kTcKeys = 128;        // keys per KV tile = 8 blocks
constexpr int kTcVStages = 2;       // V ring: a V tile is free once its PV has run
constexpr float kTcRescale = 8.f;   // raise the reference maximum past this (log2 units)

template <int D>
struct TcLayout {
  // K ring: a K tile is free once its QK^T has run
  static constexpr int kKStages = D == 64 ? 3 : 2;
  static constexpr int kHalves = D / 64;           // 128-byte swizzle rows per token row
  static constexpr int kHalfBytes = 128 * 128;     // 128 rows x 128 B
  static constexpr int kQBytes = kHalves * kHalfBytes;
  static constexpr int kKVBytes = kHalves * kHalfBytes;  // one K or V tile
  static constexpr int kPBytes = 2 * kHalfBytes;   // one P buffer: 128 rows x 128 keys x 2 B
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffP = kOffV + kTcVStages * kKVBytes;
  static constexpr int kOffBar = kOffP + 2 * kPBytes;
  // barrier indexes: qfull, qfree, kfull[KS], kempty[KS], vfull[VS], vempty[VS],
  // sfull[2], pfull[2], pfree[2], drain
  static constexpr int kBarQFull = 0, kBarQFree = 1, kBarKFull = 2;
  static constexpr int kBarKEmpty = kBarKFull + kKStages;
  static constexpr int kBarVFull = kBarKEmpty + kKStages;
  static constexpr int kBarVEmpty = kBarVFull + kTcVStages;
  static constexpr int kBarSFull = kBarVEmpty + kTcVStages;
  static constexpr int kBarPFull = kBarSFull + 2;
  static constexpr int kBarPFree = kBarPFull + 2;
  static constexpr int kBarDrain = kBarPFree + 2;
  static constexpr int kNumBars = kBarDrain + 1;
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
  constexpr int KS = L::kKStages, VS = kTcVStages;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescS = instr_desc_f16(kBf16, false, false, kTcRows, kTcKeys);
  constexpr uint32_t kIdescPV = instr_desc_f16(kBf16, false, true, kTcRows, D);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + static_cast<uint32_t>(L::kOffBar + 8 * i); };
  const uint32_t qfull = bar(L::kBarQFull), qfree = bar(L::kBarQFree), drain = bar(L::kBarDrain);
  auto kfull = [&](int st) { return bar(L::kBarKFull + st); };
  auto kempty = [&](int st) { return bar(L::kBarKEmpty + st); };
  auto vfull = [&](int st) { return bar(L::kBarVFull + st); };
  auto vempty = [&](int st) { return bar(L::kBarVEmpty + st); };
  auto sfull = [&](int b) { return bar(L::kBarSFull + b); };  // S(b) written
  auto pfull = [&](int b) { return bar(L::kBarPFull + b); };  // P(b) written (4 warps)
  auto pfree = [&](int b) { return bar(L::kBarPFree + b); };  // PV from P(b) done
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  const uint32_t q_smem = sbase + L::kOffQ;
  auto k_smem = [&](int st) { return sbase + L::kOffK + st * L::kKVBytes; };
  auto v_smem = [&](int st) { return sbase + L::kOffV + st * L::kKVBytes; };
  auto p_smem = [&](int b) { return sbase + L::kOffP + b * L::kPBytes; };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i)  // P(b) is written by the four softmax warps
      mbar_init(bar(i), (i == L::kBarPFull || i == L::kBarPFull + 1) ? 4 : 1);
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
    // Tile t of the current item is this CTA's tile gt = g + t: its K lands
    // in K stage gt % KS, its V in V stage gt % VS, its scores in S buffer
    // gt % 2 and its P in P buffer gt % 2.  Steady state, per tile t: refill
    // the K stage S(t) has freed, wait for P(t), issue PV(t), then S(t+2)
    // (its S buffer was read before P(t) was written), then refill V.
    int g = 0;  // tiles of earlier items
    int k = 0;  // items so far
    bool ok = true;
    // One lane per 16-token block issues that block's TMA boxes, so the eight
    // blocks of a tile (16 boxes for K or V) go out in parallel instead of
    // one after another from a single thread.
    auto load_blocks = [&](const Item& it, int t, uint32_t dst, const CUtensorMap* map,
                           uint32_t bar_full) {
      const int first = t * (kTcKeys / kBlock);
      const int nb = min(kTcKeys / kBlock, ceil_div(it.kv_end, kBlock) - first);
      if (lane == 0)
        mbar_arrive_expect_tx(bar_full, static_cast<uint32_t>(nb * L::kHalves * 2048));
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
          tma_load_2d(dst + h * L::kHalfBytes + lane * 2048, map, bar_full, h * 64, y);
      }
      __syncwarp();
    };
    auto issue_k = [&](const Item& it, int t) -> bool {
      const int gt = g + t, st = gt % KS;
      bool r = true;
      if (lane == 0) r = mbar_wait(kempty(st), ((gt / KS) & 1) ^ 1, kWhereWaitEmpty, abort_flag);
      r = __shfl_sync(0xffffffffu, r, 0);
      if (r) load_blocks(it, t, k_smem(st), &tm_k, kfull(st));
      return r;
    };
    auto issue_v = [&](const Item& it, int t) -> bool {
      const int gt = g + t, st = gt % VS;
      bool r = true;
      if (lane == 0) r = mbar_wait(vempty(st), ((gt / VS) & 1) ^ 1, kWhereWaitEmpty, abort_flag);
      r = __shfl_sync(0xffffffffu, r, 0);
      if (r) load_blocks(it, t, v_smem(st), &tm_v, vfull(st));
      return r;
    };
    // S(t) = Q K(t)^T into S buffer gt % 2.
    auto issue_s = [&](const Item& it, int t) -> bool {
      bool r = true;
      if (lane == 0) {
        const int gt = g + t, st = gt % KS;
        r = mbar_wait(kfull(st), (gt / KS) & 1, kWhereWaitFull, abort_flag);
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
    // O (+)= P(t) V(t), once the softmax warps have written P(t) (and, where
    // a row's reference maximum moved, rescaled its O).
    auto issue_pv = [&](const Item& it, int t) -> bool {
      const int gt = g + t, st = gt % VS, b = gt & 1;
      bool r = true;
      if (lane == 0) {
        r = mbar_wait(pfull(b), (gt >> 1) & 1, kWhereWaitMma, abort_flag) &&
            mbar_wait(vfull(st), (gt / VS) & 1, kWhereWaitFull, abort_flag);
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
                  smem_desc_sw128(p_smem(b) + (kk >> 2) * L::kHalfBytes + (kk & 3) * 32, 16, 1024),
                  smem_desc_sw128(v_smem(st) + kk * 2048, L::kHalfBytes, 1024), kIdescPV,
                  (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(pfree(b));
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
      for (int t = 0; t < min(KS, it.nkt) && ok; ++t) ok = issue_k(it, t);
      for (int t = 0; t < min(VS, it.nkt) && ok; ++t) ok = issue_v(it, t);
      if (ok && lane == 0) ok = mbar_wait(qfull, k & 1, kWhereWaitQ, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int t = 0; t < min(2, it.nkt) && ok; ++t) ok = issue_s(it, t);
      for (int t = 0; t < it.nkt && ok; ++t) {
        if (t + KS < it.nkt) ok = issue_k(it, t + KS);  // into the stage S(t) has freed
        if (ok) ok = issue_pv(it, t);
        if (ok && t + 2 < it.nkt) ok = issue_s(it, t + 2);
        if (ok && t + VS < it.nkt) ok = issue_v(it, t + VS);
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
    // Scores enter as x = s * |scale| after a sign flip of s for a negative
    // scale, so that the row maximum is always a max.
    const bool neg = scale_log2 < 0.f;
    const float sc = fabsf(scale_log2);
    int g = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
      const Item it = load_item(item);
      const int i = r / s.gs, gi = r % s.gs;
      const bool valid = i < it.nq && gi < it.rows;
      const int lim = it.pos0 + i + 1;  // keys visible to this row
      float m = -INFINITY;              // reference maximum P is taken against (log2 units)
      float l = 0.f;                    // sum of P against that reference
      for (int t = 0; t < it.nkt && ok; ++t) {
        const int gt = g + t, b = gt & 1;
        // scores of this tile, and P buffer b free (PV two tiles back done)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(sfull(b), (gt >> 1) & 1, kWhereWaitMma, abort_flag) &&
                            mbar_wait(pfree(b), ((gt >> 1) & 1) ^ 1, kWhereWaitMma, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t ra[64], rb[64];
        tmem_ld64_issue(t_s(b) + lane_base, ra);
        tmem_ld64_issue(t_s(b) + lane_base + 64, rb);
        tmem_ld_wait(ra);
        reg_tie(rb);
        float x[kTcKeys];
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          x[j] = __uint_as_float(ra[j]);
          x[64 + j] = __uint_as_float(rb[j]);
        }
        if (neg) {
#pragma unroll
          for (int j = 0; j < kTcKeys; ++j) x[j] = -x[j];
        }
        const int nvis = lim - t * kTcKeys;  // keys of this tile this row may see
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (nvis >= kTcKeys) {
#pragma unroll
          for (int j = 0; j < kTcKeys; ++j) m4[j & 3] = fmaxf(m4[j & 3], x[j]);
        } else {
#pragma unroll
          for (int j = 0; j < kTcKeys; ++j)
            if (j < nvis) m4[j & 3] = fmaxf(m4[j & 3], x[j]);
        }
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sc;
        // raise the reference maximum only when the row maximum has grown by
        // more than 2^kTcRescale (always on the first visible keys)
        const bool raise = mx > m + kTcRescale;
        float alpha = 1.f;
        if (raise) {
          alpha = ex2_approx(m - mx);  // 0 when m = -inf
          m = mx;
        }
        if (t > 0 && __any_sync(0xffffffffu, raise)) {
          // O holds PV of tiles 0 .. t-1: once PV(t-1) is done, scale it
          ok = __all_sync(0xffffffffu, mbar_wait(pfree((gt - 1) & 1), ((gt - 1) >> 1) & 1,
                                                 kWhereWaitMma, abort_flag));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 64; ++c) {
            uint32_t ro[64];
            tmem_ld64_issue(t_o + lane_base + c * 64, ro);
            tmem_ld_wait(ro);
#pragma unroll
            for (int j = 0; j < 64; ++j) ro[j] = __float_as_uint(__uint_as_float(ro[j]) * alpha);
            tmem_st64(t_o + lane_base + c * 64, ro);
          }
          tmem_st_wait();
        }
        l *= alpha;
        // P = 2^(x - m), rounded to the input type, into P buffer b
        const float nm = m == -INFINITY ? 0.f : -m;
        float ps4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[kTcKeys / 2];
        if (nvis >= kTcKeys) {
#pragma unroll
          for (int j = 0; j < kTcKeys / 2; ++j) {
            const float p0 = ex2_approx(fmaf(x[2 * j], sc, nm));
            const float p1 = ex2_approx(fmaf(x[2 * j + 1], sc, nm));
            ps4[j & 3] += p0 + p1;
            pk[j] = pack2<T>(p0, p1);
          }
        } else {
#pragma unroll
          for (int j = 0; j < kTcKeys / 2; ++j) {
            const float p0 = 2 * j < nvis ? ex2_approx(fmaf(x[2 * j], sc, nm)) : 0.f;
            const float p1 = 2 * j + 1 < nvis ? ex2_approx(fmaf(x[2 * j + 1], sc, nm)) : 0.f;
            ps4[j & 3] += p0 + p1;
            pk[j] = pack2<T>(p0, p1);
          }
        }
        // keys 64c .. 64c+63 are one 128-byte row of P half c
        const uint32_t prow = L::kOffP + b * L::kPBytes + r * 128;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int q8 = 0; q8 < 8; ++q8) {
            const int j = c * 32 + q8 * 4;
            *reinterpret_cast<uint4*>(smem + prow + c * L::kHalfBytes + ((q8 ^ (r & 7)) << 4)) =
                make_uint4(pk[j], pk[j + 1], pk[j + 2], pk[j + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull(b));
        l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
      }
      if (ok) {
        // the item's last PV done: O is final
        const int gl = g + it.nkt - 1;
        ok = __all_sync(0xffffffffu, mbar_wait(pfree(gl & 1), (gl >> 1) & 1, kWhereWaitMma,
                                               abort_flag));
        if (ok) {
          tc_fence_after();
          const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
          for (int c = 0; c < D / 64; ++c) {
            uint32_t ro[64];
            tmem_ld64_issue(t_o + lane_base + c * 64, ro);
            tmem_ld_wait(ro);
            if (valid) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                float a[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(ro[q * 8 + e]);
                store_row8<T, D>(s, out, it.token0 + i, it.head0 + gi, c * 8 + q, a, inv);
              }
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
