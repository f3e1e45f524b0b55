// Causal prefill-chunk attention on tcgen05: two query tiles share every K/V
// tile, and the next scores are computed while the softmax runs.
//
// The chunk rows of a mixed batch ("vLLM 深度拆解" §4.3 chunked prefill;
// "vLLM 架构源码解析" §3.2 / §3.3.2) are split into work items of TWO
// consecutive 128-row query tiles (A: query tokens q0 .. q0+qt-1, B: the next
// qt) of one row and KV-head slice.  Every 64-key K and V tile the load warp
// brings in serves both tiles, so the bytes a CTA pulls through L2 per FLOP
// are half of a one-tile kernel's.
//
// * TMEM (512 columns): S_A [0,64), S_B [64,128), P_A0, P_A1, P_B0, P_B1
//   [128,256) (32 columns each, 16-bit pairs), O_A [256, 256+D), O_B
//   [384, 384+D).  P is double-buffered per tile: the softmax writes P(t+1)
//   while PV(t) reads P(t).
// * The MMA warp issues, per key tile t: S_A(t+1), S_B(t+1), PV_A(t), PV_B(t).
//   S_x(t+1) needs only that the softmax warps of tile x have READ S_x(t)
//   (they signal it before computing), so the tensor core computes the next
//   scores while the softmax of the current ones runs.
// * Softmax warps 0-3 own tile A, warps 4-7 tile B; one thread per tile row
//   (TMEM lane) reads the row's 64 scores, takes the masked maximum, raises
//   the reference maximum lazily (past 2^8, rescaling its O row in TMEM once
//   the previous PV is done), writes P and keeps the row sum of the rounded P.
//
// Every wait is bounded; TMEM is freed on every path after a final commit
// has drained this CTA's MMAs.  Launched behind the decode kernel with
// programmatic dependent launch, like chunk_tc_kernel.
//
// Selected only by pa_set_path(PA_PATH_TCGEN05_PAIRS).  On B200 it computes
// the same results as chunk_tc_kernel but takes ~0.47 ms against ~0.385 ms on
// 16 causal chunks of 512 tokens (32/8 heads, head_dim 128): with one thread
// per tile row its softmax warps, not the tensor core, L2 or the MMA issue
// order, set the pace (variants with 128-key tiles and P written over S,
// with a polling MMA warp, and with single-buffered P measured the same or
// slower).
#pragma once

#include <type_traits>

#include "pa_chunk_tc.cuh"

namespace pa {

constexpr int kTpKeys = 64;  // keys per K/V tile

template <int D>
struct TcPairLayout {
  static constexpr int kKStages = D == 64 ? 8 : 5;
  static constexpr int kVStages = D == 64 ? 8 : 5;
  static constexpr int kHalves = D / 64;
  static constexpr int kQHalfBytes = 128 * 128;             // a Q tile: 128 rows x 128 B per half
  static constexpr int kQTileBytes = kHalves * kQHalfBytes;
  static constexpr int kGroupBytes = kHalves * 1024;        // 8 keys of a K or V tile
  static constexpr int kKVTileBytes = (kTpKeys / 8) * kGroupBytes;
  static constexpr int kOffQ = 0;                           // Q of tiles A and B
  static constexpr int kOffK = kOffQ + 2 * kQTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kKVTileBytes;
  // barrier indexes; [2] = one per tile (A, B)
  static constexpr int kBarQFull = 0;                       // [2]
  static constexpr int kBarQFree = 2;                       // [2]
  static constexpr int kBarKFull = 4;
  static constexpr int kBarKEmpty = kBarKFull + kKStages;
  static constexpr int kBarVFull = kBarKEmpty + kKStages;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarSFull = kBarVEmpty + kVStages;   // [2] S written
  static constexpr int kBarSFree = kBarSFull + 2;           // [2] S read (four warps)
  static constexpr int kBarPFull = kBarSFree + 2;           // [2][2] P(tile, buffer) written
  static constexpr int kBarPFree = kBarPFull + 4;           // [2][2] the PV that read it done
  static constexpr int kBarDrain = kBarPFree + 4;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffItems = kOffBar + kNumBars * 8;
  static constexpr int kItemBytes = 48;
  static constexpr int kOffTmem = kOffItems + kTcItemSlots * kItemBytes;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kBytes = kOffAbort + 12;
  // at least ~114 KB: a single CTA per SM, so its TMEM allocation never waits
  static constexpr int kSmem = (kBytes + 1024) > 116 * 1024 ? (kBytes + 1024) : 116 * 1024;
  static constexpr int kThreads = 320;  // 8 softmax warps, 1 load warp, 1 MMA warp
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffBar % 1024 == 0, "1 KB alignment");
  static_assert(kBytes + 1024 <= 232448, "shared memory budget");
};

// One pair item, as every warp of the CTA sees it.
struct TcPairItem {
  int row, token0, nqa, nqb, kvh, head0, rows, pos0, kv_end, nkt;
};

template <typename T, int D>
__global__ void __launch_bounds__(320, 1)
    chunk_pair_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_q, Shape s, T* __restrict__ out,
                      const int* __restrict__ block_tables, const int* __restrict__ qsl,
                      const int* __restrict__ seq_lens, Work w, float scale_log2) {
  using L = TcPairLayout<D>;
  constexpr int KS = L::kKStages, VS = L::kVStages;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescS = instr_desc_f16(kBf16, false, false, kTcRows, kTpKeys);
  constexpr uint32_t kIdescPV = instr_desc_f16(kBf16, false, true, kTcRows, D);
  static_assert(sizeof(TcPairItem) <= L::kItemBytes, "item slot");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + static_cast<uint32_t>(L::kOffBar + 8 * i); };
  auto qfull = [&](int x) { return bar(L::kBarQFull + x); };
  auto qfree = [&](int x) { return bar(L::kBarQFree + x); };
  auto kfull = [&](int st) { return bar(L::kBarKFull + st); };
  auto kempty = [&](int st) { return bar(L::kBarKEmpty + st); };
  auto vfull = [&](int st) { return bar(L::kBarVFull + st); };
  auto vempty = [&](int st) { return bar(L::kBarVEmpty + st); };
  auto sfull = [&](int x) { return bar(L::kBarSFull + x); };
  auto sfree = [&](int x) { return bar(L::kBarSFree + x); };
  auto pfull = [&](int x, int b) { return bar(L::kBarPFull + 2 * x + b); };
  auto pfree = [&](int x, int b) { return bar(L::kBarPFree + 2 * x + b); };
  const uint32_t drain = bar(L::kBarDrain);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  auto q_smem = [&](int x) { return sbase + L::kOffQ + x * L::kQTileBytes; };
  auto k_smem = [&](int st) { return sbase + L::kOffK + st * L::kKVTileBytes; };
  auto v_smem = [&](int st) { return sbase + L::kOffV + st * L::kKVTileBytes; };
  // item k's metadata: written by the load warp before it arms qfull(0) and
  // qfull(1) for item k, read by the other warps after those phases completed
  auto item_slot = [&](int k) {
    return reinterpret_cast<TcPairItem*>(smem + L::kOffItems + (k % kTcItemSlots) * L::kItemBytes);
  };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      const bool four = (i >= L::kBarSFree && i < L::kBarSFree + 2) ||
                        (i >= L::kBarPFull && i < L::kBarPFull + 4);
      mbar_init(bar(i), four ? 4 : 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // Q of tile B is not loaded for a pair without a second tile: keep its
  // buffer finite
  for (int i = tid; i < L::kQTileBytes / 16; i += L::kThreads)
    reinterpret_cast<uint4*>(smem + L::kOffQ + L::kQTileBytes)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(sbase + L::kOffTmem, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  auto t_s = [&](int x) { return tbase + static_cast<uint32_t>(x * kTpKeys); };
  auto t_p = [&](int x, int b) {
    return tbase + static_cast<uint32_t>(128 + (2 * x + b) * (kTpKeys / 2));
  };
  auto t_o = [&](int x) { return tbase + static_cast<uint32_t>(256 + x * 128); };

  const int count = __ldcg(&w.sched->chunk_count);
  const int items = count * head_units(s);
  // the k-th item of this CTA is blockIdx.x + k * gridDim.x
  const int my_items = static_cast<int>(blockIdx.x) < items
                           ? (items - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1
                           : 0;
  const int qt = kTcRows / s.gs;  // query tokens per tile

  if (warp == 8) {
    // ---------------------------------------------------------- TMA loads
    const int box_rows = min(s.block_size, kBlock);  // rows of one K/V TMA box
    auto entry_of = [&](int k) -> int2 {
      return k < my_items ? __ldcg(w.chunk_list + (blockIdx.x + k * gridDim.x) % count)
                          : make_int2(0, 0);
    };
    auto row_data = [&](int k, int2 ent) -> int3 {  // (qsl[row], qsl[row + 1], seq_lens[row])
      return k < my_items ? make_int3(__ldcg(qsl + ent.x), __ldcg(qsl + ent.x + 1),
                                      __ldcg(seq_lens + ent.x))
                          : make_int3(0, 0, 0);
    };
    auto make_item = [&](int k, int2 ent, int3 rd) {
      TcPairItem it;
      const int hu = (blockIdx.x + k * gridDim.x) / count;
      const int slice = hu % s.ns;
      const int q_len = rd.y - rd.x;
      it.row = ent.x;
      it.kvh = hu / s.ns;
      it.head0 = it.kvh * s.group + slice * 16;
      it.rows = min(s.gs, s.group - slice * 16);
      it.nqa = min(qt, q_len - ent.y);
      it.nqb = max(0, min(qt, q_len - ent.y - qt));
      it.token0 = rd.x + ent.y;
      it.pos0 = rd.z - q_len + ent.y;
      it.kv_end = it.pos0 + it.nqa + it.nqb;
      it.nkt = ceil_div(it.kv_end, kTpKeys);
      return it;
    };
    bool ok = true;
    // make item k current: publish its metadata and load the Q of its tiles
    auto publish = [&](int k, const TcPairItem& it) -> bool {
      bool r = true;
      if (lane == 0) {
        // both Q buffers were last read by the S MMAs of item k - 1
        r = mbar_wait(qfree(0), (k & 1) ^ 1, kWhereWaitQ, abort_flag) &&
            mbar_wait(qfree(1), (k & 1) ^ 1, kWhereWaitQ, abort_flag);
        if (r) {
          *item_slot(k) = it;
          for (int x = 0; x < 2; ++x) {
            if (x == 1 && it.nqb == 0) {
              mbar_arrive(qfull(1));  // no second tile: its rows are all masked
              continue;
            }
            mbar_arrive_expect_tx(qfull(x), static_cast<uint32_t>(L::kQTileBytes));
#pragma unroll
            for (int h = 0; h < L::kHalves; ++h)
              tma_load_3d(q_smem(x) + h * L::kQHalfBytes, &tm_q, qfull(x), h * 64, it.head0,
                          it.token0 + x * qt);
          }
        }
      }
      return __shfl_sync(0xffffffffu, r, 0);
    };
    struct Pending {
      int y, nb, gt;
    };
    Pending va{0, 0, 0}, vb{0, 0, 0};
    int npend = 0;
    auto issue_v = [&](const Pending& p) -> bool {
      const int vs = p.gt % VS;
      bool r = true;
      if (lane == 0) {
        r = mbar_wait(vempty(vs), ((p.gt / VS) & 1) ^ 1, kWhereWaitEmpty, abort_flag);
        if (r)
          mbar_arrive_expect_tx(vfull(vs),
                                static_cast<uint32_t>(p.nb * L::kHalves * box_rows * 128));
      }
      r = __shfl_sync(0xffffffffu, r, 0);
      if (r && lane < p.nb)
        tma_load_4d(v_smem(vs) + lane * (box_rows / 8) * L::kGroupBytes, &tm_v, vfull(vs), 0, 0,
                    0, p.y >> 3);
      return r;
    };
    int2 ent1 = entry_of(1);
    TcPairItem it;
    if (my_items > 0) {
      const int2 ent0 = entry_of(0);
      it = make_item(0, ent0, row_data(0, ent0));
    }
    int3 rd1 = row_data(1, ent1);
    int2 ent2 = entry_of(2);
    if (my_items > 0) ok = publish(0, it);
    int g = 0;  // tiles of earlier items
    for (int k = 0; k < my_items && ok;) {
      for (int t = 0; t < it.nkt && ok; ++t) {
        const int gt = g + t, ks = gt % KS;
        // one lane per TMA box of the tile (16 rows, or 8 with 8-token
        // blocks): its cache row, then its K box
        const int key0 = t * kTpKeys;
        const int nb = min(kTpKeys / box_rows, ceil_div(it.kv_end - key0, box_rows));
        int y = 0;
        if (lane < nb)
          y = key_row(block_tables + static_cast<size_t>(it.row) * s.table_stride,
                      key0 + lane * box_rows, s.block_size, s.num_kv_heads, it.kvh, s.num_blocks,
                      it.row);
        bool r = true;
        if (lane == 0) {
          r = mbar_wait(kempty(ks), ((gt / KS) & 1) ^ 1, kWhereWaitEmpty, abort_flag);
          if (r)
            mbar_arrive_expect_tx(kfull(ks),
                                  static_cast<uint32_t>(nb * L::kHalves * box_rows * 128));
        }
        ok = __shfl_sync(0xffffffffu, r, 0);
        if (!ok) break;
        if (lane < nb)
          tma_load_4d(k_smem(ks) + lane * (box_rows / 8) * L::kGroupBytes, &tm_k, kfull(ks), 0, 0,
                      0, y >> 3);
        // queue this tile's V; issue the previous tile's
        if (npend == 0) {
          va = Pending{y, nb, gt};
          npend = 1;
        } else {
          vb = Pending{y, nb, gt};
          ok = issue_v(va);
          va = vb;
        }
      }
      // the item's last V before the next item's Q
      if (ok && npend == 1) {
        ok = issue_v(va);
        npend = 0;
      }
      g += it.nkt;
      if (++k < my_items && ok) {
        it = make_item(k, ent1, rd1);
        ent1 = ent2;
        rd1 = row_data(k + 1, ent1);
        ent2 = entry_of(k + 2);
        ok = publish(k, it);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issue
    // Tiles of the CTA form one sequence gt = 0, 1, ... across its items;
    // per tile: S_A(gt+1), S_B(gt+1), then PV_A(gt), PV_B(gt).
    int k = 0, t = 0, nkt = 0, kv_end = 0;  // item and tile of the sequence head
    // enter item kk: wait until the Q of both tiles has landed
    auto enter = [&](int kk) -> bool {
      bool r = true;
      int n = 0, e = 0;
      if (lane == 0) {
        r = mbar_wait(qfull(0), kk & 1, kWhereWaitQ, abort_flag) &&
            mbar_wait(qfull(1), kk & 1, kWhereWaitQ, abort_flag);
        if (r) {
          n = item_slot(kk)->nkt;
          e = item_slot(kk)->kv_end;
        }
      }
      r = __shfl_sync(0xffffffffu, r, 0);
      nkt = __shfl_sync(0xffffffffu, n, 0);
      kv_end = __shfl_sync(0xffffffffu, e, 0);
      return r;
    };
    // S_x of global tile gt; `last`: the item's last tile
    auto issue_s = [&](int x, int gt, bool last) -> bool {
      const int ks = gt % KS;
      bool r = true;
      if (lane == 0) {
        if (x == 0) r = mbar_wait(kfull(ks), (gt / KS) & 1, kWhereWaitFull, abort_flag);
        // the softmax warps of tile x have read S_x(gt - 1)
        if (r && gt > 0) r = mbar_wait(sfree(x), (gt - 1) & 1, kWhereWaitMma, abort_flag);
        if (r) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qoff = (kk >> 2) * L::kQHalfBytes + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * 1024 + (kk & 3) * 32;
            umma_ss(t_s(x), smem_desc_sw128(q_smem(x) + qoff, 16, 1024),
                    smem_desc_sw128(k_smem(ks) + koff, 16, L::kGroupBytes), kIdescS, kk > 0);
          }
          umma_commit(sfull(x));
          if (x == 1) umma_commit(kempty(ks));
          if (last) umma_commit(qfree(x));
        }
      }
      return __shfl_sync(0xffffffffu, r, 0);
    };
    // PV_x of global tile gt (tile tt of its item, whose keys end at kend)
    auto issue_pv = [&](int x, int gt, int tt, int kend) -> bool {
      const int vs = gt % VS, b = gt & 1;
      bool r = true;
      if (lane == 0) {
        r = mbar_wait(pfull(x, b), (gt >> 1) & 1, kWhereWaitMma, abort_flag);
        if (r && x == 0) r = mbar_wait(vfull(vs), (gt / VS) & 1, kWhereWaitFull, abort_flag);
      }
      r = __shfl_sync(0xffffffffu, r, 0);
      if (!r) return false;
      const int valid = kend - tt * kTpKeys;  // keys of this tile that exist
      if (x == 0 && valid < kTpKeys) {
        // padding rows may hold anything (NaN included), and 0 * NaN is NaN
        const int nchunks = (kTpKeys - valid) * L::kHalves * 8;
        for (int ch = lane; ch < nchunks; ch += 32) {
          const int row = valid + ch / (L::kHalves * 8);
          const int h = (ch / 8) % L::kHalves;
          *reinterpret_cast<uint4*>(smem + L::kOffV + vs * L::kKVTileBytes +
                                    (row >> 3) * L::kGroupBytes + h * 1024 + (row & 7) * 128 +
                                    (ch % 8) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTpKeys / 16; ++kk) {
          umma_ts(t_o(x), t_p(x, b) + kk * 8,
                  smem_desc_sw128(v_smem(vs) + kk * 2 * L::kGroupBytes, 1024, L::kGroupBytes),
                  kIdescPV, (tt > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(pfree(x, b));
        if (x == 1) umma_commit(vempty(vs));
      }
      return true;
    };
    bool ok = my_items > 0 ? enter(0) : true;
    if (my_items > 0 && ok) ok = issue_s(0, 0, nkt == 1) && issue_s(1, 0, nkt == 1);
    for (int gt = 0; ok && k < my_items; ++gt) {
      // tile gt is tile t of item k: first the next tile's scores, then this
      // tile's P.V products
      const int cur_t = t, cur_end = kv_end;
      int nk = k, ntile = t + 1;
      bool has_next = true;
      if (ntile >= nkt) {
        nk = k + 1;
        ntile = 0;
        has_next = nk < my_items;
      }
      if (has_next) {
        if (nk != k) ok = enter(nk);
        if (ok) ok = issue_s(0, gt + 1, ntile == nkt - 1) && issue_s(1, gt + 1, ntile == nkt - 1);
      }
      if (ok) ok = issue_pv(0, gt, cur_t, cur_end) && issue_pv(1, gt, cur_t, cur_end);
      k = nk;
      t = ntile;
    }
    if (lane == 0) {  // no MMA of this CTA may still run when TMEM is freed
      umma_commit(drain);
      volatile int own_flag = 0;
      mbar_wait(drain, 0, kWhereWaitMma, &own_flag);
    }
  } else {
    // ------------------------------------------------------- softmax warps
    const int x = warp >> 2, quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int r = quad * 32 + lane;  // tile row = TMEM lane
    // Scores enter as v = s * |scale| after a sign flip of s for a negative
    // scale, so that the row maximum is always a max.
    const bool neg = scale_log2 < 0.f;
    const float sc = fabsf(scale_log2);
    int g = 0;
    bool ok = true;
    for (int k = 0; k < my_items && ok; ++k) {
      ok = __all_sync(0xffffffffu, mbar_wait(qfull(x), k & 1, kWhereWaitQ, abort_flag));
      if (!ok) break;
      const TcPairItem it = *item_slot(k);
      const int nq = x ? it.nqb : it.nqa;
      const int i = r / s.gs, gi = r % s.gs;
      const bool valid = i < nq && gi < it.rows;
      const int lim = it.pos0 + x * qt + i + 1;  // keys visible to this row
      float m = -INFINITY;  // reference maximum P is taken against (log2 units)
      float l = 0.f;        // sum of the rounded P of this row
      for (int t = 0; t < it.nkt && ok; ++t) {
        const int gt = g + t;
        ok = __all_sync(0xffffffffu, mbar_wait(sfull(x), gt & 1, kWhereWaitMma, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t ra[64];
        tmem_ld64_issue(t_s(x) + lane_base, ra);
        tmem_ld_wait(ra);
        // S_x is in registers: the next S_x may be computed
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sfree(x));
        float v[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = neg ? -__uint_as_float(ra[j]) : __uint_as_float(ra[j]);
        const int nvis = lim - t * kTpKeys;  // keys of this tile this row may see
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (nvis >= kTpKeys) {
#pragma unroll
          for (int j = 0; j < 64; j += 2) m4[(j >> 1) & 3] = fmax3(m4[(j >> 1) & 3], v[j], v[j + 1]);
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (j < nvis) m4[j & 3] = fmaxf(m4[j & 3], v[j]);
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
        // P buffer gt & 1 is free once PV_x(gt - 2) is done
        const int pb = gt & 1;
        if (gt > 1) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(pfree(x, pb), ((gt >> 1) & 1) ^ 1, kWhereWaitMma, abort_flag));
          if (!ok) break;
          tc_fence_after();
        }
        if (t > 0 && __any_sync(0xffffffffu, raise)) {
          // O_x holds PV of tiles 0 .. t-1 once PV_x(gt - 1) is done: bring
          // this row to the new maximum
          ok = __all_sync(0xffffffffu, mbar_wait(pfree(x, pb ^ 1), ((gt - 1) >> 1) & 1,
                                                 kWhereWaitMma, abort_flag));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t ro[32];
            tmem_ld32_issue(t_o(x) + lane_base + c, ro);
            tmem_ld_wait(ro);
#pragma unroll
            for (int j = 0; j < 32; ++j) ro[j] = __float_as_uint(__uint_as_float(ro[j]) * alpha);
            tmem_st32(t_o(x) + lane_base + c, ro);
          }
        }
        l *= alpha;
        // P = 2^(v - m), rounded to the input type
        const float nm = m == -INFINITY ? 0.f : -m;
        const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(nm, nm);
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float2 a = ffma2(make_float2(v[2 * j], v[2 * j + 1]), sc2, nm2);
          float p0 = ex2_approx(a.x), p1 = ex2_approx(a.y);
          if (nvis < kTpKeys) {
            p0 = 2 * j < nvis ? p0 : 0.f;
            p1 = 2 * j + 1 < nvis ? p1 : 0.f;
          }
          pk[j] = pack2<T>(p0, p1);
        }
        tmem_st32(t_p(x, pb) + lane_base, pk);
        float2 ps[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int j = 0; j < 32; ++j)  // sum the same rounded weights P.V uses
          ps[j & 1] = fadd2(ps[j & 1], unpack2<T>(pk[j]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull(x, pb));
        l += (ps[0].x + ps[0].y) + (ps[1].x + ps[1].y);
      }
      if (ok) {
        // the item's last PV_x done: O_x is final
        const int gl = g + it.nkt - 1;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(pfree(x, gl & 1), (gl >> 1) & 1, kWhereWaitMma, abort_flag));
        if (ok) {
          tc_fence_after();
          const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t ro[32];
            tmem_ld32_issue(t_o(x) + lane_base + c, ro);
            tmem_ld_wait(ro);
            if (valid) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float a[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(ro[q * 8 + e]);
                store_row8<T, D>(s, out, it.token0 + x * qt + i, it.head0 + gi, c / 8 + q, a,
                                 inv);
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
