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
//   by the prep kernel, each CTA its items one after another;
// * a load warp brings Q (one 3-D TMA box per 64-dim half, two buffers) and
//   K, V (K and V rings of 128-key tiles; one 4-D box of all halves per 16
//   keys, or per 8-token block) into shared memory with 128-byte swizzling.
//   Q lands as [half][128 rows][128 B], K and V as [8-key group][half][8
//   rows][128 B]: canonical K-major (Q, K) and MN-major (V) layouts for the
//   tcgen05 shared-memory descriptors, with the 8-row group stride as the
//   descriptors' stride byte offset.  It walks the CTA's tiles as one sequence, K one tile ahead of
//   V, runs ahead of the tensor core as far as the rings allow, fetches item
//   metadata one to two items ahead, and hands it to the other warps through
//   shared memory;
// * an MMA warp walks the same sequence: S = Q K^T (M=128, N=128, K=16 steps)
//   into one of two TMEM score buffers, two tiles ahead of O += P V, so the
//   tensor core computes the next scores while the softmax warps work, also
//   across the boundary between two items;
// * eight softmax warps, two threads per tile row: each reads the row's 128
//   scores with one round of tcgen05.ld and takes the row maximum under the
//   causal mask (key <= position), then exponentiates its half of the keys
//   (online softmax in the log2 domain) and writes P, rounded to the input
//   type, into TMEM, where the PV MMA reads it as its A operand;
// * O lives in TMEM for the whole item.  The running maximum that P is taken
//   against is raised only when a row's maximum grows by more than 2^8 (P then
//   stays below 256); only then is the row's O brought to the new reference
//   point, through TMEM, between two PV steps.  The epilogue adds the two
//   halves of the row sum (of the rounded P the PV MMA used), reads O once
//   and divides.
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
constexpr float kTcRescale = 8.f;   // raise the reference maximum past this (log2 units)
constexpr int kTcItemSlots = 4;     // item metadata handed from the load warp

template <int D>
struct TcLayout {
  static constexpr int kQStages = 2;
  static constexpr int kKStages = D == 64 ? 4 : 3;  // a K tile is free once its QK^T has run
  static constexpr int kVStages = D == 64 ? 4 : 2;  // a V tile is free once its PV has run
  static constexpr int kHalves = D / 64;            // 128-byte swizzle rows per token row
  static constexpr int kHalfBytes = 128 * 128;      // 128 rows x 128 B
  static constexpr int kTileBytes = kHalves * kHalfBytes;  // one Q, K or V tile
  static constexpr int kGroupBytes = kHalves * 1024;        // 8 keys of a K or V tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQStages * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  // barrier indexes
  static constexpr int kBarQFull = 0;
  static constexpr int kBarQFree = kBarQFull + kQStages;
  static constexpr int kBarKFull = kBarQFree + kQStages;
  static constexpr int kBarKEmpty = kBarKFull + kKStages;
  static constexpr int kBarVFull = kBarKEmpty + kKStages;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarSFull = kBarVEmpty + kVStages;  // S(b) written
  static constexpr int kBarPFull = kBarSFull + 2;          // P(b) written (8 warps)
  static constexpr int kBarPFree = kBarPFull + 2;          // the PV that read P(b) done
  static constexpr int kBarPair = kBarPFree + 2;           // the two warps of a row quarter
  static constexpr int kBarDrain = kBarPair + 4;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffItems = kOffBar + kNumBars * 8;
  static constexpr int kItemBytes = 48;
  static constexpr int kOffLsum = kOffItems + kTcItemSlots * kItemBytes;  // [2 halves][128 rows]
  static constexpr int kOffTmem = kOffLsum + 2 * kTcRows * 4;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kBytes = kOffAbort + 12;
  // at least ~114 KB, so that a single CTA fits per SM and its TMEM
  // allocation can never wait for another CTA's
  static constexpr int kSmem = (kBytes + 1024) > 116 * 1024 ? (kBytes + 1024) : 116 * 1024;
  static constexpr int kThreads = 320;  // 8 softmax warps, 1 load warp, 1 MMA warp
  // TMEM columns: S0 [0,128), S1 [128,256), O [256, 256 + D), P0 [384,448), P1 [448,512)
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffBar % 1024 == 0, "1 KB alignment");
  static_assert(kBytes + 1024 <= 232448, "shared memory budget");
};

// One work item, as every warp of the CTA sees it.
struct TcItem {
  int row, token0, nq, kvh, head0, rows, pos0, kv_end, nkt;
};

template <typename T, int D>
__global__ void __launch_bounds__(320, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, Shape s, T* __restrict__ out,
                    const int* __restrict__ block_tables, const int* __restrict__ qsl,
                    const int* __restrict__ seq_lens, Work w, float scale_log2) {
  using L = TcLayout<D>;
  constexpr int QS = L::kQStages, KS = L::kKStages, VS = L::kVStages;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescS = instr_desc_f16(kBf16, false, false, kTcRows, kTcKeys);
  constexpr uint32_t kIdescPV = instr_desc_f16(kBf16, false, true, kTcRows, D);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + static_cast<uint32_t>(L::kOffBar + 8 * i); };
  auto qfull = [&](int qb) { return bar(L::kBarQFull + qb); };
  auto qfree = [&](int qb) { return bar(L::kBarQFree + qb); };
  auto kfull = [&](int st) { return bar(L::kBarKFull + st); };
  auto kempty = [&](int st) { return bar(L::kBarKEmpty + st); };
  auto vfull = [&](int st) { return bar(L::kBarVFull + st); };
  auto vempty = [&](int st) { return bar(L::kBarVEmpty + st); };
  auto sfull = [&](int b) { return bar(L::kBarSFull + b); };
  auto pfull = [&](int b) { return bar(L::kBarPFull + b); };
  auto pfree = [&](int b) { return bar(L::kBarPFree + b); };
  auto pairbar = [&](int quad) { return bar(L::kBarPair + quad); };
  const uint32_t drain = bar(L::kBarDrain);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  auto q_smem = [&](int qb) { return sbase + L::kOffQ + qb * L::kTileBytes; };
  auto k_smem = [&](int st) { return sbase + L::kOffK + st * L::kTileBytes; };
  auto v_smem = [&](int st) { return sbase + L::kOffV + st * L::kTileBytes; };
  // item k's metadata: written by the load warp before it arms qfull(k % 2),
  // read by the other warps after that phase has completed
  auto item_slot = [&](int k) {
    return reinterpret_cast<TcItem*>(smem + L::kOffItems + (k % kTcItemSlots) * L::kItemBytes);
  };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      int n = 1;
      if (i == L::kBarPFull || i == L::kBarPFull + 1) n = 8;  // the eight softmax warps
      if (i >= L::kBarPair && i < L::kBarPair + 4) n = 2;     // the two warps of a pair
      mbar_init(bar(i), n);
    }
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
  auto t_s = [&](int b) { return tbase + static_cast<uint32_t>(b * kTcKeys); };
  const uint32_t t_o = tbase + 2 * kTcKeys;
  auto t_p = [&](int b) { return tbase + static_cast<uint32_t>(3 * kTcKeys + b * kTcKeys / 2); };

  const int count = __ldcg(&w.sched->chunk_count);
  const int items = count * head_units(s);
  // the k-th item of this CTA is blockIdx.x + k * gridDim.x
  const int my_items = static_cast<int>(blockIdx.x) < items
                           ? (items - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1
                           : 0;

  if (warp == 8) {
    // ---------------------------------------------------------- TMA loads
    const int qt = kTcRows / s.gs;
    const int box_rows = min(s.block_size, kBlock);  // rows of one K/V TMA box
    // Item metadata is fetched ahead: the chunk-list entry of item k + 2 and
    // the row data of item k + 1 are in flight while item k is issued.
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
      TcItem it;
      const int hu = (blockIdx.x + k * gridDim.x) / count;
      const int slice = hu % s.ns;
      const int q_len = rd.y - rd.x;
      it.row = ent.x;
      it.kvh = hu / s.ns;
      it.head0 = it.kvh * s.group + slice * 16;
      it.rows = min(s.gs, s.group - slice * 16);
      it.nq = min(qt, q_len - ent.y);
      it.token0 = rd.x + ent.y;
      it.pos0 = rd.z - q_len + ent.y;
      it.kv_end = it.pos0 + it.nq;
      it.nkt = ceil_div(it.kv_end, kTcKeys);
      return it;
    };
    bool ok = true;
    // The last Q, K and V loads issued (a CTA that gives up waits for them
    // before it exits), and the test hook: every CTA leaves its first K tile
    // unissued (see g_debug_lost_load).
    int q_last = -1, k_last = -1, v_last = -1;
    const int lost = g_debug_lost_load == 2 ? 0 : -1;
    // make item k current: publish its metadata and load its Q
    auto publish = [&](int k, const TcItem& it) -> bool {
      const int qb = k % QS;
      bool r = true;
      if (lane == 0) {
        // Q buffer qb was last read by the S MMAs of item k - 2
        r = mbar_wait(qfree(qb), ((k / QS) & 1) ^ 1, kWhereWaitQ, abort_flag);
        if (r) {
          *item_slot(k) = it;
          mbar_arrive_expect_tx(qfull(qb), static_cast<uint32_t>(L::kTileBytes));
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_3d(q_smem(qb) + h * L::kHalfBytes, &tm_q, qfull(qb), h * 64, it.head0,
                        it.token0);
        }
      }
      r = __shfl_sync(0xffffffffu, r, 0);
      if (r) q_last = k;
      return r;
    };
    // V of a tile reuses the block ids its K looked up; at most two tiles
    // wait for their V (the older one is issued right after a new K).
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
      if (r) v_last = p.gt;
      return r;
    };
    int2 ent1 = entry_of(1);
    TcItem it;
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
        // one lane per TMA box of the tile (box = 16 rows, or 8 rows with
        // 8-token blocks): its cache row, then its K boxes
        const int key0 = t * kTcKeys;
        const int nb = min(kTcKeys / box_rows, ceil_div(it.kv_end - key0, box_rows));
        int y = 0;
        if (lane < nb)
          y = key_row(block_tables + static_cast<size_t>(it.row) * s.table_stride,
                      key0 + lane * box_rows, s.block_size, s.num_kv_heads, it.kvh, s.num_blocks,
                      it.row);
        bool r = true;
        if (lane == 0) {
          r = mbar_wait(kempty(ks), ((gt / KS) & 1) ^ 1, kWhereWaitEmpty, abort_flag);
          if (r && gt != lost)
            mbar_arrive_expect_tx(kfull(ks),
                                  static_cast<uint32_t>(nb * L::kHalves * box_rows * 128));
        }
        ok = __shfl_sync(0xffffffffu, r, 0);
        if (!ok) break;
        if (lane < nb && gt != lost)
          tma_load_4d(k_smem(ks) + lane * (box_rows / 8) * L::kGroupBytes, &tm_k, kfull(ks), 0, 0,
                      0, y >> 3);
        k_last = gt;
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
      g += it.nkt;
      if (++k < my_items && ok) {
        it = make_item(k, ent1, rd1);
        ent1 = ent2;
        rd1 = row_data(k + 1, ent1);
        ent2 = entry_of(k + 2);
        ok = publish(k, it);
      }
    }
    if (ok && npend == 1) ok = issue_v(va);  // the last tile's V
    if (!ok && lane == 0) {
      // A wait gave up: let the copies already issued land before the CTA
      // exits (each wait bounded again, independently of the abort flag).
      volatile int own_flag = 0;
      for (int i = max(0, q_last - QS + 1); i <= q_last; ++i)
        mbar_wait(qfull(i % QS), (i / QS) & 1, kWhereWaitQ, &own_flag);
      for (int i = max(0, k_last - KS + 1); i <= k_last; ++i)
        if (i != lost) mbar_wait(kfull(i % KS), (i / KS) & 1, kWhereWaitFull, &own_flag);
      for (int i = max(0, v_last - VS + 1); i <= v_last; ++i)
        mbar_wait(vfull(i % VS), (i / VS) & 1, kWhereWaitFull, &own_flag);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issue
    // The CTA's tiles form one sequence gt = 0, 1, 2, ... across its items.
    // S(gt + 2) is issued right after PV(gt): by then the softmax warps have
    // read S buffer gt % 2 (they wrote P(gt) after reading it).  Two cursors
    // walk the sequence, the S cursor two tiles ahead of the PV cursor.
    struct Cursor {
      int k, t, g0, nkt, kv_end;
    };
    // enter item c.k: wait until its Q has landed (its metadata with it)
    auto enter = [&](Cursor& c, bool wait_q) -> bool {
      if (c.k >= my_items) return true;
      bool r = true;
      int nkt = 0, kv_end = 0;
      if (lane == 0) {  // the lane that observed qfull reads the slot
        if (wait_q) r = mbar_wait(qfull(c.k % QS), (c.k / QS) & 1, kWhereWaitQ, abort_flag);
        if (r) {
          nkt = item_slot(c.k)->nkt;
          kv_end = item_slot(c.k)->kv_end;
        }
      }
      r = __shfl_sync(0xffffffffu, r, 0);
      c.nkt = __shfl_sync(0xffffffffu, nkt, 0);
      c.kv_end = __shfl_sync(0xffffffffu, kv_end, 0);
      return r;
    };
    auto advance = [&](Cursor& c) {  // true when it moved on to the next item
      if (++c.t < c.nkt) return false;
      c.g0 += c.nkt;
      c.t = 0;
      ++c.k;
      return true;
    };
    auto issue_s = [&](const Cursor& c) -> bool {
      const int gt = c.g0 + c.t, ks = gt % KS, qb = c.k % QS;
      bool r = true;
      if (lane == 0) {
        r = mbar_wait(kfull(ks), (gt / KS) & 1, kWhereWaitFull, abort_flag);
        if (r) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qoff = (kk >> 2) * L::kHalfBytes + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * 1024 + (kk & 3) * 32;
            umma_ss(t_s(gt & 1), smem_desc_sw128(q_smem(qb) + qoff, 16, 1024),
                    smem_desc_sw128(k_smem(ks) + koff, 16, L::kGroupBytes), kIdescS, kk > 0);
          }
          umma_commit(sfull(gt & 1));
          umma_commit(kempty(ks));
          if (c.t == c.nkt - 1) umma_commit(qfree(qb));
        }
      }
      return __shfl_sync(0xffffffffu, r, 0);
    };
    auto issue_pv = [&](const Cursor& c) -> bool {
      const int gt = c.g0 + c.t, vs = gt % VS, b = gt & 1;
      bool r = true;
      if (lane == 0) {
        r = mbar_wait(pfull(b), (gt >> 1) & 1, kWhereWaitMma, abort_flag) &&
            mbar_wait(vfull(vs), (gt / VS) & 1, kWhereWaitFull, abort_flag);
      }
      r = __shfl_sync(0xffffffffu, r, 0);
      if (!r) return false;
      const int valid = c.kv_end - c.t * kTcKeys;  // keys of this tile that exist
      if (valid < kTcKeys) {
        // padding rows may hold anything (NaN included), and 0 * NaN is NaN
        const int nchunks = (kTcKeys - valid) * L::kHalves * 8;
        for (int ch = lane; ch < nchunks; ch += 32) {
          const int row = valid + ch / (L::kHalves * 8);
          const int h = (ch / 8) % L::kHalves;
          *reinterpret_cast<uint4*>(smem + L::kOffV + vs * L::kTileBytes +
                                    (row >> 3) * L::kGroupBytes + h * 1024 + (row & 7) * 128 +
                                    (ch % 8) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTcKeys / 16; ++kk) {
          umma_ts(t_o, t_p(b) + kk * 8,
                  smem_desc_sw128(v_smem(vs) + kk * 2 * L::kGroupBytes, 1024, L::kGroupBytes),
                  kIdescPV, (c.t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(pfree(b));
        umma_commit(vempty(vs));
      }
      return true;
    };
    Cursor cs{0, 0, 0, 0, 0}, cp{0, 0, 0, 0, 0};
    bool ok = enter(cs, true);
    for (int j = 0; j < 2 && ok && cs.k < my_items; ++j) {
      ok = issue_s(cs);
      if (ok && advance(cs)) ok = enter(cs, true);
    }
    if (ok) ok = enter(cp, false);  // the S cursor has waited for item 0's Q
    while (ok && cp.k < my_items) {
      ok = issue_pv(cp);
      if (ok && advance(cp)) ok = enter(cp, false);  // the S cursor is past it already
      if (ok && cs.k < my_items) {
        ok = issue_s(cs);
        if (ok && advance(cs)) ok = enter(cs, true);
      }
    }
    if (lane == 0) {  // no MMA of this CTA may still run when TMEM is freed
      umma_commit(drain);
      volatile int own_flag = 0;
      mbar_wait(drain, 0, kWhereWaitMma, &own_flag);
    }
  } else {
    // ------------------------------------------------------- softmax warps
    // Warps q and q + 4 share TMEM lanes 32q .. 32q + 31 (tile rows): both
    // take the row maximum over all 128 keys of a tile, warp q exponentiates
    // keys 0 .. 63, warp q + 4 keys 64 .. 127, and O's columns are split the
    // same way.
    const int quad = warp & 3, h = warp >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int r = quad * 32 + lane;  // tile row = TMEM lane
    float* lsum = reinterpret_cast<float*>(smem + L::kOffLsum);  // [2][128]
    // Scores enter as x = s * |scale| after a sign flip of s for a negative
    // scale, so that the row maximum is always a max.
    const bool neg = scale_log2 < 0.f;
    const float sc = fabsf(scale_log2);
    constexpr int kHalfD = D / 2;
    int g = 0;
    bool ok = true;
    for (int k = 0; k < my_items && ok; ++k) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(qfull(k % QS), (k / QS) & 1, kWhereWaitQ, abort_flag));
      if (!ok) break;
      const TcItem it = *item_slot(k);
      const int i = r / s.gs, gi = r % s.gs;
      const bool valid = i < it.nq && gi < it.rows;
      const int lim = it.pos0 + i + 1;  // keys visible to this row
      float m = -INFINITY;              // reference maximum P is taken against (log2 units)
      float l = 0.f;                    // this half's sum of the rounded P
      for (int t = 0; t < it.nkt && ok; ++t) {
        const int gt = g + t, b = gt & 1;
        // scores of this tile, and P buffer b free (the PV two tiles back done)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(sfull(b), (gt >> 1) & 1, kWhereWaitMma, abort_flag) &&
                            mbar_wait(pfree(b), ((gt >> 1) & 1) ^ 1, kWhereWaitMma, abort_flag));
        if (!ok) break;
        tc_fence_after();
        // x: this thread's half of the keys (h*64 ..), y: the other half
        uint32_t ra[64], rb[64];
        tmem_ld64_issue(t_s(b) + lane_base + h * 64, ra);
        tmem_ld64_issue(t_s(b) + lane_base + (h ^ 1) * 64, rb);
        tmem_ld_wait(ra);
        reg_tie(rb);
        float x[64], y[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          x[j] = __uint_as_float(ra[j]);
          y[j] = __uint_as_float(rb[j]);
        }
        if (neg) {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            x[j] = -x[j];
            y[j] = -y[j];
          }
        }
        const int nvis = lim - t * kTcKeys;  // keys of this tile this row may see
        const int hv = nvis - h * 64;        // ... of this thread's half
        const int ov = nvis - (h ^ 1) * 64;  // ... of the other half
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (nvis >= kTcKeys) {
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            m4[(j >> 1) & 1] = fmax3(m4[(j >> 1) & 1], x[j], x[j + 1]);
            m4[2 + ((j >> 1) & 1)] = fmax3(m4[2 + ((j >> 1) & 1)], y[j], y[j + 1]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            if (j < hv) m4[j & 1] = fmaxf(m4[j & 1], x[j]);
            if (j < ov) m4[2 + (j & 1)] = fmaxf(m4[2 + (j & 1)], y[j]);
          }
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
          // O holds PV of tiles 0 .. t-1: once PV(t-1) is done, scale this
          // thread's half of the row
          ok = __all_sync(0xffffffffu, mbar_wait(pfree((gt - 1) & 1), ((gt - 1) >> 1) & 1,
                                                 kWhereWaitMma, abort_flag));
          if (!ok) break;
          tc_fence_after();
          if constexpr (kHalfD == 64) {
            uint32_t ro[64];
            tmem_ld64_issue(t_o + lane_base + h * kHalfD, ro);
            tmem_ld_wait(ro);
#pragma unroll
            for (int j = 0; j < 64; ++j) ro[j] = __float_as_uint(__uint_as_float(ro[j]) * alpha);
            tmem_st64(t_o + lane_base + h * kHalfD, ro);
          } else {
            uint32_t ro[32];
            tmem_ld32_issue(t_o + lane_base + h * kHalfD, ro);
            tmem_ld_wait(ro);
#pragma unroll
            for (int j = 0; j < 32; ++j) ro[j] = __float_as_uint(__uint_as_float(ro[j]) * alpha);
            tmem_st32(t_o + lane_base + h * kHalfD, ro);
          }
        }
        l *= alpha;
        // P = 2^(x - m) for this half, rounded to the input type, into P(b)
        const float nm = m == -INFINITY ? 0.f : -m;
        const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(nm, nm);
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float2 a = ffma2(make_float2(x[2 * j], x[2 * j + 1]), sc2, nm2);
          float p0 = ex2_approx(a.x), p1 = ex2_approx(a.y);
          if (hv < 64) {
            p0 = 2 * j < hv ? p0 : 0.f;
            p1 = 2 * j + 1 < hv ? p1 : 0.f;
          }
          pk[j] = pack2<T>(p0, p1);
        }
        tmem_st32(t_p(b) + lane_base + h * 32, pk);
        float2 ps[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int j = 0; j < 32; ++j)  // sum the same rounded weights P.V uses
          ps[j & 1] = fadd2(ps[j & 1], unpack2<T>(pk[j]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull(b));
        l += (ps[0].x + ps[0].y) + (ps[1].x + ps[1].y);
      }
      if (ok) {
        // both halves of the row sum, through shared memory
        lsum[h * kTcRows + r] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(pairbar(quad));
        ok = __all_sync(0xffffffffu, mbar_wait(pairbar(quad), k & 1, kWhereWaitMma, abort_flag));
        const float lt = l + lsum[(h ^ 1) * kTcRows + r];
        // the item's last PV done: O is final
        const int gl = g + it.nkt - 1;
        if (ok)
          ok = __all_sync(0xffffffffu, mbar_wait(pfree(gl & 1), (gl >> 1) & 1, kWhereWaitMma,
                                                 abort_flag));
        if (ok) {
          tc_fence_after();
          const float inv = lt > 0.f ? 1.f / lt : 0.f;
          if constexpr (kHalfD == 64) {
            uint32_t ro[64];
            tmem_ld64_issue(t_o + lane_base + h * kHalfD, ro);
            tmem_ld_wait(ro);
            if (valid) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                float a[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(ro[q * 8 + e]);
                store_row8<T, D>(s, out, it.token0 + i, it.head0 + gi, h * 8 + q, a, inv);
              }
            }
          } else {
            uint32_t ro[32];
            tmem_ld32_issue(t_o + lane_base + h * kHalfD, ro);
            tmem_ld_wait(ro);
            if (valid) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float a[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(ro[q * 8 + e]);
                store_row8<T, D>(s, out, it.token0 + i, it.head0 + gi, h * 4 + q, a, inv);
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
