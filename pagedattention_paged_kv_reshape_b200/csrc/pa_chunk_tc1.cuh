// Causal prefill-chunk attention on tcgen05 at head_dim 256: one query tile
// per work item, 64-key K/V tiles, S double-buffered in tensor memory.
//
// The same computation as chunk_tc2_kernel ("vLLM 深度拆解" §4.3 chunked
// prefill; "vLLM 架构源码解析" §3.2 / §3.3.2): a chunk row's q_len query tokens
// sit at positions seq_len - q_len + i over a cached context and see keys
// 0 .. position.  At head_dim 256 two query tiles do not fit an SM's 512
// TMEM columns (S 128 + O 256 each), so a work item is (chunk row, one query
// tile of 128/gs tokens x gs heads = 128 rows, KV-head slice), and keys come
// in tiles of 64:
//
// * shared memory: Q (128 rows x 256 dims, 64 KB, four 128-byte-swizzled
//   64-dim halves), a 2-stage K ring and a 2-stage V ring of 64-key tiles
//   (32 KB each, the decode kernel's grouped layout: one 4-D TMA box per
//   16-key block) -- 192 KB;
// * TMEM, 512 columns: S0 [0,64), S1 [64,128), O [256,512).  S of tile g goes
//   to S(g % 2); P of that tile is written over its first 32 columns (16-bit
//   pairs) and read from there by the P.V MMA;
// * warp 0 loads K and V (V one tile behind K), warp 2 loads each item's Q
//   once the previous item's last S has completed (prefetching the next
//   item's Q into L2 first), one thread of warp 1 issues the MMAs in the
//   order S(0), S(1), P.V(0), S(2), P.V(1), S(3), ...: S(g + 2) reuses the
//   columns P.V(g) reads and follows it on the tensor core, so the tensor
//   core computes the next S while the softmax works on the current one;
//   one thread of warp 3 does the bookkeeping of those steps (cursors,
//   checks that K, V and Q have landed, V padding rows) and hands each step
//   over ahead of time;
// * warps 4-7: one thread per tile row reads its 64 scores, takes the masked
//   maximum, raises the reference maximum lazily (by more than 2^8 only; only
//   then is O rescaled, after the previous P.V has completed), writes P
//   rounded to the input type and sums it; at the end of an item it reads
//   its O row once, divides by the sum and stores it.
//
// Padding keys are masked in the softmax (-inf before the exponent), and the
// V rows of the last 16-key step past the item's last key are zeroed (a
// padding slot may hold anything, and 0 * NaN is NaN); P.V stops at the
// 16-key step holding the tile's last visible key.  Every wait is bounded; a
// CTA that gives up lets its issued copies land, drains its MMAs and frees
// TMEM.
#pragma once

#include <type_traits>

#include "pa_chunk_tc2.cuh"

namespace pa {

constexpr int kTc1Keys = 64;  // keys per K/V tile

template <int D>
struct Tc1Layout {
  static_assert(D == 256, "the one-tile form is the head_dim-256 chunk kernel");
  static constexpr int kHalves = D / 64;                   // 64-dim halves of a row
  static constexpr int kHalfBytes = 128 * 128;             // one half of the Q tile
  static constexpr int kQBytes = kHalves * kHalfBytes;     // 64 KB
  static constexpr int kGroupBytes = kHalves * 1024;       // 8 rows of a K or V tile
  static constexpr int kKVBytes = kTc1Keys / 8 * kGroupBytes;  // 32 KB
  // (a third K stage measured within 1%: the K loads are not what waits)
  static constexpr int kKStages = 2;                       // a K tile is free once its S ran
  static constexpr int kVStages = 2;                       // a V tile, once its P.V ran
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kVStages * kKVBytes;
  static constexpr int kBarQFull = 0;
  static constexpr int kBarQFree = 1;                      // the item's last S done
  static constexpr int kBarKFull = 2;                      // [kKStages]
  static constexpr int kBarKEmpty = kBarKFull + kKStages;  // [kKStages]
  static constexpr int kBarVFull = kBarKEmpty + kKStages;  // [2]
  static constexpr int kBarVEmpty = kBarVFull + 2;         // [2]
  static constexpr int kBarSFull = kBarVEmpty + 2;         // [2] one per S buffer
  static constexpr int kBarPFull = kBarSFull + 2;          // [2] four warps each
  // [2] P.V of tiles g with g % 2 = 0, 1.  S runs two tiles ahead of P.V, so
  // when the softmax waits for P.V(g) only P.V(g - 2) is known complete (S(g)
  // followed it): one barrier for every P.V could already show P.V(g - 2)'s
  // phase, of the same parity, while P.V(g - 1) is still running.
  static constexpr int kBarPDone = kBarPFull + 2;
  static constexpr int kBarDrain = kBarPDone + 2;
  static constexpr int kStepSlots = 4;                     // MMA step ring (warp 3 -> warp 1)
  static constexpr int kBarStepFull = kBarDrain + 1;       // [kStepSlots]
  static constexpr int kBarStepFree = kBarStepFull + kStepSlots;  // [kStepSlots]
  static constexpr int kNumBars = kBarStepFree + kStepSlots;
  static constexpr int kOffItems = kOffBar + kNumBars * 8;
  static constexpr int kItemBytes = 64;
  static constexpr int kItemSlots = 8;
  static constexpr int kOffSteps = kOffItems + kItemSlots * kItemBytes;
  static constexpr int kStepBytes = 32;
  static constexpr int kOffTmem = kOffSteps + kStepSlots * kStepBytes;
  static constexpr int kOffAbort = kOffTmem + 4;
  static constexpr int kBytes = kOffAbort + 12;
  static constexpr int kSmem = kBytes + 1024;  // slack to align the base to 1 KB
  // warps 0: K/V loads, 1: MMA issue, 2: Q loads, 3: MMA step preparation,
  // 4-7: softmax
  static constexpr int kThreads = 256;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffBar % 1024 == 0, "1 KB alignment");
  static_assert(kSmem <= 232448, "shared memory budget");
};

// One MMA step of the one-tile form, as warp 3 prepares it for the issuing
// thread: P.V of tile pv_g and S of tile s_g (two tiles ahead), their
// operands checked to have landed.
struct Tc1Step {
  int flags;        // kStep1* bits
  int pv_g, vs, steps;
  int s_g, ks;
};
constexpr int kStep1Pv = 1, kStep1S = 2, kStep1QFree = 4, kStep1Acc = 8, kStep1End = 16;

// One work item of the one-tile form.
struct Tc1Item {
  int row, token0, kvh, head0, rows;
  int pos0;    // position of the tile's first query token
  int nq;      // tokens of the tile
  int kv_end;  // one past the last key the tile's rows may see
  int nkt;     // 64-key tiles it reads
};

// The item `idx` of the chunk list (idx = entry + count * head unit).
__device__ __forceinline__ Tc1Item tc1_item(const Shape& s, const Work& w,
                                            const int* __restrict__ qsl,
                                            const int* __restrict__ seq_lens, int count, int idx,
                                            int qt) {
  Tc1Item it;
  const int2 ent = __ldcg(w.chunk_list + idx % count);  // (row, first query of the tile)
  const int hu = idx / count;
  const int slice = hu % s.ns;
  const int q0 = __ldcg(qsl + ent.x), q_len = __ldcg(qsl + ent.x + 1) - q0;
  const int seq_len = __ldcg(seq_lens + ent.x);
  it.row = ent.x;
  it.kvh = hu / s.ns;
  it.head0 = it.kvh * s.group + slice * 16;
  it.rows = min(s.gs, s.group - slice * 16);
  it.token0 = q0 + ent.y;
  it.pos0 = seq_len - q_len + ent.y;
  it.nq = min(qt, q_len - ent.y);
  it.kv_end = it.pos0 + it.nq;
  it.nkt = ceil_div(it.kv_end, kTc1Keys);
  return it;
}

template <typename T, int D>
__global__ void __launch_bounds__(256, 1)
    chunk_tc1_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_q, Shape s, T* __restrict__ out,
                     const int* __restrict__ block_tables, const int* __restrict__ qsl,
                     const int* __restrict__ seq_lens, Work w, float scale_log2) {
  using L = Tc1Layout<D>;
  constexpr int KS = L::kKStages, VS = L::kVStages;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescS = instr_desc_f16(kBf16, false, false, kTcRows, kTc1Keys);
  constexpr uint32_t kIdescPV = instr_desc_f16(kBf16, false, true, kTcRows, D);
  static_assert(sizeof(Tc1Item) <= L::kItemBytes, "item slot");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + static_cast<uint32_t>(L::kOffBar + 8 * i); };
  const uint32_t qfull = bar(L::kBarQFull), qfree = bar(L::kBarQFree);
  auto kfull = [&](int st) { return bar(L::kBarKFull + st); };
  auto kempty = [&](int st) { return bar(L::kBarKEmpty + st); };
  auto vfull = [&](int st) { return bar(L::kBarVFull + st); };
  auto vempty = [&](int st) { return bar(L::kBarVEmpty + st); };
  auto sfull = [&](int b) { return bar(L::kBarSFull + b); };
  auto pfull = [&](int b) { return bar(L::kBarPFull + b); };
  auto pdone = [&](int b) { return bar(L::kBarPDone + b); };
  const uint32_t drain = bar(L::kBarDrain);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  const uint32_t q_smem = sbase + L::kOffQ;
  auto k_smem = [&](int st) { return sbase + L::kOffK + st * L::kKVBytes; };
  auto v_smem = [&](int st) { return sbase + L::kOffV + st * L::kKVBytes; };
  auto item_slot = [&](int k) {
    return reinterpret_cast<Tc1Item*>(smem + L::kOffItems + (k % L::kItemSlots) * L::kItemBytes);
  };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i)
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
  auto t_s = [&](int b) { return tbase + static_cast<uint32_t>(b * kTc1Keys); };
  const uint32_t t_o = tbase + L::kColO;

  const int count = __ldcg(&w.sched->chunk_count);
  const int items = count * head_units(s);
  // the k-th item of this CTA (chunk_item_index)
  const int my_items = chunk_items_of_cta(items);
  const int qt = kTcRows / s.gs;  // query tokens per tile
  auto item_of = [&](int k) {
    return tc1_item(s, w, qsl, seq_lens, count, chunk_item_index(k), qt);
  };

  if (warp == 0) {
    // ------------------------------------------------------- K / V loads
    const int box_rows = min(s.block_size, kBlock);  // rows of one K/V TMA box
    bool ok = true;
    // the last K and V loads issued, for the drain of a CTA that gives up;
    // the test hook leaves every CTA's first K tile unissued
    int k_last = -1, v_last = -1;
    const int lost = g_debug_lost_load == 2 ? 0 : -1;
    struct Pending {
      int y, nb, gt;
    };
    Pending va{0, 0, 0};
    bool pend = false;
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
    Tc1Item it{};
    if (my_items > 0) it = item_of(0);
    Tc1Item nxt = it;
    if (my_items > 1) nxt = item_of(1);
    int g = 0;  // K/V tiles of earlier items
    for (int k = 0; k < my_items && ok; ++k) {
      for (int t = 0; t < it.nkt && ok; ++t) {
        const int gt = g + t, ks = gt % KS;
        // one lane per TMA box of the tile: its cache row, then its K box
        const int key0 = t * kTc1Keys;
        const int nb = min(kTc1Keys / box_rows, ceil_div(it.kv_end - key0, box_rows));
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
        // this tile's V waits; the previous tile's V goes now
        if (pend) ok = issue_v(va);
        va = Pending{y, nb, gt};
        pend = true;
      }
      g += it.nkt;
      it = nxt;
      if (k + 2 < my_items) nxt = item_of(k + 2);
    }
    if (ok && pend) ok = issue_v(va);  // the last tile's V
    if (!ok && lane == 0) {
      // a wait gave up: let the copies already issued land (bounded again,
      // independently of the abort flag)
      volatile int own_flag = 0;
      for (int i = max(0, k_last - KS + 1); i <= k_last; ++i)
        if (i != lost) mbar_wait(kfull(i % KS), (i / KS) & 1, kWhereWaitFull, &own_flag);
      for (int i = max(0, v_last - VS + 1); i <= v_last; ++i)
        mbar_wait(vfull(i % VS), (i / VS) & 1, kWhereWaitFull, &own_flag);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ Q loads
    // Item k's metadata goes to its slot, then its Q tile comes in once the
    // last S of item k - 1 has completed; the next item's Q is prefetched
    // into L2 meanwhile.
    if (lane == 0) {
      int q_last = -1;
      bool ok = true;
      Tc1Item nxt{};
      if (my_items > 0) nxt = item_of(0);
      for (int k = 0; k < my_items && ok; ++k) {
        const Tc1Item it = nxt;
        if (k + 1 < my_items) nxt = item_of(k + 1);
        *item_slot(k) = it;
        ok = mbar_wait(qfree, (k & 1) ^ 1, kWhereWaitQ, abort_flag);
        if (!ok) break;
        mbar_arrive_expect_tx(qfull, static_cast<uint32_t>(L::kQBytes));
#pragma unroll
        for (int h = 0; h < L::kHalves; ++h)
          tma_load_3d(q_smem + h * L::kHalfBytes, &tm_q, qfull, h * 64, it.head0, it.token0);
        q_last = k;
        if (k + 1 < my_items) {
#pragma unroll
          for (int h = 0; h < L::kHalves; ++h) tma_prefetch_3d(&tm_q, h * 64, nxt.head0, nxt.token0);
        }
      }
      if (!ok && q_last >= 0) {  // a wait gave up: let the Q copies already issued land
        volatile int own_flag = 0;
        mbar_wait(qfull, q_last & 1, kWhereWaitQ, &own_flag);
      }
    }
  } else if (warp == 3) {
    // ---------------------------------------------------- MMA step preparation
    // One thread walks the CTA's tiles with two cursors, the S cursor two
    // tiles ahead of the P.V cursor, waits until each step's V and K tiles
    // (and a new item's Q) have landed, zeroes the V rows of an item's last
    // 16-key step past its last key (padding slots, or rows no box covered),
    // and hands the step to the issuing thread through a ring of shared-memory
    // slots, so that the issuing thread only waits for P and issues.
    if (lane == 0) {
      struct Cursor {
        int k, t, g, nkt, kv_end;
      };
      auto load_item = [&](Cursor& c, bool wait_q) -> bool {
        if (c.k >= my_items) return true;
        if (wait_q && !mbar_wait(qfull, c.k & 1, kWhereWaitQ, abort_flag)) return false;
        const Tc1Item* it = item_slot(c.k);
        c.nkt = it->nkt;
        c.kv_end = it->kv_end;
        return true;
      };
      auto advance = [&](Cursor& c) -> bool {  // true when it moved on to the next item
        ++c.g;
        if (++c.t < c.nkt) return false;
        c.t = 0;
        ++c.k;
        return true;
      };
      int j = 0;  // steps handed over
      auto emit = [&](const Tc1Step& st) -> bool {
        const int slot = j % L::kStepSlots;
        if (!mbar_wait(bar(L::kBarStepFree + slot), ((j / L::kStepSlots) & 1) ^ 1, kWhereWaitMma,
                       abort_flag))
          return false;
        *reinterpret_cast<Tc1Step*>(smem + L::kOffSteps + slot * L::kStepBytes) = st;
        mbar_arrive(bar(L::kBarStepFull + slot));
        ++j;
        return true;
      };
      // S of the S cursor's tile: its K tile landed
      auto s_part = [&](const Cursor& c, Tc1Step& st) -> bool {
        const int ks = c.g % KS;
        if (!mbar_wait(kfull(ks), (c.g / KS) & 1, kWhereWaitFull, abort_flag)) return false;
        st.flags |= kStep1S | (c.t == c.nkt - 1 ? kStep1QFree : 0);  // the item's last S
        st.s_g = c.g;
        st.ks = ks;
        return true;
      };
      Cursor cs{}, cp{};  // the S cursor runs two tiles ahead of the P.V cursor
      bool ok = true;
      if (my_items > 0) {
        ok = load_item(cs, true);
        for (int i = 0; i < 2 && ok && cs.k < my_items; ++i) {
          Tc1Step st{0, 0, 0, 0, 0, 0};
          ok = s_part(cs, st) && emit(st);
          if (ok && advance(cs)) ok = load_item(cs, true);
        }
        if (ok) ok = load_item(cp, false);  // the S cursor has waited for item 0's Q
      }
      while (ok && cp.k < my_items) {
        const int vs = cp.g % VS;
        const int valid = min(kTc1Keys, cp.kv_end - cp.t * kTc1Keys);
        ok = mbar_wait(vfull(vs), (cp.g / VS) & 1, kWhereWaitFull, abort_flag);
        if (!ok) break;
        if (cp.t == cp.nkt - 1) {
          const int pad1 = min(kTc1Keys, (valid + 15) & ~15);
          for (int row = valid; row < pad1; ++row) {
            uint8_t* dst = smem + L::kOffV + vs * L::kKVBytes + (row >> 3) * L::kGroupBytes +
                           (row & 7) * 128;
#pragma unroll
            for (int h = 0; h < L::kHalves; ++h)
#pragma unroll
              for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4*>(dst + h * 1024 + ch * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        Tc1Step st{kStep1Pv | (cp.t > 0 ? kStep1Acc : 0), cp.g, vs, (valid + 15) >> 4, 0, 0};
        const bool s_next = cs.k < my_items;
        if (s_next) ok = s_part(cs, st);
        if (ok) ok = emit(st);
        if (ok && s_next && advance(cs)) ok = load_item(cs, true);
        if (ok && advance(cp)) ok = load_item(cp, false);  // the S cursor is past it already
      }
      // the end of the CTA's steps (also when it has no items: the issuing
      // thread waits for this)
      if (ok) emit(Tc1Step{kStep1End, 0, 0, 0, 0, 0});
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    // One thread.  Tile g of the CTA's sequence: S(g) into S(g % 2) (after
    // P.V(g - 2), which read that buffer's P), P.V(g) once its P is written;
    // per step P.V(g) then S(g + 2), as warp 3 hands them over.
    if (lane == 0) {
      auto issue_s = [&](int g, int ks) {
        const uint64_t qd = smem_desc_sw128(q_smem, 16, 1024);
        const uint64_t kd = smem_desc_sw128(k_smem(ks), 16, L::kGroupBytes);
        const uint32_t ts = t_s(g & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // descriptor start addresses advance in 16-byte units
          const uint64_t qoff = ((kk >> 2) * L::kHalfBytes + (kk & 3) * 32) >> 4;
          const uint64_t koff = ((kk >> 2) * 1024 + (kk & 3) * 32) >> 4;
          umma_ss(ts, qd + qoff, kd + koff, kIdescS, kk > 0);
        }
        umma_commit(sfull(g & 1));
        umma_commit(kempty(ks));
      };
      auto issue_pv = [&](int g, int vs, int steps, uint32_t acc0) -> bool {
        const uint64_t vd = smem_desc_sw128(v_smem(vs), 1024, L::kGroupBytes);
        const uint32_t ts = t_s(g & 1);
        if (!mbar_wait(pfull(g & 1), (g >> 1) & 1, kWhereWaitMma, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTc1Keys / 16; ++kk)
          umma_ts(t_o, ts + kk * 8, vd + ((kk * 2 * L::kGroupBytes) >> 4), kIdescPV,
                  kk > 0 ? 1u : acc0, kk < steps);
        umma_commit(pdone(g & 1));
        umma_commit(vempty(vs));
        return true;
      };
      for (int j = 0;; ++j) {
        const int slot = j % L::kStepSlots;
        if (!mbar_wait(bar(L::kBarStepFull + slot), (j / L::kStepSlots) & 1, kWhereWaitMma,
                       abort_flag))
          break;
        const Tc1Step st =
            *reinterpret_cast<const Tc1Step*>(smem + L::kOffSteps + slot * L::kStepBytes);
        mbar_arrive(bar(L::kBarStepFree + slot));
        if (st.flags & kStep1End) break;
        if ((st.flags & kStep1Pv) &&
            !issue_pv(st.pv_g, st.vs, st.steps, (st.flags & kStep1Acc) ? 1u : 0u))
          break;
        if (st.flags & kStep1S) {
          issue_s(st.s_g, st.ks);
          if (st.flags & kStep1QFree) umma_commit(qfree);  // the item's last S: Q may be replaced
        }
      }
      // no MMA of this CTA may still run when TMEM is freed
      umma_commit(drain);
      volatile int own_flag = 0;
      mbar_wait(drain, 0, kWhereWaitMma, &own_flag);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------- softmax warps
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int r = (warp & 3) * 32 + lane;  // tile row = TMEM lane
    const int i = r / s.gs, gi = r % s.gs;
    // Scores enter as x = s * |scale| after a sign flip of s for a negative
    // scale; masked keys hold -inf (a zero scale is taken as 2^-100, so that
    // -inf * scale stays -inf).
    const bool neg = scale_log2 < 0.f;
    const float sc = fmaxf(fabsf(scale_log2), 7.8886091e-31f);
    const bool out32 = (reinterpret_cast<uintptr_t>(out) & 31) == 0;
    int gtile = 0;  // tiles processed so far (P written), over the CTA's items
    bool ok = true;
    Tc1Item nxt{};
    if (my_items > 0) nxt = item_of(0);
    for (int k = 0; k < my_items && ok; ++k) {
      const Tc1Item it = nxt;
      if (k + 1 < my_items) nxt = item_of(k + 1);
      const bool valid = i < it.nq && gi < it.rows;
      const int lim = it.pos0 + i + 1;  // keys visible to this row
      float m = -INFINITY;              // reference maximum (log2 units)
      float l = 0.f;                    // sum of P
      for (int t = 0; t < it.nkt && ok; ++t, ++gtile) {
        const int b = gtile & 1;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(sfull(b), (gtile >> 1) & 1, kWhereWaitMma, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t ra[64];
        tmem_ld64_issue(t_s(b) + lane_base, ra);
        tmem_ld_wait(ra);
        float v[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = __uint_as_float(ra[j]);
        if (neg) {
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = -v[j];
        }
        const int nvis = lim - t * kTc1Keys;  // keys of this tile this row may see
        if (nvis < kTc1Keys) {
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = j < nvis ? v[j] : -INFINITY;
        }
        float m8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = fmaxf(v[2 * c], v[2 * c + 1]);
#pragma unroll
        for (int j = 16; j < 64; j += 2) m8[(j >> 1) & 7] = fmax3(m8[(j >> 1) & 7], v[j], v[j + 1]);
        const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                               fmaxf(m8[6], m8[7])) * sc;
        const bool raise = mx > m + kTcRescale;
        float alpha = 1.f;
        if (raise) {
          alpha = ex2_approx(m - mx);  // 0 when m = -inf
          m = mx;
        }
        l *= alpha;
        const float nm = m == -INFINITY ? 0.f : -m;
        const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(nm, nm);
        float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float2 a = ffma2(make_float2(v[2 * j], v[2 * j + 1]), sc2, nm2);
          const float2 e = make_float2(ex2_approx(a.x), ex2_approx(a.y));
          pk[j] = pack2<T>(e.x, e.y);
          ps[j & 3] = fadd2(ps[j & 3], e);
        }
        tmem_st32(t_s(b) + lane_base, pk);
        if (t > 0 && __any_sync(0xffffffffu, raise)) {
          // O holds P.V of the item's tiles 0 .. t-1: once the last of them
          // (tile gtile - 1) is done, bring the row to the new reference
          ok = __all_sync(0xffffffffu, mbar_wait(pdone((gtile - 1) & 1), ((gtile - 1) >> 1) & 1,
                                                 kWhereWaitMma, abort_flag));
          if (!ok) break;
          tc_fence_after();
          uint32_t ro[64];
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 64) {
            tmem_ld64_issue(t_o + lane_base + c0, ro);
            tmem_ld_wait(ro);
#pragma unroll
            for (int j = 0; j < 64; ++j) ro[j] = __float_as_uint(__uint_as_float(ro[j]) * alpha);
            tmem_st64(t_o + lane_base + c0, ro);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull(b));
        l += ((ps[0].x + ps[0].y) + (ps[1].x + ps[1].y)) + ((ps[2].x + ps[2].y) + (ps[3].x + ps[3].y));
      }
      if (ok && it.nkt > 0) {
        // the item's last P.V (tile gtile - 1) done: O is final
        ok = __all_sync(0xffffffffu, mbar_wait(pdone((gtile - 1) & 1), ((gtile - 1) >> 1) & 1,
                                               kWhereWaitMma, abort_flag));
        if (ok) {
          tc_fence_after();
          const float inv = l > 0.f ? 1.f / l : 0.f;
          T* orow = out + (static_cast<size_t>(it.token0 + i) * s.num_q_heads + it.head0 + gi) * D;
          uint32_t ro[64];
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 64) {
            tmem_ld64_issue(t_o + lane_base + c0, ro);
            tmem_ld_wait(ro);
            if (valid) {
              if (out32) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  uint32_t wv[8];
#pragma unroll
                  for (int e = 0; e < 8; ++e)
                    wv[e] = pack2<T>(__uint_as_float(ro[q * 16 + 2 * e]) * inv,
                                     __uint_as_float(ro[q * 16 + 2 * e + 1]) * inv);
                  st_global_v8(orow + c0 + q * 16, wv);
                }
              } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  uint4 wv;
                  wv.x = pack2<T>(__uint_as_float(ro[q * 8]) * inv, __uint_as_float(ro[q * 8 + 1]) * inv);
                  wv.y = pack2<T>(__uint_as_float(ro[q * 8 + 2]) * inv, __uint_as_float(ro[q * 8 + 3]) * inv);
                  wv.z = pack2<T>(__uint_as_float(ro[q * 8 + 4]) * inv, __uint_as_float(ro[q * 8 + 5]) * inv);
                  wv.w = pack2<T>(__uint_as_float(ro[q * 8 + 6]) * inv, __uint_as_float(ro[q * 8 + 7]) * inv);
                  *reinterpret_cast<uint4*>(orow + c0 + q * 8) = wv;
                }
              }
            }
          }
          // the next item's first P.V overwrites O: the reads above complete
          // before this thread's next arrival on pfull
          tc_fence_before();
        }
      }
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
