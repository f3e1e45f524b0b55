// Causal prefill-chunk attention on tcgen05: two query tiles share every K/V
// tile, and each has its own softmax warpgroup.
//
// A chunk row of a mixed batch ("vLLM 深度拆解" §4.3 chunked prefill;
// "vLLM 架构源码解析" §3.2 / §3.3.2) has q_len query tokens at positions
// seq_len - q_len + i over a cached context; its QK^T and P.V are dense
// contractions.  A work item is (chunk row, two consecutive query tiles A and
// B of 128/gs tokens x gs heads = 128 rows each, KV-head slice).  Every
// 128-key K and V tile is brought into shared memory once and used by both
// query tiles, so the bytes a CTA streams from L2 per FLOP are half those of
// a one-tile item (one tile per item needs ~2,100 SM cycles of loads per
// 1,024 cycles of tensor-core work on B200; two tiles bring the loads under
// the MMA time).
//
// * TMEM, 512 columns: S_A [0,128), S_B [128,256), O_A [256,256+D),
//   O_B [384,384+D).  P is written over the first 64 columns of its S
//   (16-bit pairs); the P.V MMA reads it from there as its A operand, and
//   the next S of that tile is issued after that P.V, in order.
// * warp 0 loads the K and V tiles of the CTA's items (one 4-D box of all
//   halves per 16 keys, or per 8-token block) into a K ring and a V ring; V
//   trails K by one tile.  Warp 2 loads Q_A and Q_B (one 3-D TMA box per
//   64-dim half) of each item as soon as the last S of the previous item that
//   read them has completed, so the K/V stream never waits for Q.
// * one thread of warp 1 issues the MMAs in the order P.V_A(t), S_A(t+1),
//   P.V_B(t), S_B(t+1), ...: while softmax A works on S_A the tensor core
//   runs P.V_B and S_B, and the other way round.  One thread of warp 3 does
//   the bookkeeping of those steps (cursors, checks that K, V and Q have
//   landed, V padding rows) and hands each step over, ahead of time.
// * warps 4-7 (tile A) and 8-11 (tile B): one thread per tile row (TMEM lane)
//   reads the row's 128 scores, takes the masked maximum (key <= position),
//   writes P rounded to the input type, and keeps the row sum of P.  The
//   reference maximum that P is taken against is raised only when the row
//   maximum grows past it by more than 2^8; only then is the row's O
//   rescaled in TMEM, after the previous P.V of that tile has completed.  At
//   the end of the item the thread reads its O row once, divides by the sum
//   and stores it.
//
// Tile B may hold fewer tokens than tile A's 128/gs (the row's last pair) or
// none; its rows past the row's tokens are computed and dropped.  Tile A
// sees fewer keys than tile B; the key tiles past its last visible key are
// skipped for A.  Padding keys are masked in the softmax, and the V rows of
// the last 16-key step past the item's last key are zeroed (a padding slot
// may hold anything, NaN included, and 0 * NaN is NaN); P.V stops at the
// 16-key step that holds the tile's last visible key.
//
// Every wait is bounded; a CTA that gives up lets its issued copies land,
// drains its MMAs and frees TMEM.  Launched behind the decode kernel with
// programmatic dependent launch so that it fills that kernel's tail.
#pragma once

#include <type_traits>

#include "pa_sched.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

constexpr int kTcRows = 128;       // query-tile rows = TMEM lanes
constexpr int kTcKeys = 128;       // keys per K/V tile = 8 blocks of 16
constexpr float kTcRescale = 8.f;  // raise the reference maximum past this (log2 units)


template <int D>
struct Tc2Layout {
  static constexpr int kHalves = D / 64;                    // 128-byte swizzle rows per token row
  static constexpr int kHalfBytes = 128 * 128;              // 128 rows x 128 B
  static constexpr int kTileBytes = kHalves * kHalfBytes;   // one Q, K or V tile (128 rows)
  static constexpr int kGroupBytes = kHalves * 1024;        // 8 rows of a K or V tile
  static constexpr int kKStages = D == 64 ? 4 : 3;
  static constexpr int kVStages = D == 64 ? 4 : 2;
  static constexpr int kOffQ = 0;                           // Q_A, Q_B
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  // barrier indexes; [2] = one per query tile (A, B)
  static constexpr int kBarQFull = 0;                       // [2]
  static constexpr int kBarQFree = 2;                       // [2] the item's last S of the tile done
  static constexpr int kBarKFull = 4;
  static constexpr int kBarKEmpty = kBarKFull + kKStages;
  static constexpr int kBarVFull = kBarKEmpty + kKStages;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarSFull = kBarVEmpty + kVStages;   // [2] S written
  static constexpr int kBarPFull = kBarSFull + 2;           // [2] P written (four warps)
  static constexpr int kBarPDone = kBarPFull + 2;           // [2] the P.V that read P done
  static constexpr int kBarDrain = kBarPDone + 2;
  static constexpr int kStepSlots = 4;                      // MMA step ring (warp 3 -> warp 1)
  static constexpr int kBarStepFull = kBarDrain + 1;        // [kStepSlots]
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
  static constexpr int kSmem = kBytes + 1024;               // slack to align the base to 1 KB
  // warps 0: K/V loads, 1: MMA issue, 2: Q loads, 3: MMA step preparation,
  // 4-7: softmax of tile A, 8-11: softmax of tile B
  static constexpr int kThreads = 384;
  // Registers per thread after the split (setmaxnreg): the 128 threads of
  // warps 0-3 give up what the 256 softmax threads take.  Launched with 168
  // (65,536 / 384, rounded down to 8): 128 x 80 + 256 x 208 = 63,488 of the
  // 64,512 the block holds.
  static constexpr int kRegsLaunch = 168;
  static constexpr int kRegsIssue = 80;
  static constexpr int kRegsSoftmax = 208;
  static_assert(128 * kRegsIssue + 256 * kRegsSoftmax <= kThreads * kRegsLaunch,
                "register split within the block's allocation");
  static constexpr uint32_t kTmemCols = 512;
  static_assert(D == 64 || D == 128, "two O accumulators of D columns next to two S");
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffBar % 1024 == 0, "1 KB alignment");
  static_assert(kSmem <= 232448, "shared memory budget");
};

// One work item, as every warp of the CTA sees it.
struct Tc2Item {
  int row, token0, kvh, head0, rows;
  int pos0;        // position of tile A's first query token (tile B's is pos0 + qt)
  int nqa, nqb;    // tokens of tile A and of tile B (nqb may be 0)
  int kv_end_a;    // one past the last key tile A's rows may see
  int kv_end;      // ... tile B's (>= kv_end_a): the item's key range
  int nkt_a, nkt;  // 128-key tiles tile A reads, and the item reads
};

// One step of the MMA issue (P.V of one key tile and S of the next, for both
// query tiles), as warp 3 prepares it for the issuing thread: the checks that
// the step's operands have landed are done, and every stage index and count
// the MMAs need is here.
struct Tc2Step {
  int flags;            // kStep* bits
  int vs, ks;           // V stage of the P.V tile, K stage of the S tile
  int steps_a, steps_b; // 16-key P.V steps holding keys visible to tile A / B
};
constexpr int kStepPvA = 1, kStepPvB = 2, kStepSA = 4, kStepSB = 8, kStepQFreeA = 16,
              kStepQFreeB = 32, kStepAcc = 64, kStepEnd = 128;

// The item `idx` of the chunk list (idx = entry + count * head unit).  Every
// warp role computes it itself from the list and the row metadata.
__device__ __forceinline__ Tc2Item tc2_item(const Shape& s, const Work& w,
                                            const int* __restrict__ qsl,
                                            const int* __restrict__ seq_lens, int count, int idx,
                                            int qt) {
  Tc2Item it;
  const int2 ent = __ldcg(w.chunk_list + idx % count);  // (row, first query of tile A)
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
  it.nqa = min(qt, q_len - ent.y);
  it.nqb = max(0, min(qt, q_len - ent.y - qt));
  it.kv_end_a = it.pos0 + it.nqa;
  it.kv_end = it.nqb > 0 ? it.pos0 + qt + it.nqb : it.kv_end_a;
  it.nkt_a = ceil_div(it.kv_end_a, kTcKeys);
  it.nkt = ceil_div(it.kv_end, kTcKeys);
  return it;
}

// The k-th item of this CTA: rounds of gridDim.x items, visited in
// alternating directions (CTA b takes item b of even rounds and item
// gridDim.x - 1 - b of odd ones), so that a CTA that drew long items in one
// round draws short ones in the next (causal items grow along a chunk row;
// on prefill_16x512 the longest CTA has 3% more key tiles than the mean,
// against 6% for a plain round robin).
__device__ __forceinline__ int chunk_item_index(int k) {
  const int g = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
  return k * g + ((k & 1) ? g - 1 - b : b);
}

// How many items chunk_item_index gives this CTA out of `items`.
__device__ __forceinline__ int chunk_items_of_cta(int items) {
  const int g = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
  const int rounds = items / g, rem = items - rounds * g;
  return rounds + ((rounds & 1) ? (b >= g - rem) : (b < rem));
}

template <typename T, int D>
__global__ void __launch_bounds__(384, 1)
    chunk_tc2_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_q, Shape s, T* __restrict__ out,
                     const int* __restrict__ block_tables, const int* __restrict__ qsl,
                     const int* __restrict__ seq_lens, Work w, float scale_log2) {
  using L = Tc2Layout<D>;
  constexpr int KS = L::kKStages, VS = L::kVStages;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescS = instr_desc_f16(kBf16, false, false, kTcRows, kTcKeys);
  constexpr uint32_t kIdescPV = instr_desc_f16(kBf16, false, true, kTcRows, D);
  static_assert(sizeof(Tc2Item) <= L::kItemBytes, "item slot");
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
  auto pfull = [&](int x) { return bar(L::kBarPFull + x); };
  auto pdone = [&](int x) { return bar(L::kBarPDone + x); };
  const uint32_t drain = bar(L::kBarDrain);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  auto q_smem = [&](int x) { return sbase + L::kOffQ + x * L::kTileBytes; };
  auto k_smem = [&](int st) { return sbase + L::kOffK + st * L::kTileBytes; };
  auto v_smem = [&](int st) { return sbase + L::kOffV + st * L::kTileBytes; };
  // item k's metadata: written by the load warp before it arms qfull(A) of
  // item k, read by the other warps after that phase has completed
  auto item_slot = [&](int k) {
    return reinterpret_cast<Tc2Item*>(smem + L::kOffItems + (k % L::kItemSlots) * L::kItemBytes);
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
  auto t_s = [&](int x) { return tbase + static_cast<uint32_t>(x * kTcKeys); };
  auto t_o = [&](int x) { return tbase + static_cast<uint32_t>(2 * kTcKeys + x * 128); };

  const int count = __ldcg(&w.sched->chunk_count);
  const int items = count * head_units(s);
  // the k-th item of this CTA (chunk_item_index)
  const int my_items = chunk_items_of_cta(items);
  const int qt = kTcRows / s.gs;  // query tokens per tile
  auto item_of = [&](int k) {
    return tc2_item(s, w, qsl, seq_lens, count, chunk_item_index(k), qt);
  };

  if (warp < 4) {
    // load, MMA-issue and Q warps: they need few registers, and the softmax
    // warpgroups take the rest (a row of scores, P and their sums)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(L::kRegsIssue));
    if (warp == 0) {
      // ------------------------------------------------------- K / V loads
      const int box_rows = min(s.block_size, kBlock);  // rows of one K/V TMA box
      bool ok = true;
      // The last K and V loads issued, for the drain of a CTA that gives up, and
      // the test hook: every CTA leaves its first K tile unissued (see
      // g_debug_lost_load).
      int k_last = -1, v_last = -1;
      const int lost = g_debug_lost_load == 2 ? 0 : -1;
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
      Tc2Item it{};
      if (my_items > 0) it = item_of(0);
      Tc2Item nxt = it;
      if (my_items > 1) nxt = item_of(1);
      int g = 0;  // K/V tiles of earlier items
      for (int k = 0; k < my_items && ok; ++k) {
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
        it = nxt;
        if (k + 2 < my_items) nxt = item_of(k + 2);
      }
      if (ok && npend == 1) ok = issue_v(va);  // the last tile's V
      if (!ok && lane == 0) {
        // A wait gave up: let the copies already issued land before the CTA
        // exits (each wait bounded again, independently of the abort flag).
        volatile int own_flag = 0;
        for (int i = max(0, k_last - KS + 1); i <= k_last; ++i)
          if (i != lost) mbar_wait(kfull(i % KS), (i / KS) & 1, kWhereWaitFull, &own_flag);
        for (int i = max(0, v_last - VS + 1); i <= v_last; ++i)
          mbar_wait(vfull(i % VS), (i / VS) & 1, kWhereWaitFull, &own_flag);
      }
    } else if (warp == 2) {
      // ------------------------------------------------------------ Q loads
      // Item k's metadata goes to its slot, then its Q_A and Q_B tiles come in
      // as soon as the last S of item k - 1 that read each buffer has completed.
      if (lane == 0) {
        int q_last = -1;
        bool ok = true;
        Tc2Item nxt{};
        if (my_items > 0) nxt = item_of(0);
        for (int k = 0; k < my_items && ok; ++k) {
          const Tc2Item it = nxt;
          if (k + 1 < my_items) nxt = item_of(k + 1);
          *item_slot(k) = it;
#pragma unroll
          for (int x = 0; x < 2 && ok; ++x) {
            ok = mbar_wait(qfree(x), (k & 1) ^ 1, kWhereWaitQ, abort_flag);
            if (!ok) break;
            mbar_arrive_expect_tx(qfull(x), static_cast<uint32_t>(L::kTileBytes));
#pragma unroll
            for (int h = 0; h < L::kHalves; ++h)
              tma_load_3d(q_smem(x) + h * L::kHalfBytes, &tm_q, qfull(x), h * 64, it.head0,
                          it.token0 + x * qt);
          }
          if (ok) q_last = k;
          // the next item's Q tiles into L2 now, so that their loads, which
          // wait for this item's last S, take an L2 hit
          if (ok && k + 1 < my_items) {
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
              for (int h = 0; h < L::kHalves; ++h)
                tma_prefetch_3d(&tm_q, h * 64, nxt.head0, nxt.token0 + x * qt);
          }
        }
        if (!ok && q_last >= 0) {
          // a wait gave up: let the Q copies already issued land
          volatile int own_flag = 0;
          mbar_wait(qfull(0), q_last & 1, kWhereWaitQ, &own_flag);
          mbar_wait(qfull(1), q_last & 1, kWhereWaitQ, &own_flag);
        }
      }
    } else if (warp == 3) {
      // ---------------------------------------------------- MMA step preparation
      // One thread walks the CTA's (item, key tile) sequence with two cursors,
      // the S cursor one tile ahead of the P.V cursor, waits until each step's
      // V and K tiles (and a new item's Q tiles) have landed, zeroes the V rows
      // of an item's last 16-key step past its last key (padding slots, or rows
      // no box covered; 0 * NaN is NaN), and hands the step to the issuing
      // thread through a ring of shared-memory slots.  The issuing thread then
      // only waits for P and issues: the tensor core accepts only a few MMAs
      // ahead, so bookkeeping in the issuing thread itself would leave it idle.
      if (lane == 0) {
        struct Cursor {
          int k, t, nkt, nkt_a, kv_end_a, kv_end;
          int ks, kph, vs, vph;  // K and V ring stage of the tile, and its phase parity
        };
        auto load_item = [&](Cursor& c, bool wait_q) -> bool {
          if (c.k >= my_items) return true;
          if (wait_q && !mbar_wait(qfull(0), c.k & 1, kWhereWaitQ, abort_flag)) return false;
          const Tc2Item* it = item_slot(c.k);
          c.nkt = it->nkt;
          c.nkt_a = it->nkt_a;
          c.kv_end_a = it->kv_end_a;
          c.kv_end = it->kv_end;
          return true;
        };
        auto advance = [&](Cursor& c) -> bool {  // true when it moved on to the next item
          if (++c.ks == KS) {
            c.ks = 0;
            c.kph ^= 1;
          }
          if (++c.vs == VS) {
            c.vs = 0;
            c.vph ^= 1;
          }
          if (++c.t < c.nkt) return false;
          c.t = 0;
          ++c.k;
          return true;
        };
        int j = 0;  // steps handed over
        auto emit = [&](const Tc2Step& st) -> bool {
          const int slot = j % L::kStepSlots;
          if (!mbar_wait(bar(L::kBarStepFree + slot), ((j / L::kStepSlots) & 1) ^ 1,
                         kWhereWaitMma, abort_flag))
            return false;
          *reinterpret_cast<Tc2Step*>(smem + L::kOffSteps + slot * L::kStepBytes) = st;
          mbar_arrive(bar(L::kBarStepFull + slot));
          ++j;
          return true;
        };
        // the P.V tile's V has landed, its padding rows zeroed
        auto v_ready = [&](const Cursor& c) -> bool {
          if (!mbar_wait(vfull(c.vs), c.vph, kWhereWaitFull, abort_flag)) return false;
          if (c.t == c.nkt - 1) {
            const int key0 = c.t * kTcKeys;
            const int last = min(kTcKeys, c.kv_end - key0);
            const int pad1 = min(kTcKeys, (last + 15) & ~15);
            for (int row = last; row < pad1; ++row) {
              uint8_t* dst = smem + L::kOffV + c.vs * L::kTileBytes + (row >> 3) * L::kGroupBytes +
                             (row & 7) * 128;
#pragma unroll
              for (int h = 0; h < L::kHalves; ++h)
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                  *reinterpret_cast<uint4*>(dst + h * 1024 + ch * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
          return true;
        };
        auto s_flags = [&](const Cursor& c) {
          int f = kStepSB;
          if (c.t < c.nkt_a) f |= kStepSA;
          if (c.t == c.nkt_a - 1) f |= kStepQFreeA;
          if (c.t == c.nkt - 1) f |= kStepQFreeB;
          return f;
        };
        Cursor cs{}, cp{};
        bool ok = true;
        if (my_items > 0) {  // S of the first tile
          ok = load_item(cs, true) &&
               mbar_wait(kfull(cs.ks), cs.kph, kWhereWaitFull, abort_flag) &&
               mbar_wait(qfull(1), 0, kWhereWaitQ, abort_flag) &&
               emit(Tc2Step{s_flags(cs), 0, cs.ks, 0, 0});
          if (ok && advance(cs)) ok = load_item(cs, true);
          if (ok) ok = load_item(cp, false);  // the S cursor has waited for item 0's Q
        }
        while (ok && cp.k < my_items) {
          const bool s_next = cs.k < my_items;
          ok = v_ready(cp) &&
               (!s_next || mbar_wait(kfull(cs.ks), cs.kph, kWhereWaitFull, abort_flag));
          if (!ok) break;
          Tc2Step st;
          st.flags = kStepPvB | (cp.t < cp.nkt_a ? kStepPvA : 0) | (cp.t > 0 ? kStepAcc : 0) |
                     (s_next ? s_flags(cs) : 0);
          st.vs = cp.vs;
          st.ks = cs.ks;
          st.steps_a = (min(kTcKeys, cp.kv_end_a - cp.t * kTcKeys) + 15) >> 4;
          st.steps_b = (min(kTcKeys, cp.kv_end - cp.t * kTcKeys) + 15) >> 4;
          if (s_next && cs.t == 0) {
            // S_B of a new item waits for its Q_B: hand over the rest of the
            // step first, then S_B on its own
            Tc2Step first = st;
            first.flags &= ~(kStepSB | kStepQFreeB);
            ok = emit(first) && mbar_wait(qfull(1), cs.k & 1, kWhereWaitQ, abort_flag) &&
                 emit(Tc2Step{kStepSB | (st.flags & kStepQFreeB), st.vs, st.ks, 0, 0});
          } else {
            ok = emit(st);
          }
          if (ok && advance(cs)) ok = load_item(cs, true);
          if (ok && advance(cp)) ok = load_item(cp, false);  // the S cursor is past it already
        }
        // the end of the CTA's steps (also when it has no items: the issuing
        // thread waits for this)
        if (ok) emit(Tc2Step{kStepEnd, 0, 0, 0, 0});
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issue
      // One thread.  Per step, in this order: P.V_A(t), S_A(t+1), P.V_B(t),
      // S_B(t+1) (steps prepared by warp 3).  S_x(t+1) overwrites the columns
      // P.V_x(t) reads P from; it is issued after that P.V, and the tensor core
      // executes them in order.  The P.V operands are computed before the wait
      // for P, and the P.V MMAs past the last visible key are predicated off
      // inside the instruction, not branched around.  (The other lanes go
      // straight to the teardown barrier: this warp shares its SM
      // sub-partition with two softmax warps.)
      if (lane == 0) {
        int na = 0, nb = 0;  // P.V issued so far for tile A and tile B
        auto issue_s = [&](int x, int ks) {
          // (no tcgen05 fence here: the softmax threads' last reads of S_x were
          // ordered before this thread's tcgen05 operations by the fence after
          // its wait on their P, earlier in this thread's program order)
          const uint64_t qd = smem_desc_sw128(q_smem(x), 16, 1024);
          const uint64_t kd = smem_desc_sw128(k_smem(ks), 16, L::kGroupBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            // descriptor start addresses advance in 16-byte units
            const uint64_t qoff = ((kk >> 2) * L::kHalfBytes + (kk & 3) * 32) >> 4;
            const uint64_t koff = ((kk >> 2) * 1024 + (kk & 3) * 32) >> 4;
            umma_ss(t_s(x), qd + qoff, kd + koff, kIdescS, kk > 0);
          }
          umma_commit(sfull(x));
        };
        auto issue_pv = [&](int x, int vs, int steps, uint32_t acc0, int nx) -> bool {
          const uint64_t vd = smem_desc_sw128(v_smem(vs), 1024, L::kGroupBytes);
          if (!mbar_wait(pfull(x), nx & 1, kWhereWaitMma, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTcKeys / 16; ++kk)
            umma_ts(t_o(x), t_s(x) + kk * 8, vd + ((kk * 2 * L::kGroupBytes) >> 4), kIdescPV,
                    kk > 0 ? 1u : acc0, kk < steps);
          umma_commit(pdone(x));
          return true;
        };
        bool ok = true;
        for (int j = 0; ok; ++j) {
          const int slot = j % L::kStepSlots;
          if (!mbar_wait(bar(L::kBarStepFull + slot), (j / L::kStepSlots) & 1, kWhereWaitMma,
                         abort_flag))
            break;
          const Tc2Step st = *reinterpret_cast<const Tc2Step*>(smem + L::kOffSteps +
                                                               slot * L::kStepBytes);
          mbar_arrive(bar(L::kBarStepFree + slot));
          if (st.flags & kStepEnd) break;
          const uint32_t acc0 = (st.flags & kStepAcc) ? 1u : 0u;
          if (st.flags & kStepPvA) {
            ok = issue_pv(0, st.vs, st.steps_a, acc0, na);
            if (!ok) break;
            ++na;
          }
          if (st.flags & kStepSA) {
            issue_s(0, st.ks);
            if (st.flags & kStepQFreeA) umma_commit(qfree(0));
          }
          if (st.flags & kStepPvB) {
            ok = issue_pv(1, st.vs, st.steps_b, acc0, nb);
            if (!ok) break;
            ++nb;
            umma_commit(vempty(st.vs));  // both tiles' P.V of this V tile issued
          }
          if (st.flags & kStepSB) {
            issue_s(1, st.ks);
            if (st.flags & kStepQFreeB) umma_commit(qfree(1));
            umma_commit(kempty(st.ks));  // both tiles' S of this K tile issued
          }
        }
        // no MMA of this CTA may still run when TMEM is freed
        umma_commit(drain);
        volatile int own_flag = 0;
        mbar_wait(drain, 0, kWhereWaitMma, &own_flag);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(L::kRegsSoftmax));
    {
      // ------------------------------------------------------- softmax warps
      const int x = (warp - 4) >> 2;                        // 0: tile A, 1: tile B
      const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const int r = (warp & 3) * 32 + lane;                 // tile row = TMEM lane
      const int i = r / s.gs, gi = r % s.gs;
      // Scores enter as x = s * |scale| after a sign flip of s for a negative
      // scale, so that the row maximum is always a max.  Masked keys hold
      // -inf, which the exponent turns into 0; a zero scale is taken as
      // 2^-100 so that -inf * scale stays -inf (every visible x is then 0 to
      // within fp32, as with the zero scale).
      const bool neg = scale_log2 < 0.f;
      const bool out32 = (reinterpret_cast<uintptr_t>(out) & 31) == 0;
      const float sc = fmaxf(fabsf(scale_log2), 7.8886091e-31f);
      int nx = 0;  // tiles of this query tile processed so far (P written)
      bool ok = true;
      Tc2Item nxt{};
      if (my_items > 0) nxt = item_of(0);
      for (int k = 0; k < my_items && ok; ++k) {
        // (the metadata comes from the chunk list itself: waiting on the Q
        // barrier for it could observe a phase two items ahead)
        const Tc2Item it = nxt;
        if (k + 1 < my_items) nxt = item_of(k + 1);
        const int nq = x == 0 ? it.nqa : it.nqb;
        const int ntiles = x == 0 ? it.nkt_a : it.nkt;
        const bool valid = i < nq && gi < it.rows;
        const int lim = it.pos0 + x * qt + i + 1;  // keys visible to this row
        float m = -INFINITY;                       // reference maximum (log2 units)
        float l = 0.f;                             // sum of the rounded P
        for (int t = 0; t < ntiles && ok; ++t) {
          ok = __all_sync(0xffffffffu, mbar_wait(sfull(x), nx & 1, kWhereWaitMma, abort_flag));
          if (!ok) break;
          tc_fence_after();
          uint32_t ra[64], rb[64];
          tmem_ld64_issue(t_s(x) + lane_base, ra);
          tmem_ld64_issue(t_s(x) + lane_base + 64, rb);
          tmem_ld_wait(ra);
          reg_tie(rb);
          float v[128];
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            v[j] = __uint_as_float(ra[j]);
            v[64 + j] = __uint_as_float(rb[j]);
          }
          if (neg) {
#pragma unroll
            for (int j = 0; j < 128; ++j) v[j] = -v[j];
          }
          const int nvis = lim - t * kTcKeys;  // keys of this tile this row may see
          if (nvis < kTcKeys) {
#pragma unroll
            for (int j = 0; j < 128; ++j) v[j] = j < nvis ? v[j] : -INFINITY;
          }
          // (eight independent chains: the maximum is on the critical path)
          float m8[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) m8[c] = fmaxf(v[2 * c], v[2 * c + 1]);
#pragma unroll
          for (int j = 16; j < 128; j += 2) m8[(j >> 1) & 7] = fmax3(m8[(j >> 1) & 7], v[j], v[j + 1]);
          const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                                 fmaxf(m8[6], m8[7])) * sc;
          // raise the reference maximum only when the row maximum has grown by
          // more than 2^kTcRescale (always on the first visible keys)
          const bool raise = mx > m + kTcRescale;
          float alpha = 1.f;
          if (raise) {
            alpha = ex2_approx(m - mx);  // 0 when m = -inf
            m = mx;
          }
          l *= alpha;
          // P = 2^(v * sc - m), rounded to the input type, over the first 64
          // columns of S (the scores are all in registers by now).  The row
          // sum adds the weights before their rounding to the input type (the
          // rounding is unbiased; its effect on the normalised output is of
          // order 2^-9 / sqrt(keys)).
          const float nm = m == -INFINITY ? 0.f : -m;
          const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(nm, nm);
          float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float2 a =
                  ffma2(make_float2(v[64 * hh + 2 * j], v[64 * hh + 2 * j + 1]), sc2, nm2);
              const float2 e = make_float2(ex2_approx(a.x), ex2_approx(a.y));
              pk[j] = pack2<T>(e.x, e.y);
              ps[j & 3] = fadd2(ps[j & 3], e);
            }
            tmem_st32(t_s(x) + lane_base + hh * 32, pk);
          }
          if (t > 0 && __any_sync(0xffffffffu, raise)) {
            // O holds P.V of tiles 0 .. t-1: once the last of them is done,
            // bring the row to the new reference point (before P.V of tile t,
            // which waits for this thread's arrival below)
            ok = __all_sync(0xffffffffu,
                            mbar_wait(pdone(x), (nx - 1) & 1, kWhereWaitMma, abort_flag));
            if (!ok) break;
            tc_fence_after();
            uint32_t ro[64];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 64) {
              tmem_ld64_issue(t_o(x) + lane_base + c0, ro);
              tmem_ld_wait(ro);
#pragma unroll
              for (int j = 0; j < 64; ++j) ro[j] = __float_as_uint(__uint_as_float(ro[j]) * alpha);
              tmem_st64(t_o(x) + lane_base + c0, ro);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(pfull(x));
          l += ((ps[0].x + ps[0].y) + (ps[1].x + ps[1].y)) + ((ps[2].x + ps[2].y) + (ps[3].x + ps[3].y));
          ++nx;
        }
        if (ok && ntiles > 0) {
          // the item's last P.V of this tile done: O is final
          ok = __all_sync(0xffffffffu, mbar_wait(pdone(x), (nx - 1) & 1, kWhereWaitMma,
                                                 abort_flag));
          if (ok) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            T* orow = out + (static_cast<size_t>(it.token0 + x * qt + i) * s.num_q_heads +
                             it.head0 + gi) * D;
            uint32_t ro[64];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 64) {
              tmem_ld64_issue(t_o(x) + lane_base + c0, ro);
              tmem_ld_wait(ro);
              if (valid) {
                // each lane writes its own row: whole 32-byte sectors where the
                // output is 32-byte aligned (rows are 128 or 256 bytes)
                if (out32) {
#pragma unroll
                  for (int q = 0; q < 4; ++q) {
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                      w[e] = pack2<T>(__uint_as_float(ro[q * 16 + 2 * e]) * inv,
                                      __uint_as_float(ro[q * 16 + 2 * e + 1]) * inv);
                    st_global_v8(orow + c0 + q * 16, w);
                  }
                } else {
#pragma unroll
                  for (int q = 0; q < 8; ++q) {
                    uint4 w;
                    w.x = pack2<T>(__uint_as_float(ro[q * 8]) * inv, __uint_as_float(ro[q * 8 + 1]) * inv);
                    w.y = pack2<T>(__uint_as_float(ro[q * 8 + 2]) * inv, __uint_as_float(ro[q * 8 + 3]) * inv);
                    w.z = pack2<T>(__uint_as_float(ro[q * 8 + 4]) * inv, __uint_as_float(ro[q * 8 + 5]) * inv);
                    w.w = pack2<T>(__uint_as_float(ro[q * 8 + 6]) * inv, __uint_as_float(ro[q * 8 + 7]) * inv);
                    *reinterpret_cast<uint4*>(orow + c0 + q * 8) = w;
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
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, L::kTmemCols);
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace pa
