// Paged attention on sm_100a: TMA-staged K/V tiles + warp-level tensor-core MMA.
//
// Persistent, warp-specialised CTA: NCW consumer warps, one TMA warp, one
// scheduler warp.
//
// * The scheduler warp claims work units (pa_sched.cuh) from a global counter,
//   decodes them and loads the request's block-table entries for the unit's
//   partition ("vLLM 深度拆解" §3.3: physical = block_tables[seq*stride +
//   logical]) into a ring of shared-memory slots, running several units ahead
//   so that the dependent global loads of that lookup never delay the stream.
// * The TMA warp takes each slot and issues cp.async.bulk.tensor loads of the
//   tile's query rows and of every 16-key K tile and V tile of the unit --
//   16 tokens x head_dim, 4 KB each at bf16 x 128 -- into a STAGES-deep ring
//   of shared-memory stages completed on mbarriers.  A 16-bit tile lands as
//   [8-row group][64-dim half][8 rows][128 B]: one 4-D box per tile for 16-
//   and 32-token blocks, one 3-D box per block for two 8-token blocks (the
//   count and size of boxes set the achievable bandwidth: 1 KB boxes cap it
//   near 73% of the copy rate, 4 KB boxes do not).  The tensor maps use
//   128-byte swizzling, so the ldmatrix reads below are free of bank conflicts.
// * Consumer warp w takes the unit's blocks w, w+NCW, ...: S = Q K^T (16 tile
//   rows x 16 tokens, m16n8k16 MMAs, fp32 accumulate), masking of keys past
//   each row's limit, online softmax in the log2 domain (running max m, sum
//   l), P rounded to the input type, O += P V with the same MMA.  A whole GQA
//   group (up to 16 query heads) shares one K/V tile, so each KV block is read
//   once per KV head.
// * At the end of a unit the consumer warps merge their states and write the
//   output row, or the partition's partial for the split-K reduce.
#pragma once

#include "pa_sched.cuh"

namespace pa {

constexpr int kMetaSlots = 4;
constexpr float kLazyRaise = 8.f;  // see the online softmax of attn_mma_kernel (log2 units)
constexpr int kIssueLanes = 2;     // lanes of the TMA warp that issue K/V loads

// One scheduler-ring slot: a decoded unit and, for each 16-key tile of its
// partition, the cache row of the tile's first key (y0) and, with 8-token
// blocks, of its ninth key (y1; -1 when the tile has no second block).
struct MetaSlot {
  Unit u;
  int y0[kPart / kBlock];
  int y1[kPart / kBlock];
};

// KV8: the cache holds FP8 e4m3 codes and a stage holds the 1-byte K and V
// tiles (16 rows x D bytes).  At head_dim 128 they are 128 B-swizzled and the
// consumers build their MMA operands straight from them (see fp8_direct
// below); at head_dim 64 and 256 they are unswizzled and each consumer warp
// first converts its tile into a 16-bit staging tile laid out like a 16-bit
// stage.
template <int D, int NCW, int STAGES, bool KV8 = false, bool NARROW = false>
struct MmaLayout {
  static constexpr bool kStaging = KV8 && D != 128;
  static constexpr int kHalves = D / 64;             // 64 16-bit elements = one 128 B swizzle row
  static constexpr int kHalfBytes = kBlock * 128;    // 16 rows x 128 B
  static constexpr int kTileBytes = kHalves * kHalfBytes;          // a 16-bit K or V tile
  // a 16-bit tile is [2 groups of 8 rows][kHalves][8 rows][128 B]
  static constexpr int kGroupBytes = kHalves * 8 * 128;
  static constexpr int kKVTileBytes = KV8 ? kBlock * D : kTileBytes;  // ... as loaded
  static constexpr int kStageBytes = 2 * kKVTileBytes;  // K tile then V tile
  // a query tile of at most 8 rows in the NARROW form, else 16: [half][rows][128 B]
  static constexpr int kQRows = NARROW ? 8 : kRows;
  static constexpr int kQSlotBytes = kHalves * kQRows * 128;
  static constexpr int kQSlots = 2;
  static constexpr int kOffQ = STAGES * kStageBytes;
  static constexpr int kOffCo = kOffQ + kQSlots * kQSlotBytes;
  static constexpr int kCoRows = NARROW ? 8 : kRows;  // tile rows the merge buffer holds
  static constexpr int kCoBytes = NCW * kCoRows * (D + 8) * 4;
  static constexpr int kOffCm = kOffCo + kCoBytes;
  static constexpr int kOffCl = kOffCm + NCW * kCoRows * 4;
  static constexpr int kOffBar = kOffCl + NCW * kCoRows * 4;
  // full[S], empty[S], qfull[2], qempty[2], meta_full[M], meta_empty[M], consumers
  static constexpr int kNumBars = 2 * STAGES + 2 * kQSlots + 2 * kMetaSlots + 1;
  static constexpr int kOffDesc = kOffBar + kNumBars * 8;
  static constexpr int kOffMeta = kOffDesc + kQSlots * static_cast<int>(sizeof(Unit));
  static constexpr int kOffFlags = kOffMeta + kMetaSlots * static_cast<int>(sizeof(MetaSlot));
  // KV8: per consumer warp a 16-bit K and V staging tile
  static constexpr int kOffStg = (kOffFlags + 16 + 1023) / 1024 * 1024;
  static constexpr int kBytes = kStaging ? kOffStg + NCW * 2 * kTileBytes : kOffFlags + 16;
  static constexpr int kSmem = kBytes + 1024;  // slack to align the base to 1024 B
  static constexpr int kThreads = (NCW + 2) * 32;
  static_assert(kOffQ % 1024 == 0 && kQSlotBytes % 1024 == 0, "swizzled tiles need 1 KB alignment");
  // Inside one unit, consumer warp w takes the tiles j = w, w + NCW, ... and
  // tile j uses stage (n0 + j) % STAGES: with STAGES a multiple of NCW every
  // refill of a stage within a unit goes to the warp that drained it, so no
  // warp can wait on a stage's phase while another warp still holds the
  // previous one (across units the consumers meet at the epilogue barrier).
  static_assert(STAGES % NCW == 0, "a stage must stay with one consumer warp inside a unit");
  // two CTAs per SM up to head_dim 128 (four in the NARROW form); one at 256
  static_assert(D > 128 || kSmem <= 116 * 1024, "two CTAs per SM");
  static_assert(!NARROW || kSmem <= 56 * 1024, "four CTAs per SM");
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
};

// Byte offset, inside one 128 B-swizzled tile half, of the 16-byte chunk `ch`
// (0..7) of row `r`.  TMA's 128-byte swizzle stores chunk ch of row r at
// chunk ch ^ (r % 8).
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return static_cast<uint32_t>(r * 128 + ((ch ^ (r & 7)) << 4));
}

// Byte offset of chunk `ch` of row `r` (0..15), half `h`, in a 16-bit K/V
// tile laid out [r / 8][h][r % 8][128 B] (group stride `group_bytes`).
__device__ __forceinline__ uint32_t kv_off(int r, int h, int ch, int group_bytes) {
  return static_cast<uint32_t>((r >> 3) * group_bytes + h * 1024) + swz(r & 7, ch);
}

// Two e4m3 codes (low byte first) -> f16x2 (exact).
__device__ __forceinline__ uint32_t fp8x2_to_f16x2(uint32_t two) {
  const __half2_raw h =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xffffu), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// Four e4m3 codes -> two f16x2: codes 0, 1 into `lo`, codes 2, 3 into `hi`.
__device__ __forceinline__ void fp8x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\t"
      "mov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

__device__ __forceinline__ void lds128(uint32_t addr, uint32_t (&w)[4]) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
               : "r"(addr)
               : "memory");
}

// The 8x8 16-bit matrix whose row t / 4, columns 2 (t % 4) and + 1 lane t
// holds, transposed: lane t receives row t / 4 of the transpose.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// One FP8 tile (16 rows x D codes, row-major, as TMA lands it) -> the 16-bit
// (f16) tile layout of a 128 B-swizzled stage, [8-row group][64-dim half][8
// rows][128 B] (kv_off).  Lane l converts 16-byte groups l, l + 32, ...;
// every e4m3 value is exact in f16.
template <int D>
__device__ __forceinline__ void convert_fp8_tile(uint32_t src, uint32_t dst, int lane) {
  constexpr int kGroups = D / 16;  // 16-code groups per row
  constexpr int kGroupBytes = D / 64 * 1024;  // one 8-row group of all halves
#pragma unroll
  for (int c = lane; c < kBlock * kGroups; c += 32) {
    const int r = c / kGroups, g = c % kGroups;
    uint32_t w[4];
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "r"(src + c * 16));
    uint32_t hv[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>(w[i] & 0xffffu), __NV_E4M3);
      const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
      hv[2 * i] = static_cast<uint32_t>(lo.x) | (static_cast<uint32_t>(lo.y) << 16);
      hv[2 * i + 1] = static_cast<uint32_t>(hi.x) | (static_cast<uint32_t>(hi.y) << 16);
    }
    // codes 16g .. 16g+15 = dims of half g/4, 16-byte chunks 2(g%4) and 2(g%4)+1
    const uint32_t base = dst + (r >> 3) * kGroupBytes + (g >> 2) * 1024;
    const int ch = (g & 3) * 2;
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + swz(r & 7, ch)),
                 "r"(hv[0]), "r"(hv[1]), "r"(hv[2]), "r"(hv[3])
                 : "memory");
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + swz(r & 7, ch + 1)),
                 "r"(hv[4]), "r"(hv[5]), "r"(hv[6]), "r"(hv[7])
                 : "memory");
  }
}

template <typename T, int D, int NCW, int STAGES, bool KV8 = false, bool NARROW = false>
__global__ void __launch_bounds__((NCW + 2) * 32, NARROW ? 4 : (D > 128 ? 1 : 2))
    attn_mma_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, Shape s, T* __restrict__ out,
                    const int* __restrict__ block_tables, const int* __restrict__ qsl,
                    const int* __restrict__ seq_lens, Work w, float scale_log2,
                    const float* __restrict__ k_scale, const float* __restrict__ v_scale) {
  using L = MmaLayout<D, NCW, STAGES, KV8, NARROW>;
  // operand type of the MMAs: the input type, or f16 for an FP8 cache (every
  // e4m3 value is exact in f16; q and P are converted to it)
  using MT = typename std::conditional<KV8, __half, T>::type;
  // fp8_direct (FP8, head_dim 128): the contraction dims of QK^T are visited in
  // a permuted order that gives each lane one contiguous 16-byte run of a key
  // row per four k-steps -- lane quad q4 of k-step 4G + s takes dims
  // 64G + 16 q4 + 4s + {0,1} (fragment k 2q4, 2q4+1) and + {2,3} (k 2q4+8,
  // 2q4+9), for K and, loaded the same way, for Q.  The output dims of P.V
  // are permuted too: n-tile j, column n is head dim 16 n + j, so lane group g
  // reads the 16 bytes of dims 16g .. 16g+15 of each of its four keys.  The
  // epilogue writes every accumulator to its own head dim.
  constexpr bool fp8_direct = KV8 && !L::kStaging;
  // NARROW (FP8 direct, tiles of at most 8 rows: decode with a group of up to
  // 8 heads): P.V is taken transposed, O^T = V^T P^T, as D/16 m16n8k16 MMAs
  // whose 8 columns are the tile's rows -- half the MMAs and half the
  // accumulators of the 16-row form, whose rows 8-15 would be padding.  P^T
  // is the B operand straight from the QK^T accumulators of rows 0-7.  Row i
  // of m-tile mt is head dim 16 (i % 8) + 2 mt + i / 8, so that lane group g
  // again reads the 16 bytes of dims 16g .. 16g+15 of its four keys.
  static_assert(!NARROW || fp8_direct, "the transposed P.V is built on the FP8 direct operands");
  constexpr int KSTEPS = D / 16;  // k-steps of QK^T, also n-tile pairs of PV
  constexpr int NT = D / 8;       // PV n-tiles of 8 dims
  constexpr int NO = NARROW ? D / 16 : NT;  // accumulator tiles of O (or of O^T)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kOffBar;
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (STAGES + st); };
  auto qfull_bar = [&](int qs) { return bar0 + 8u * (2 * STAGES + qs); };
  auto qempty_bar = [&](int qs) { return bar0 + 8u * (2 * STAGES + L::kQSlots + qs); };
  auto mfull_bar = [&](int ms) { return bar0 + 8u * (2 * STAGES + 2 * L::kQSlots + ms); };
  auto mempty_bar = [&](int ms) {
    return bar0 + 8u * (2 * STAGES + 2 * L::kQSlots + kMetaSlots + ms);
  };
  const uint32_t cons_bar = bar0 + 8u * (2 * STAGES + 2 * L::kQSlots + 2 * kMetaSlots);
  Unit* desc = reinterpret_cast<Unit*>(smem + L::kOffDesc);
  MetaSlot* meta = reinterpret_cast<MetaSlot*>(smem + L::kOffMeta);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffFlags);
  float* cm = reinterpret_cast<float*>(smem + L::kOffCm);
  float* cl = reinterpret_cast<float*>(smem + L::kOffCl);
  auto co = reinterpret_cast<float(*)[L::kCoRows][D + 8]>(smem + L::kOffCo);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(full_bar(st), 1);
      mbar_init(empty_bar(st), 1);
    }
    for (int qs = 0; qs < L::kQSlots; ++qs) {
      mbar_init(qfull_bar(qs), 1);
      mbar_init(qempty_bar(qs), NCW);
    }
    for (int ms = 0; ms < kMetaSlots; ++ms) {
      mbar_init(mfull_bar(ms), 1);
      mbar_init(mempty_bar(ms), 1);
    }
    mbar_init(cons_bar, NCW);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // unused query rows of a tile must hold finite values
  for (int i = tid; i < L::kQSlots * L::kQSlotBytes / 16; i += L::kThreads)
    reinterpret_cast<uint4*>(smem + L::kOffQ)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  __syncthreads();
  // Everything above overlapped the prep kernel; its results are read below.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == NCW + 1) {
    // ----------------------------------------------------------- scheduler
    const int total_a = __ldcg(&w.sched->total_a);
    const int total = total_a + __ldcg(&w.sched->total_b);
    int cur_a = 0, cur_b = 0, j = 0;
    int next = 0;
    if (lane == 0) next = atomicAdd(&w.sched->next, 1);
    next = __shfl_sync(0xffffffffu, next, 0);
    while (true) {
      const int unit = next;
      const bool done = unit >= total;
      if (!done) {  // claim the following unit now; its value is needed next round
        int nx = 0;
        if (lane == 0) nx = atomicAdd(&w.sched->next, 1);
        next = __shfl_sync(0xffffffffu, nx, 0);
      }
      Unit un;
      int e = 0, e1 = -1;
      if (!done) {
        int local, cls;
        const int row = locate_unit_warp(s, w, total_a, unit, cur_a, cur_b, local, cls);
        const RowInfo ri = load_row(s, qsl, seq_lens, row);
        un = decode_unit(s, ri, row, local, cls);
        if (un.kv_begin >= un.kv_end) continue;  // no key of this partition is visible
        const int nblk = ceil_div(un.kv_end - un.kv_begin, kBlock);
        if (lane < nblk) {
          const int* table = block_tables + static_cast<size_t>(row) * s.table_stride;
          const int key = un.kv_begin + lane * kBlock;
          e = key_row(table, key, s.block_size, s.num_kv_heads, un.kvh, s.num_blocks, row);
          if (s.block_size < kBlock)
            e1 = key + 8 < un.kv_end ? key_row(table, key + 8, s.block_size, s.num_kv_heads,
                                               un.kvh, s.num_blocks, row)
                                     : -1;
        }
      } else {
        un.row = -1;
      }
      const int ms = j % kMetaSlots;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(mempty_bar(ms), ((j / kMetaSlots) & 1) ^ 1, kWhereWaitQ,
                                    abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      meta[ms].y0[lane] = e;
      meta[ms].y1[lane] = e1;
      if (lane == 0) meta[ms].u = un;
      __syncwarp();
      if (lane == 0) mbar_arrive(mfull_bar(ms));
      ++j;
      if (done) break;
    }
    return;
  }

  if (warp == NCW) {
    // ----------------------------------------------------------------- TMA
    // kIssueLanes lanes: lane 0 handles each unit's metadata and query tile,
    // lane i issues the unit's tiles i, i + kIssueLanes, ...  (The loads of a
    // tile keep the issuing thread busy for a few hundred cycles; with the
    // FP8 form's 4 KB stages one thread could not keep up with its consumers.)
    if (lane >= kIssueLanes) return;
    constexpr unsigned kIssueMask = (1u << kIssueLanes) - 1u;
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_q);
    }
    const uint32_t q_bytes = static_cast<uint32_t>(L::kHalves * 128 * s.gs * s.qpt);
    // issued: tiles 0 .. issued-1 all have their loads issued (for the drain)
    int n = 0, issued = 0;
    // test hook: every CTA leaves its first tile unissued (see g_debug_lost_load)
    const int lost = g_debug_lost_load == 1 ? 0 : -1;
    bool ok = true;
    for (int j = 0; ok; ++j) {
      const int ms = j % kMetaSlots;
      ok = __all_sync(kIssueMask,
                      mbar_wait(mfull_bar(ms), (j / kMetaSlots) & 1, kWhereWaitQ, abort_flag));
      if (!ok) break;
      const Unit un = meta[ms].u;
      const int qs = j & 1;
      ok = __all_sync(kIssueMask, mbar_wait(qempty_bar(qs), ((j >> 1) & 1) ^ 1, kWhereWaitQ,
                                            abort_flag));
      if (!ok) break;
      if (un.row < 0) {
        if (lane == 0) {
          desc[qs] = un;
          mbar_arrive(qfull_bar(qs));
        }
        break;
      }
      if (lane == 0) {
        desc[qs] = un;
        mbar_arrive_expect_tx(qfull_bar(qs), q_bytes);
        const uint32_t qdst = sbase + L::kOffQ + qs * L::kQSlotBytes;
#pragma unroll
        for (int h = 0; h < L::kHalves; ++h)
          tma_load_3d(qdst + h * (L::kQRows * 128), &tm_q, qfull_bar(qs), h * 64, un.head0,
                      un.token0);
      }
      const int nblk = ceil_div(un.kv_end - un.kv_begin, kBlock);
      for (int jj0 = 0; jj0 < nblk; jj0 += kIssueLanes) {
        const int jj = jj0 + lane;
        const int nn = n + jj;
        const int st = nn % STAGES;
        const bool mine = jj < nblk;
        bool r = true;
        if (mine) {
          const int y = meta[ms].y0[jj];
          r = mbar_wait(empty_bar(st), ((nn / STAGES) & 1) ^ 1, kWhereWaitEmpty, abort_flag);
          if (r && nn != lost) {
            const uint32_t kdst = sbase + st * L::kStageBytes;
            const uint32_t vdst = kdst + L::kKVTileBytes;
            if constexpr (KV8) {
              // one box of D bytes x 16 rows, or of 8 rows twice with 8-token blocks
              if (s.block_size >= kBlock) {
                mbar_arrive_expect_tx(full_bar(st), L::kStageBytes);
                tma_load_2d(kdst, &tm_k, full_bar(st), 0, y);
                tma_load_2d(vdst, &tm_v, full_bar(st), 0, y);
              } else {
                const int y1 = meta[ms].y1[jj];
                mbar_arrive_expect_tx(full_bar(st),
                                      y1 >= 0 ? L::kStageBytes : L::kStageBytes / 2);
                tma_load_2d(kdst, &tm_k, full_bar(st), 0, y);
                tma_load_2d(vdst, &tm_v, full_bar(st), 0, y);
                if (y1 >= 0) {
                  tma_load_2d(kdst + L::kKVTileBytes / 2, &tm_k, full_bar(st), 0, y1);
                  tma_load_2d(vdst + L::kKVTileBytes / 2, &tm_v, full_bar(st), 0, y1);
                }
              }
            } else if (s.block_size >= kBlock) {
              // the maps view the cache as (64 dims, 8 rows, half, row group): one
              // box of 2 row groups is the whole tile
              mbar_arrive_expect_tx(full_bar(st), L::kStageBytes);
              tma_load_4d(kdst, &tm_k, full_bar(st), 0, 0, 0, y >> 3);
              tma_load_4d(vdst, &tm_v, full_bar(st), 0, 0, 0, y >> 3);
            } else {  // 8-token blocks: one row group per block, the second if present
              const int y1 = meta[ms].y1[jj];
              mbar_arrive_expect_tx(full_bar(st), y1 >= 0 ? L::kStageBytes : L::kStageBytes / 2);
              tma_load_4d(kdst, &tm_k, full_bar(st), 0, 0, 0, y >> 3);
              tma_load_4d(vdst, &tm_v, full_bar(st), 0, 0, 0, y >> 3);
              if (y1 >= 0) {
                tma_load_4d(kdst + L::kGroupBytes, &tm_k, full_bar(st), 0, 0, 0, y1 >> 3);
                tma_load_4d(vdst + L::kGroupBytes, &tm_v, full_bar(st), 0, 0, 0, y1 >> 3);
              }
            }
          }
        }
        ok = __all_sync(kIssueMask, r);
        if (!ok) {
          // another lane gave up: this lane's tile, if issued, lands before the
          // CTA leaves (bounded again, independently of the abort flag)
          if (mine && r && nn != lost) {
            volatile int own_flag = 0;
            mbar_wait(full_bar(st), (nn / STAGES) & 1, kWhereWaitFull, &own_flag);
          }
          break;
        }
        issued = n + min(jj0 + kIssueLanes, nblk);
      }
      if (!ok) break;
      n += nblk;
      __syncwarp(kIssueMask);  // both lanes are done with the slot's block rows
      if (lane == 0) mbar_arrive(mempty_bar(ms));
    }
    if (!ok && lane == 0) {
      // A wait gave up: let the loads already issued land before leaving
      // (each wait bounded again, independently of the CTA's abort flag).
      volatile int drain_flag = 0;
      for (int st = 0; st < STAGES && st < issued; ++st) {
        const int last = issued - 1 - ((issued - 1 - st) % STAGES);
        if (last == lost) continue;  // nothing was issued for it
        if (!mbar_wait(full_bar(st), (last / STAGES) & 1, kWhereWaitFull, &drain_flag)) break;
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int r0 = lane >> 2, r1 = r0 + 8;
  const int quad = lane & 3;
  int n = 0, k = 0, syncs = 0;
  // Barrier over the consumer warps only, bounded like every other wait.
  auto consumers_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(cons_bar);
    const bool r = mbar_wait(cons_bar, syncs & 1, kWhereWaitMma, abort_flag);
    ++syncs;
    return r;
  };
  while (true) {
    const int qs = k & 1;
    const uint32_t qph = (k >> 1) & 1;
    if (!mbar_wait(qfull_bar(qs), qph, kWhereWaitQ, abort_flag)) return;
    const Unit u = desc[qs];
    if (u.row < 0) {
      // no more work for this CTA: a dependent reduce kernel may start launching
      asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
      break;
    }
    uint32_t qa[KSTEPS][4];
    if constexpr (fp8_direct) {
      const uint32_t qb = sbase + L::kOffQ + qs * L::kQSlotBytes;
      const int g = lane >> 2, q4 = lane & 3;
#pragma unroll
      for (int G = 0; G < D / 64; ++G) {
        uint32_t a0[4], a1[4], b0[4], b1[4];  // rows g, g+8; dims 16q4 .. +7, +8 .. +15
        lds128(qb + G * (L::kQRows * 128) + swz(g, 2 * q4), a0);
        lds128(qb + G * (L::kQRows * 128) + swz(g, 2 * q4 + 1), a1);
        if constexpr (NARROW) {  // the slot holds rows 0-7 only; rows 8-15 are padding
#pragma unroll
          for (int e = 0; e < 4; ++e) b0[e] = b1[e] = 0u;
        } else {
          lds128(qb + G * (L::kQRows * 128) + swz(g + 8, 2 * q4), b0);
          lds128(qb + G * (L::kQRows * 128) + swz(g + 8, 2 * q4 + 1), b1);
        }
#pragma unroll
        for (int st2 = 0; st2 < 2; ++st2) {
          const uint32_t* ra = st2 ? a1 : a0;
          const uint32_t* rb = st2 ? b1 : b0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t* f = qa[4 * G + 2 * st2 + h];
            f[0] = ra[2 * h];
            f[1] = rb[2 * h];
            f[2] = ra[2 * h + 1];
            f[3] = rb[2 * h + 1];
          }
        }
      }
    } else {
      const uint32_t qb = sbase + L::kOffQ + qs * L::kQSlotBytes;
      const int mi = lane >> 3;
      const int r = (lane & 7) + ((mi & 1) << 3);
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int ch = (kk & 3) * 2 + (mi >> 1);
        ldsm_x4(qb + (kk >> 2) * (L::kQRows * 128) + swz(r, ch), qa[kk][0], qa[kk][1], qa[kk][2],
                qa[kk][3]);
      }
    }
    if constexpr (KV8 && !std::is_same<T, __half>::value) {  // q to the f16 operand type
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack2<T>(qa[kk][e]);
          qa[kk][e] = pack2<__half>(f.x, f.y);
        }
    }
    if constexpr (NARROW) {  // rows 8-15 are padding: a zero operand, no registers
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) qa[kk][1] = qa[kk][3] = 0u;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(qempty_bar(qs));
    ++k;

    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[NO][4];
#pragma unroll
    for (int t = 0; t < NO; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    // FP8: the K scale of this KV head folds into the softmax scale
    const float sl = KV8 ? scale_log2 * __ldg(k_scale + u.kvh) : scale_log2;
    const int lim0 = u.lim0 + r0 / s.gs;
    const int lim1 = u.lim0 + r1 / s.gs;
    const int nblk = ceil_div(u.kv_end - u.kv_begin, kBlock);

    for (int j = warp; j < nblk; j += NCW) {
      const int nn = n + j;
      const int st = nn % STAGES;
      if (!mbar_wait(full_bar(st), (nn / STAGES) & 1, kWhereWaitFull, abort_flag)) return;
      uint32_t kb = sbase + st * L::kStageBytes;
      uint32_t vb = kb + L::kKVTileBytes;
      if constexpr (L::kStaging) {
        // FP8 codes -> f16 staging tiles of this warp, then the stage is free
        const uint32_t stg = sbase + L::kOffStg + warp * 2 * L::kTileBytes;
        convert_fp8_tile<D>(kb, stg, lane);
        convert_fp8_tile<D>(kb + L::kKVTileBytes, stg + L::kTileBytes, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(st));
        kb = stg;
        vb = stg + L::kTileBytes;
      }
      // FP8 direct: this lane's V bytes come into registers as soon as the
      // stage lands (keys 2q4, 2q4+1, 2q4+8, 2q4+9; head dims 16g .. 16g+15).
      // In the NARROW form the stage is then released right after QK^T, its
      // last reader; the 16-row form releases it at the end of the tile.
      uint32_t va[4], vb1[4], vc[4], vd[4];
      if constexpr (fp8_direct) {
        const int g = lane >> 2, q4 = lane & 3;
        lds128(vb + swz(2 * q4, g), va);
        lds128(vb + swz(2 * q4 + 1, g), vb1);
        lds128(vb + swz(2 * q4 + 8, g), vc);
        lds128(vb + swz(2 * q4 + 9, g), vd);
      }
      const int blk_start = u.kv_begin + j * kBlock;

      uint32_t pa[4];  // P as the A operand of P.V; NARROW: P^T's B fragments in pa[0], pa[2]
      if constexpr (NARROW) {
        // ---- S^T = K Q^T over this block's 16 keys: keys g and g + 8 (the
        // rows) of tile rows 2 quad and 2 quad + 1 (the columns) -- one MMA
        // per k-step instead of two, as rows 8-15 of the tile are padding.
        // Its A fragments are the K codes the 16-row form takes as B, its B
        // fragments Q's rows g.  Even and odd k-steps in two chains.
        const int g = lane >> 2, q4 = lane & 3;
        float sk[2][4];  // even / odd k-steps
#pragma unroll
        for (int e = 0; e < 4; ++e) sk[0][e] = sk[1][e] = 0.f;
#pragma unroll
        for (int G = 0; G < D / 64; ++G) {
          uint32_t w[2][4];  // keys g and 8 + g, dims 64G + 16 q4 .. +15
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) lds128(kb + swz(nt * 8 + g, 4 * G + q4), w[nt]);
#pragma unroll
          for (int s4 = 0; s4 < 4; ++s4) {
            uint32_t ka[4];
            fp8x4_to_f16x2x2(w[0][s4], ka[0], ka[2]);
            fp8x4_to_f16x2x2(w[1][s4], ka[1], ka[3]);
            mma_16816<MT>(sk[s4 & 1], ka, qa[4 * G + s4][0], qa[4 * G + s4][2]);
          }
        }
        // y[e]: key g + 8 (e / 2), tile row 2 quad + e % 2; m0, l0 and m1, l1
        // belong to rows 2 quad and 2 quad + 1 here
        float y[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) y[e] = (sk[0][e] + sk[1][e]) * sl;
        if (blk_start + kBlock > u.lim0) {  // some key of this block is past some row's limit
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = blk_start + g + 8 * (e >> 1);
            if (key >= u.lim0 + (2 * quad + (e & 1)) / s.gs) y[e] = -INFINITY;
          }
        }
        // the same lazy reference maximum as the 16-row form below; a row's
        // keys are spread over the eight lanes of its quad position
        const float lx0 = fmaxf(y[0], y[2]), lx1 = fmaxf(y[1], y[3]);
        if (__any_sync(0xffffffffu, lx0 > m0 + kLazyRaise || lx1 > m1 + kLazyRaise)) {
          float mx0 = lx0, mx1 = lx1;
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
          }
          const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
          const float a0 = ex2_approx(m0 - (mn0 == -INFINITY ? 0.f : mn0));
          const float a1 = ex2_approx(m1 - (mn1 == -INFINITY ? 0.f : mn1));
          l0 *= a0;
          l1 *= a1;
#pragma unroll
          for (int t = 0; t < NO; ++t) {  // O^T columns: rows 2 quad (c0, c2), 2 quad + 1
            o[t][0] *= a0;
            o[t][1] *= a1;
            o[t][2] *= a0;
            o[t][3] *= a1;
          }
          m0 = mn0;
          m1 = mn1;
        }
        const float mu0 = m0 == -INFINITY ? 0.f : m0;
        const float mu1 = m1 == -INFINITY ? 0.f : m1;
        const uint32_t plo = pack2<MT>(ex2_approx(y[0] - mu0), ex2_approx(y[1] - mu1));
        const uint32_t phi = pack2<MT>(ex2_approx(y[2] - mu0), ex2_approx(y[3] - mu1));
        const float2 flo = unpack2<MT>(plo), fhi = unpack2<MT>(phi);
        l0 += flo.x + fhi.x;  // this lane's keys; the quad positions are summed at the end
        l1 += flo.y + fhi.y;
        // P^T's B fragments (keys 2 quad, 2 quad + 1 and + 8 of tile row g):
        // the two 8x8 blocks of P^T that plo and phi hold, transposed
        pa[0] = movmatrix_t(plo);
        pa[2] = movmatrix_t(phi);
        pa[1] = pa[3] = 0u;
        // every read of this stage is done: V is in registers and the K codes
        // fed the MMAs above (each of which waited for its loads), so the
        // stage goes back to the TMA warp now rather than after P.V
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(st));
      } else {
        // ---- S = Q K^T over this block's 16 tokens
        // (two partial sums per n-tile, over even and odd k-steps: four
        // independent MMA chains instead of two halve the latency of this phase)
        float sacc[2][4], sodd[2][4];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[t][e] = sodd[t][e] = 0.f;
        if constexpr (fp8_direct) {
          const int g = lane >> 2, q4 = lane & 3;
#pragma unroll
          for (int G = 0; G < D / 64; ++G) {
            uint32_t w[2][4];  // keys g and 8+g, dims 64G + 16 q4 .. +15
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) lds128(kb + swz(nt * 8 + g, 4 * G + q4), w[nt]);
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4)
#pragma unroll
              for (int nt = 0; nt < 2; ++nt) {
                uint32_t b0, b1;
                fp8x4_to_f16x2x2(w[nt][s4], b0, b1);
                mma_16816<MT>((s4 & 1) ? sodd[nt] : sacc[nt], qa[4 * G + s4], b0, b1);
              }
          }
        } else {
          const int mi = lane >> 3;
          const int tk = (lane & 7) + ((mi >> 1) << 3);
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk) {
            uint32_t b0, b1, b2, b3;
            const int ch = (kk & 3) * 2 + (mi & 1);
            ldsm_x4(kb + kv_off(tk, kk >> 2, ch, L::kGroupBytes), b0, b1, b2, b3);
            mma_16816<MT>((kk & 1) ? sodd[0] : sacc[0], qa[kk], b0, b1);
            mma_16816<MT>((kk & 1) ? sodd[1] : sacc[1], qa[kk], b2, b3);
          }
        }
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[t][e] += sodd[t][e];
        float x[2][4];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) x[t][e] = sacc[t][e] * sl;
        if (blk_start + kBlock > u.lim0) {  // some key of this block is past some row's limit
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int key = blk_start + t * 8 + 2 * quad + (e & 1);
              if (key >= (e < 2 ? lim0 : lim1)) x[t][e] = -INFINITY;
            }
        }
        // ---- online softmax (rows r0 and r1 of this thread), against a
        // reference maximum per row that is raised only when a score of the row
        // passes it by more than 2^8 (so P <= 256, exact enough in the 16-bit
        // operand type); until then no shuffle, no rescale.
        const float lx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        const float lx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
        if (__any_sync(0xffffffffu, lx0 > m0 + kLazyRaise || lx1 > m1 + kLazyRaise)) {
          float mx0 = lx0, mx1 = lx1;
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
          const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
          // factor from the old reference to the new: 1 for rows that keep it,
          // 0 for rows that had none (m = -inf)
          const float a0 = ex2_approx(m0 - (mn0 == -INFINITY ? 0.f : mn0));
          const float a1 = ex2_approx(m1 - (mn1 == -INFINITY ? 0.f : mn1));
          l0 *= a0;
          l1 *= a1;
#pragma unroll
          for (int t = 0; t < NO; ++t) {
            o[t][0] *= a0;
            o[t][1] *= a0;
            o[t][2] *= a1;
            o[t][3] *= a1;
          }
          m0 = mn0;
          m1 = mn1;
        }
        const float mu0 = m0 == -INFINITY ? 0.f : m0;
        const float mu1 = m1 == -INFINITY ? 0.f : m1;
        pa[0] = pack2<MT>(ex2_approx(x[0][0] - mu0), ex2_approx(x[0][1] - mu0));
        pa[1] = pack2<MT>(ex2_approx(x[0][2] - mu1), ex2_approx(x[0][3] - mu1));
        pa[2] = pack2<MT>(ex2_approx(x[1][0] - mu0), ex2_approx(x[1][1] - mu0));
        pa[3] = pack2<MT>(ex2_approx(x[1][2] - mu1), ex2_approx(x[1][3] - mu1));
        // the normaliser sums the same rounded weights the P.V product uses
        const float2 p00 = unpack2<MT>(pa[0]), p01 = unpack2<MT>(pa[1]);
        const float2 p10 = unpack2<MT>(pa[2]), p11 = unpack2<MT>(pa[3]);
        l0 += (p00.x + p00.y) + (p10.x + p10.y);
        l1 += (p01.x + p01.y) + (p11.x + p11.y);
      }
      // ---- O += P V ; V rows at or past the unit's last visible key are
      // zeroed (padding may hold anything, and 0 * NaN is NaN)
      uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
      if (blk_start + kBlock > u.kv_end) {
        const int nv = u.kv_end - blk_start, t0 = 2 * quad;
        vm0 = (t0 < nv ? 0x0000ffffu : 0u) | (t0 + 1 < nv ? 0xffff0000u : 0u);
        vm1 = (t0 + 8 < nv ? 0x0000ffffu : 0u) | (t0 + 9 < nv ? 0xffff0000u : 0u);
      }
      if constexpr (NARROW) {  // O^T += V^T P^T, V^T from the bytes loaded above
        auto pvn = [&](bool masked) {
#pragma unroll
          for (int mt = 0; mt < NO; ++mt) {
            // bytes 2(mt%2), +1 of word mt/2: dims 16g + 2mt (rows g) and
            // 16g + 2mt + 1 (rows g + 8) of keys 2q4, 2q4+1 and 2q4+8, 2q4+9
            const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
            uint32_t av[4];
            fp8x4_to_f16x2x2(prmt(va[mt >> 1], vb1[mt >> 1], sel), av[0], av[1]);
            fp8x4_to_f16x2x2(prmt(vc[mt >> 1], vd[mt >> 1], sel), av[2], av[3]);
            if (masked) {
              av[0] &= vm0;
              av[1] &= vm0;
              av[2] &= vm1;
              av[3] &= vm1;
            }
            mma_16816<MT>(o[mt], av, pa[0], pa[2]);
          }
        };
        if (blk_start + kBlock > u.kv_end)  // padding rows: only the last tile has them
          pvn(true);
        else
          pvn(false);
      } else if constexpr (fp8_direct) {  // V from the bytes loaded above
        auto pv8 = [&](bool masked) {
#pragma unroll
          for (int jw = 0; jw < 4; ++jw) {
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {  // bytes 2hb, 2hb+1 of word jw: n-tiles 4jw+2hb, +1
              const uint32_t sel = hb ? 0x7362u : 0x5140u;
              uint32_t l0, l1, h0, h1;  // (key 2q4, 2q4+1) and (key 2q4+8, 2q4+9), two dims
              fp8x4_to_f16x2x2(prmt(va[jw], vb1[jw], sel), l0, l1);
              fp8x4_to_f16x2x2(prmt(vc[jw], vd[jw], sel), h0, h1);
              if (masked) {
                l0 &= vm0;
                l1 &= vm0;
                h0 &= vm1;
                h1 &= vm1;
              }
              const int j = 4 * jw + 2 * hb;
              mma_16816<MT>(o[j], pa, l0, h0);
              mma_16816<MT>(o[j + 1], pa, l1, h1);
            }
          }
        };
        if (blk_start + kBlock > u.kv_end)  // padding rows: only the last tile has them
          pv8(true);
        else
          pv8(false);
      } else {
        const int mi = lane >> 3;
        const int tk = (lane & 7) + ((mi & 1) << 3);
        auto pv16 = [&](bool masked) {
#pragma unroll
          for (int jj = 0; jj < KSTEPS; ++jj) {
            uint32_t b0, b1, b2, b3;
            const int ch = (jj & 3) * 2 + (mi >> 1);
            ldsm_x4_t(vb + kv_off(tk, jj >> 2, ch, L::kGroupBytes), b0, b1, b2, b3);
            if (masked) {
              b0 &= vm0;
              b1 &= vm1;
              b2 &= vm0;
              b3 &= vm1;
            }
            mma_16816<MT>(o[2 * jj], pa, b0, b1);
            mma_16816<MT>(o[2 * jj + 1], pa, b2, b3);
          }
        };
        if (blk_start + kBlock > u.kv_end)  // padding rows: only the last tile has them
          pv16(true);
        else
          pv16(false);
      }
      __syncwarp();  // (FP8 through staging: every lane is done with the staging tiles)
      if (!L::kStaging && !NARROW && lane == 0) mbar_arrive(empty_bar(st));
    }
    n += nblk;

    if constexpr (KV8) {  // the V scale of this KV head
      const float vsc = __ldg(v_scale + u.kvh);
#pragma unroll
      for (int t = 0; t < NO; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[t][e] *= vsc;
    }
    // ---- merge the warps' states
    if constexpr (NARROW) {  // rows 2 quad, 2 quad + 1; keys over the eight lanes g
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      }
      if (lane < 4) {
        cm[warp * L::kCoRows + 2 * quad] = m0;
        cl[warp * L::kCoRows + 2 * quad] = l0;
        cm[warp * L::kCoRows + 2 * quad + 1] = m1;
        cl[warp * L::kCoRows + 2 * quad + 1] = l1;
      }
    } else {
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      if (quad == 0) {
        cm[warp * kRows + r0] = m0;
        cl[warp * kRows + r0] = l0;
        cm[warp * kRows + r1] = m1;
        cl[warp * kRows + r1] = l1;
      }
    }
    if constexpr (NARROW) {
      // m-tile mt holds dims 16g + 2mt (c0, c1) and 16g + 2mt + 1 (c2, c3) of
      // rows 2 quad (c0, c2) and 2 quad + 1 (c1, c3)
#pragma unroll
      for (int rs = 0; rs < 2; ++rs)
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          *reinterpret_cast<float4*>(&co[warp][2 * quad + rs][16 * r0 + 4 * c4]) =
              make_float4(o[2 * c4][rs], o[2 * c4][2 + rs], o[2 * c4 + 1][rs],
                          o[2 * c4 + 1][2 + rs]);
    } else if constexpr (fp8_direct) {
      // n-tile t, columns 2q, 2q+1 hold head dims 32q + t and 32q + 16 + t: this
      // lane has dims 32q .. 32q+31 of rows r0 and r1, stored as eight float4
      // chunks per row in the swizzled layout (conflict-free; plain offsets put
      // the four quads of a warp on one bank)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int h = kk >> 2, t0 = 4 * (kk & 3);
        const int off = co_swizzled(8 * quad + kk);
        *reinterpret_cast<float4*>(&co[warp][r0][off]) =
            make_float4(o[t0][h], o[t0 + 1][h], o[t0 + 2][h], o[t0 + 3][h]);
        *reinterpret_cast<float4*>(&co[warp][r1][off]) =
            make_float4(o[t0][2 + h], o[t0 + 1][2 + h], o[t0 + 2][2 + h], o[t0 + 3][2 + h]);
      }
    } else {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        *reinterpret_cast<float2*>(&co[warp][r0][t * 8 + 2 * quad]) =
            make_float2(o[t][0], o[t][1]);
        *reinterpret_cast<float2*>(&co[warp][r1][t * 8 + 2 * quad]) =
            make_float2(o[t][2], o[t][3]);
      }
    }
    if (!consumers_sync()) return;
    epilogue<T, D, NCW, fp8_direct && !NARROW, L::kCoRows>(s, u, cm, cl, co, out, w, tid,
                                                           NCW * 32);
    if (!consumers_sync()) return;
  }
}

}  // namespace pa
