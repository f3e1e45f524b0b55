// Paged attention on sm_100a: TMA-staged K/V tiles + warp-level tensor-core MMA.
//
// Persistent, warp-specialised CTA (NCW consumer warps + 1 producer warp):
//
// * The producer walks this CTA's work units (pa_sched.cuh), looks each
//   logical block up in the request's block-table row ("vLLM 深度拆解" §3.3:
//   physical = block_tables[seq*stride + logical]) and issues
//   cp.async.bulk.tensor loads of the (block, KV head) K tile and V tile --
//   16 tokens x head_dim, 4 KB each at bf16 x 128 -- into a STAGES-deep ring
//   of shared-memory stages, completed on mbarriers.  It also loads the tile's
//   query rows.  The tensor maps use 128-byte swizzling so the ldmatrix reads
//   below are free of bank conflicts.  Nothing else sits between HBM and the
//   MMA, and no load waits for compute: the ring keeps up to STAGES * 8 KB in
//   flight per CTA.
// * Consumer warp w takes the unit's blocks w, w+NCW, ...  For each block it
//   computes S = Q K^T (16 tile rows x 16 tokens, m16n8k16 MMAs, fp32
//   accumulate), masks keys past each row's limit, updates its online softmax
//   in the log2 domain (running max m, sum l), rounds P to the input type and
//   accumulates O += P V with the same MMA.  A whole GQA group (up to 16 query
//   heads) shares one K/V tile, so each KV block is read once per KV head.
// * At the end of a unit the consumer warps merge their (m, l, O) states and
//   write the output row, or the partition's partial for the split-K reduce.
#pragma once

#include "pa_sched.cuh"

namespace pa {

template <int D, int NCW, int STAGES>
struct MmaLayout {
  static constexpr int kHalves = D / 64;             // 64 16-bit elements = one 128 B swizzle row
  static constexpr int kHalfBytes = kBlock * 128;    // 16 rows x 128 B
  static constexpr int kTileBytes = kHalves * kHalfBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;  // K tile then V tile
  static constexpr int kQSlotBytes = kHalves * kRows * 128;
  static constexpr int kQSlots = 2;
  static constexpr int kOffQ = STAGES * kStageBytes;
  static constexpr int kOffCo = kOffQ + kQSlots * kQSlotBytes;
  static constexpr int kCoBytes = NCW * kRows * (D + 8) * 4;
  static constexpr int kOffCm = kOffCo + kCoBytes;
  static constexpr int kOffCl = kOffCm + NCW * kRows * 4;
  static constexpr int kOffBar = kOffCl + NCW * kRows * 4;
  static constexpr int kNumBars = 2 * STAGES + 2 * kQSlots + 1;  // + consumer barrier
  static constexpr int kOffDesc = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffDesc + kQSlots * static_cast<int>(sizeof(Unit));
  static constexpr int kBytes = kOffAbort + 16;
  static constexpr int kSmem = kBytes + 1024;  // slack to align the base to 1024 B
  static_assert(kOffQ % 1024 == 0 && kQSlotBytes % 1024 == 0, "swizzled tiles need 1 KB alignment");
};

// Byte offset, inside one 128 B-swizzled tile half, of the 16-byte chunk `ch`
// (0..7) of row `r`.  TMA's 128-byte swizzle stores chunk ch of row r at
// chunk ch ^ (r % 8).
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return static_cast<uint32_t>(r * 128 + ((ch ^ (r & 7)) << 4));
}

template <typename T, int D, int NCW, int STAGES>
__global__ void __launch_bounds__((NCW + 1) * 32, 2)
    attn_mma_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, Shape s, T* __restrict__ out,
                    const int* __restrict__ block_tables, const int* __restrict__ qsl,
                    const int* __restrict__ seq_lens, const int* __restrict__ row_start,
                    float scale_log2, float* __restrict__ part_o, float* __restrict__ part_lse) {
  using L = MmaLayout<D, NCW, STAGES>;
  constexpr int KSTEPS = D / 16;  // k-steps of QK^T, also n-tile pairs of PV
  constexpr int NT = D / 8;       // PV n-tiles of 8 dims
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kOffBar;
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (STAGES + st); };
  auto qfull_bar = [&](int qs) { return bar0 + 8u * (2 * STAGES + qs); };
  auto qempty_bar = [&](int qs) { return bar0 + 8u * (2 * STAGES + L::kQSlots + qs); };
  const uint32_t cons_bar = bar0 + 8u * (2 * STAGES + 2 * L::kQSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  Unit* desc = reinterpret_cast<Unit*>(smem + L::kOffDesc);
  float* cm = reinterpret_cast<float*>(smem + L::kOffCm);
  float* cl = reinterpret_cast<float*>(smem + L::kOffCl);
  auto co = reinterpret_cast<float(*)[kRows][D + 8]>(smem + L::kOffCo);

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
    mbar_init(cons_bar, NCW);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // unused query rows of a tile must hold finite values
  for (int i = tid; i < L::kQSlots * L::kQSlotBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + L::kOffQ)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  __syncthreads();

  const int total = row_start[s.num_seqs];

  if (warp == NCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_q);
    }
    const uint32_t q_bytes = static_cast<uint32_t>(L::kHalves * 128 * s.gs * s.qpt);
    int n = 0, k = 0, cursor = 0, issued = 0;
    bool ok = true;
    for (int unit = blockIdx.x; ok; unit += gridDim.x) {
      const bool done = unit >= total;
      Unit un;
      if (!done) {
        int start;
        const int row = find_row_warp(row_start, s.num_seqs, unit, cursor, start);
        cursor = row;
        const RowInfo ri = load_row(s, qsl, seq_lens, row);
        un = decode_unit(s, ri, row, unit - start);
        if (un.kv_begin >= un.kv_end) continue;  // no key of this partition is visible
      } else {
        un.row = -1;
      }
      const int qs = k & 1;
      const uint32_t qph = (k >> 1) & 1;
      if (lane == 0) {
        ok = mbar_wait(qempty_bar(qs), qph ^ 1, kWhereWaitQ, abort_flag);
        if (ok) {
          desc[qs] = un;
          if (done) {
            mbar_arrive(qfull_bar(qs));
          } else {
            mbar_arrive_expect_tx(qfull_bar(qs), q_bytes);
            const uint32_t qdst = sbase + L::kOffQ + qs * L::kQSlotBytes;
#pragma unroll
            for (int h = 0; h < L::kHalves; ++h)
              tma_load_3d(qdst + h * (kRows * 128), &tm_q, qfull_bar(qs), h * 64, un.head0,
                          un.token0);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++k;
      if (done || !ok) break;
      const int nblk = ceil_div(un.kv_end - un.kv_begin, kBlock);
      const int* table = block_tables + static_cast<size_t>(un.row) * s.table_stride +
                         un.kv_begin / kBlock;
      for (int c = 0; c < nblk && ok; c += 32) {
        int e = 0;
        if (c + lane < nblk) {
          e = __ldg(table + c + lane);
          if (e < 0 || e >= s.num_blocks) {
            report_error(PA_ERR_DEVICE_BOUNDS, kWhereBlockId, un.row, e);
            e = 0;
          }
        }
        const int cnt = min(32, nblk - c);
        for (int jj = 0; jj < cnt; ++jj) {
          const int pb = __shfl_sync(0xffffffffu, e, jj);
          if (lane == 0 && ok) {
            const int st = n % STAGES;
            const uint32_t ph = (n / STAGES) & 1;
            ok = mbar_wait(empty_bar(st), ph ^ 1, kWhereWaitEmpty, abort_flag);
            if (ok) {
              ++issued;
              mbar_arrive_expect_tx(full_bar(st), L::kStageBytes);
              const int y = (pb * s.num_kv_heads + un.kvh) * kBlock;
              const uint32_t kdst = sbase + st * L::kStageBytes;
#pragma unroll
              for (int h = 0; h < L::kHalves; ++h) {
                tma_load_2d(kdst + h * L::kHalfBytes, &tm_k, full_bar(st), h * 64, y);
                tma_load_2d(kdst + L::kTileBytes + h * L::kHalfBytes, &tm_v, full_bar(st), h * 64,
                            y);
              }
            }
          }
          ++n;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    if (!ok && lane == 0) {
      // A wait gave up: let the loads already issued land before leaving
      // (each wait bounded again, independently of the CTA's abort flag).
      volatile int drain_flag = 0;
      for (int st = 0; st < STAGES && st < issued; ++st) {
        const int last = issued - 1 - ((issued - 1 - st) % STAGES);
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
    if (u.row < 0) break;
    uint32_t qa[KSTEPS][4];
    {
      const uint32_t qb = sbase + L::kOffQ + qs * L::kQSlotBytes;
      const int mi = lane >> 3;
      const int r = (lane & 7) + ((mi & 1) << 3);
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int ch = (kk & 3) * 2 + (mi >> 1);
        ldsm_x4(qb + (kk >> 2) * (kRows * 128) + swz(r, ch), qa[kk][0], qa[kk][1], qa[kk][2],
                qa[kk][3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(qempty_bar(qs));
    ++k;

    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    const int lim0 = u.lim0 + r0 / s.gs;
    const int lim1 = u.lim0 + r1 / s.gs;
    const int nblk = ceil_div(u.kv_end - u.kv_begin, kBlock);

    for (int j = warp; j < nblk; j += NCW) {
      const int nn = n + j;
      const int st = nn % STAGES;
      if (!mbar_wait(full_bar(st), (nn / STAGES) & 1, kWhereWaitFull, abort_flag)) return;
      const uint32_t kb = sbase + st * L::kStageBytes;
      const uint32_t vb = kb + L::kTileBytes;
      const int blk_start = u.kv_begin + j * kBlock;

      // ---- S = Q K^T over this block's 16 tokens
      float sacc[2][4];
#pragma unroll
      for (int t = 0; t < 2; ++t) sacc[t][0] = sacc[t][1] = sacc[t][2] = sacc[t][3] = 0.f;
      {
        const int mi = lane >> 3;
        const int tk = (lane & 7) + ((mi >> 1) << 3);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          uint32_t b0, b1, b2, b3;
          const int ch = (kk & 3) * 2 + (mi & 1);
          ldsm_x4(kb + (kk >> 2) * L::kHalfBytes + swz(tk, ch), b0, b1, b2, b3);
          mma_16816<T>(sacc[0], qa[kk], b0, b1);
          mma_16816<T>(sacc[1], qa[kk], b2, b3);
        }
      }
      float x[2][4];
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) x[t][e] = sacc[t][e] * scale_log2;
      if (blk_start + kBlock > u.lim0) {  // some key of this block is past some row's limit
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = blk_start + t * 8 + 2 * quad + (e & 1);
            if (key >= (e < 2 ? lim0 : lim1)) x[t][e] = -INFINITY;
          }
      }
      // ---- online softmax (rows r0 and r1 of this thread)
      float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
      const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
      const float a0 = exp2f(m0 - mu0), a1 = exp2f(m1 - mu1);
      uint32_t pa[4];
      pa[0] = pack2<T>(exp2f(x[0][0] - mu0), exp2f(x[0][1] - mu0));
      pa[1] = pack2<T>(exp2f(x[0][2] - mu1), exp2f(x[0][3] - mu1));
      pa[2] = pack2<T>(exp2f(x[1][0] - mu0), exp2f(x[1][1] - mu0));
      pa[3] = pack2<T>(exp2f(x[1][2] - mu1), exp2f(x[1][3] - mu1));
      // the normaliser sums the same rounded weights the P.V product uses
      const float2 p00 = unpack2<T>(pa[0]), p01 = unpack2<T>(pa[1]);
      const float2 p10 = unpack2<T>(pa[2]), p11 = unpack2<T>(pa[3]);
      l0 = l0 * a0 + ((p00.x + p00.y) + (p10.x + p10.y));
      l1 = l1 * a1 + ((p01.x + p01.y) + (p11.x + p11.y));
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        o[t][0] *= a0;
        o[t][1] *= a0;
        o[t][2] *= a1;
        o[t][3] *= a1;
      }
      // ---- O += P V ; V rows at or past the unit's last visible key are
      // zeroed (padding may hold anything, and 0 * NaN is NaN)
      uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
      if (blk_start + kBlock > u.kv_end) {
        const int nv = u.kv_end - blk_start, t0 = 2 * quad;
        vm0 = (t0 < nv ? 0x0000ffffu : 0u) | (t0 + 1 < nv ? 0xffff0000u : 0u);
        vm1 = (t0 + 8 < nv ? 0x0000ffffu : 0u) | (t0 + 9 < nv ? 0xffff0000u : 0u);
      }
      {
        const int mi = lane >> 3;
        const int tk = (lane & 7) + ((mi & 1) << 3);
#pragma unroll
        for (int jj = 0; jj < KSTEPS; ++jj) {
          uint32_t b0, b1, b2, b3;
          const int ch = (jj & 3) * 2 + (mi >> 1);
          ldsm_x4_t(vb + (jj >> 2) * L::kHalfBytes + swz(tk, ch), b0, b1, b2, b3);
          mma_16816<T>(o[2 * jj], pa, b0 & vm0, b1 & vm1);
          mma_16816<T>(o[2 * jj + 1], pa, b2 & vm0, b3 & vm1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(st));
    }
    n += nblk;

    // ---- merge the warps' states
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
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      *reinterpret_cast<float2*>(&co[warp][r0][t * 8 + 2 * quad]) = make_float2(o[t][0], o[t][1]);
      *reinterpret_cast<float2*>(&co[warp][r1][t * 8 + 2 * quad]) = make_float2(o[t][2], o[t][3]);
    }
    if (!consumers_sync()) return;
    combine_and_store<T, D, NCW>(s, u, cm, cl, co, out, part_o, part_lse, tid);
    if (!consumers_sync()) return;
  }
}

}  // namespace pa
