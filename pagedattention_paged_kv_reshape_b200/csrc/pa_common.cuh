// Device-side building blocks shared by the paged-attention kernels (sm_100a).
//
// * the per-device error word that kernels use instead of faulting,
// * mbarrier / TMA (cp.async.bulk.tensor) wrappers with bounded waits,
// * ldmatrix and warp-level bf16/f16 MMA wrappers,
// * 16-bit <-> fp32 packing helpers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "pa.h"

namespace pa {

// Tokens per physical block ("vLLM 架构源码解析" §1.1: 16 tokens by default).
// Keys are processed in tiles of kBlock = 16 consecutive tokens whatever the
// physical block size: a 32-token block holds two such tiles, an 8-token
// block half of one (key_row below finds a key's row in the cache).
constexpr int kBlock = 16;
// Tokens per split-K partition.  Contexts longer than this are cut into
// partitions whose partial softmax states are merged by log-sum-exp.
constexpr int kPart = 512;
// Query rows (query token x query head pairs) one tile of the MMA kernel holds.
constexpr int kRows = 16;

// ---------------------------------------------------------------------------
// Device error word.  The first kernel that meets bad metadata or a wait that
// ran out records (code, where, a, b); later events are dropped.  The host
// reads and clears it with pa_get_device_error.
// ---------------------------------------------------------------------------
struct DeviceError {
  unsigned int code;
  int where;
  long long a;
  long long b;
};

__device__ DeviceError g_device_error;

enum ErrWhere : int {
  kWhereReshapeSlot = 1,
  kWhereBlockId = 2,
  kWhereRowMeta = 3,
  kWhereWaitFull = 4,
  kWhereWaitEmpty = 5,
  kWhereWaitQ = 6,
  kWhereTmem = 7,
  kWhereWaitMma = 8,
  kWhereCopyPair = 9,
  kWhereRopePos = 10,
};

__device__ __forceinline__ void report_error(unsigned code, int where, long long a, long long b) {
  if (atomicCAS(&g_device_error.code, 0u, code) == 0u) {
    g_device_error.where = where;
    g_device_error.a = a;
    g_device_error.b = b;
    __threadfence();
  }
}

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers, bounded waits.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// About one second at the B200's top SM clock: a wait that lasts longer than
// this means a lost arrival, never slow memory.
constexpr long long kWaitLimitCycles = 2000000000LL;

// The limit every bounded wait uses (SM cycles).  kWaitLimitCycles unless a
// test shortened it with pa_debug_lost_load.
__device__ long long g_wait_limit_cycles = kWaitLimitCycles;

// Test hook, 0 in normal operation (pa_debug_lost_load): 1 makes the load
// warp of every CTA of attn_mma_kernel, 2 that of chunk_tc2_kernel, leave its
// first K/V tile unissued (no copy and no arrival on its barrier), so the
// warp that waits for that tile runs into the wait limit.
__device__ int g_debug_lost_load = 0;

// Wait for the phase with the given parity to complete.  Returns false, after
// recording PA_ERR_TIMEOUT and raising the CTA's abort flag, if it did not
// complete within g_wait_limit_cycles; returns false at once if another warp
// of the CTA already raised the flag.  Every wait in these kernels goes
// through here, so no CTA can wait without bound.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int where,
                                          volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  const long long limit = g_wait_limit_cycles;
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      report_error(PA_ERR_TIMEOUT, where, bar, parity);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// Row of key `key` of a request, in the cache viewed as rows of head_dim
// elements: physical block table[key / block_size], KV head kvh, slot
// key % block_size ("vLLM 深度拆解" §3.3: block_tables[seq * stride +
// block_idx]).  An entry outside [0, num_blocks) is recorded and replaced by
// block 0, so the access stays inside the pool.
__device__ __forceinline__ int key_row(const int* __restrict__ table, int key, int block_size,
                                       int num_kv_heads, int kvh, int num_blocks, int row) {
  const int shift = __ffs(block_size) - 1;  // block sizes are powers of two
  int pb = __ldg(table + (key >> shift));
  if (pb < 0 || pb >= num_blocks) {
    report_error(PA_ERR_DEVICE_BOUNDS, kWhereBlockId, row, pb);
    pb = 0;
  }
  return (pb * num_kv_heads + kvh) * block_size + (key & (block_size - 1));
}

// ---------------------------------------------------------------------------
// TMA tensor loads (no multicast).  The tensor map lives in kernel parameter
// space (__grid_constant__); coordinates are element indices, innermost first.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int x, int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// 2^x on the special-function unit (flushes subnormal results to zero;
// 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 32 bytes to global memory in one store (the address 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Bring the box at (x, y, z) of a tensor map into L2, without a destination
// in shared memory or a barrier.
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------------------
// ldmatrix / mma.sync (m16n8k16, fp32 accumulate)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

template <typename T>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1);

template <>
__device__ __forceinline__ void mma_16816<__nv_bfloat16>(float (&d)[4], const uint32_t (&a)[4],
                                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <>
__device__ __forceinline__ void mma_16816<__half>(float (&d)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// 16-bit packing.  Element `lo` goes to the low half (lower address).
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);

template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <typename T>
__device__ __forceinline__ float2 unpack2(uint32_t v);

template <>
__device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t v) {
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

template <>
__device__ __forceinline__ float2 unpack2<__half>(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace pa
