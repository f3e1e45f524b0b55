// Whole-block copies between KV pools: copy-on-write inside one pool and
// swapping between the device pool and a pool in page-locked host memory.
//
// * Copy-on-write: blocks are shared by reference count ("2. 核心思想"
//   §核心抽象: ref_cnt supports copy-on-write and sharing across requests;
//   "vLLM 架构源码解析" §4.3.2: parallel samples share the prompt's blocks);
//   before a request writes into a block another request still references,
//   the engine gives it a private copy of that block.
// * Swap: the v0 scheduler preempts a request by swapping its KV cache out to
//   CPU memory and swaps it back in when the request resumes
//   ("vLLM 架构源码解析" §1, the preemption table: v0 (Swap)).
//
// Both are the same operation: for each pair i, physical block map[2i+1] of
// the destination pools becomes a byte copy of block map[2i] of the source
// pools, for K and for V, every KV head and every slot.  A block of one pool
// is one contiguous run of num_kv_heads * block_size * head_dim elements, so
// the copy is a plain 16-byte-vector stream.  Host memory is reached through
// its device-visible address (unified addressing of page-locked memory), so
// one kernel serves both directions and needs no per-block copy calls.
#pragma once

#include "pa_common.cuh"

namespace pa {

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;  // 16-byte loads in flight per thread

// grid.x: (pair, chunk of kCopyThreads * kCopyUnroll vectors of one block),
// grid.y: 0 = K, 1 = V.
__global__ void __launch_bounds__(kCopyThreads)
    copy_blocks_kernel(const uint4* __restrict__ src_k, const uint4* __restrict__ src_v,
                       uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                       const int* __restrict__ map, int src_blocks, int dst_blocks,
                       int block_vecs, int chunks) {
  const int pair = blockIdx.x / chunks, chunk = blockIdx.x % chunks;
  const int src = map[2 * pair], dst = map[2 * pair + 1];
  if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
    if (threadIdx.x == 0 && chunk == 0 && blockIdx.y == 0)
      report_error(PA_ERR_DEVICE_BOUNDS, kWhereCopyPair, pair,
                   src < 0 || src >= src_blocks ? src : dst);
    return;
  }
  const uint4* s = (blockIdx.y == 0 ? src_k : src_v) + static_cast<size_t>(src) * block_vecs;
  uint4* d = (blockIdx.y == 0 ? dst_k : dst_v) + static_cast<size_t>(dst) * block_vecs;
  if (s == d) return;
  const int base = chunk * kCopyThreads * kCopyUnroll + threadIdx.x;
  uint4 v[kCopyUnroll];
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int i = base + u * kCopyThreads;
    if (i < block_vecs) v[u] = s[i];
  }
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int i = base + u * kCopyThreads;
    if (i < block_vecs) d[i] = v[u];
  }
}

}  // namespace pa
