// Host side of the C ABI declared in include/pa.h: argument checks, workspace
// carving, TMA tensor-map encoding, kernel choice and launches.  Every entry
// point validates on the host before touching the device, returns a status
// and never synchronises (except pa_get_device_error).
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "pa_attn_mma.cuh"
#include "pa_attn_simt.cuh"
#include "pa_blocks.cuh"
#include "pa_chunk_tc1.cuh"
#include "pa_chunk_tc2.cuh"
#include "pa_reduce.cuh"

#include "pa_reshape.cuh"
#include "pa_sched.cuh"

namespace {

thread_local std::string g_msg;
std::atomic<int> g_path{PA_PATH_AUTO};

pa_status fail(pa_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
pa_status fail(pa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_msg = buf;
  return st;
}

pa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int elem_bytes(pa_dtype dt) { return dt == PA_F32 ? 4 : dt == PA_E4M3 ? 1 : 2; }

bool valid_dtype(int dt) { return dt == PA_F32 || dt == PA_BF16 || dt == PA_F16; }

int sm_count() {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  cache[dev] = n;
  return n;
}

// Set the dynamic shared-memory limit of a kernel and return its occupancy,
// once per (kernel, device).
template <typename K>
cudaError_t prepare(K kernel, int threads, int smem, int* occ) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *occ = it->second;
    return cudaSuccess;
  }
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, kernel, threads, smem);
  if (e != cudaSuccess) return e;
  if (*occ < 1) return cudaErrorInvalidConfiguration;
  cache[key] = *occ;
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime, so the
// library does not link libcuda directly).
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D view of a 16-bit K or V cache of `rows` rows x d elements (rows a
// multiple of 8): (64 elements of a half, row within a group of 8, half,
// row group), strides 2 B, d * 2 B, 128 B, 8 * d * 2 B.  A box {64, 8, d/64,
// groups} lands in shared memory as [group][half][8 rows][128 B], 128 B-swizzled.
pa_status make_map_kv(CUtensorMap* map, const void* base, pa_dtype dt, uint64_t d,
                      uint64_t rows, uint32_t groups) {
  auto fn = encode_fn();
  if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[4] = {64, 8, d / 64, rows / 8};
  const cuuint64_t strides[3] = {d * 2, 128, 8 * d * 2};
  const cuuint32_t box[4] = {64, 8, static_cast<cuuint32_t>(d / 64), groups};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, dt == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (kv) failed: %d", r);
  return PA_OK;
}

// 2-D view [rows][inner] of a 1-byte tensor (FP8 codes), box {inner, box_rows};
// 128-byte rows are 128 B-swizzled (the consumers read them with swizzled
// 16-byte loads), 64-byte rows are not.
pa_status make_map_2d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                         uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(inner), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        inner == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (u8) failed: %d", r);
  return PA_OK;
}

// 3-D view [d2][d1][inner] of a 16-bit tensor, box {64, b1, b2}, 128 B swizzle.
pa_status make_map_3d(CUtensorMap* map, const void* base, pa_dtype dt, uint64_t inner,
                      uint64_t d1, uint64_t d2, uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[3] = {inner, d1, d2};
  const cuuint64_t strides[2] = {inner * 2, inner * d1 * 2};
  const cuuint32_t box[3] = {64, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, dt == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (3d) failed: %d", r);
  return PA_OK;
}

// ---------------------------------------------------------------------------
// Attention (decode and varlen share everything below)
// ---------------------------------------------------------------------------
struct AttnArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  int table_stride;
  const int32_t* qsl;  // null for decode
  const int32_t* seq_lens;
  int num_seqs, total_q, max_query_len, max_seq_len;
  int num_q_heads, num_kv_heads, head_dim, block_size, num_blocks;
  float scale;
  void* workspace;
  size_t workspace_bytes;
  pa_dtype dtype;
  cudaStream_t stream;
  // FP8 (e4m3) cache: per-KV-head scales of K and V; null for a 16/32-bit cache
  const float* k_scale = nullptr;
  const float* v_scale = nullptr;
  bool kv8() const { return k_scale != nullptr; }
};

#ifndef PA_STAGES
#define PA_STAGES 8  // K/V stages of 8 KB per CTA (two CTAs per SM)
#endif
constexpr int kNcw = 4;
constexpr int kStages = PA_STAGES;

struct Plan {
  pa::Shape s;
  size_t off_row_a, off_row_b, off_chunk, off_part_lse, off_part_o, bytes;
  long long max_units;
  int chunk_qt;         // query tokens per tcgen05 chunk tile (0: no chunk kernel possible)
  long long chunk_cap;  // capacity of the chunk-tile list
};

// The tcgen05 chunk kernel tiles 128 rows = (128 / gs) query tokens x gs heads.
int chunk_tile_tokens(int group) {
  const int gs = group < pa::kRows ? group : pa::kRows;
  return (gs == 1 || gs == 2 || gs == 4 || gs == 8 || gs == 16) ? pa::kTcRows / gs : 0;
}

// Workspace layout: the schedule block (Sched), the two per-row unit prefixes,
// the chunk-tile list (varlen batches whose head grouping the tcgen05 kernel
// supports), then the split-K partials (only when some context can exceed
// one partition).
Plan make_plan(int num_seqs, int total_q, int hq, int hkv, int d, int max_len, bool varlen) {
  Plan p{};
  pa::Shape& s = p.s;
  s.num_seqs = num_seqs;
  s.num_q_heads = hq;
  s.num_kv_heads = hkv;
  s.group = hkv > 0 ? hq / hkv : 1;
  s.gs = s.group < pa::kRows ? s.group : pa::kRows;
  s.ns = (s.group + pa::kRows - 1) / pa::kRows;
  s.qpt = varlen ? (pa::kRows / s.gs > 0 ? pa::kRows / s.gs : 1) : 1;
  s.head_dim = d;
  s.total_q = total_q;
  s.p_stride = max_len > 0 ? (max_len + pa::kPart - 1) / pa::kPart : 1;
  s.chunk_qt = 0;
  s.chunk_cap = 0;
  s.chunk_span = 0;
  const size_t rows = static_cast<size_t>(num_seqs) + 1;
  p.off_row_a = sizeof(pa::Sched);
  p.off_row_b = p.off_row_a + rows * 4;
  size_t off = align256(p.off_row_b + rows * 4);
  p.off_chunk = off;
  p.chunk_qt = varlen ? chunk_tile_tokens(s.group) : 0;
  if (p.chunk_qt > 0) {  // a chunk row of q_len tokens yields ceil(q_len / qt) <= 2 q_len / qt tiles
    p.chunk_cap = 2LL * ((total_q + p.chunk_qt - 1) / p.chunk_qt) + 1;
    off = align256(off + static_cast<size_t>(p.chunk_cap) * sizeof(int2));
  }
  p.off_part_lse = off;
  p.off_part_o = off;
  if (s.p_stride > 1) {
    const size_t slots = static_cast<size_t>(total_q) * hq * s.p_stride;
    off = align256(off + slots * 4);
    p.off_part_o = off;
    off = align256(off + slots * d * 4);
  }
  p.bytes = num_seqs > 0 ? off : 0;
  const long long items =
      varlen ? (static_cast<long long>(total_q) + static_cast<long long>(num_seqs) * (s.qpt - 1)) /
                   s.qpt
             : num_seqs;
  p.max_units = items * s.p_stride * hkv * s.ns;
  return p;
}

pa::Work carve(void* workspace, const Plan& p) {
  char* ws = static_cast<char*>(workspace);
  pa::Work w;
  w.sched = reinterpret_cast<pa::Sched*>(ws);
  w.row_a = reinterpret_cast<int*>(ws + p.off_row_a);
  w.row_b = reinterpret_cast<int*>(ws + p.off_row_b);
  w.chunk_list = reinterpret_cast<int2*>(ws + p.off_chunk);
  w.part_lse = reinterpret_cast<float*>(ws + p.off_part_lse);
  w.part_o = reinterpret_cast<float*>(ws + p.off_part_o);
  return w;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel on the stream (the prep kernel) runs; it calls
// griddepcontrol.wait before reading that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

bool supported_block_size(int bs) { return bs == 8 || bs == 16 || bs == 32; }

pa_status check_common(const AttnArgs& a) {
  if (!valid_dtype(a.dtype)) return fail(PA_ERR_INVALID_ARG, "unknown dtype %d", a.dtype);
  if (a.num_seqs < 0 || a.total_q < 0 || a.max_query_len < 0 || a.max_seq_len < 0 ||
      a.num_blocks < 0 || a.table_stride < 0)
    return fail(PA_ERR_INVALID_ARG, "negative size");
  if (a.num_q_heads <= 0 || a.num_kv_heads <= 0 || a.num_q_heads % a.num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                a.num_q_heads, a.num_kv_heads);
  if (a.head_dim != 64 && a.head_dim != 128 && a.head_dim != 256)
    return fail(PA_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128, 256)", a.head_dim);
  if (!supported_block_size(a.block_size))
    return fail(PA_ERR_UNSUPPORTED, "block_size %d (supported: 8, 16, 32)", a.block_size);
  if (!(std::isfinite(a.scale))) return fail(PA_ERR_INVALID_ARG, "scale is not finite");
  if (static_cast<long long>(a.num_blocks) * a.num_kv_heads * a.block_size > 0x7fffffffLL)
    return fail(PA_ERR_UNSUPPORTED, "pool of %d blocks x %d heads exceeds 2^31 token rows",
                a.num_blocks, a.num_kv_heads);
  if (static_cast<long long>(a.total_q) * a.num_q_heads > 0x7fffffffLL)
    return fail(PA_ERR_UNSUPPORTED, "too many query rows");
  if (a.total_q == 0 || a.num_seqs == 0) return PA_OK;
  const void* ptrs[] = {a.out, a.q, a.k_cache, a.v_cache};
  for (const void* p : ptrs) {
    if (!p) return fail(PA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(p, 16)) return fail(PA_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  }
  if (!a.block_tables || !a.seq_lens) return fail(PA_ERR_INVALID_ARG, "null metadata pointer");
  if (!aligned(a.block_tables, 4) || !aligned(a.seq_lens, 4))
    return fail(PA_ERR_INVALID_ARG, "metadata pointer not 4-byte aligned");
  if (a.num_blocks == 0) return fail(PA_ERR_INVALID_ARG, "empty KV pool");
  if (a.table_stride == 0) return fail(PA_ERR_INVALID_ARG, "block_table_stride is 0");
  return PA_OK;
}

template <typename T, int D, bool KV8>
pa_status launch_simt(const AttnArgs& a, const Plan& p, const pa::Work& w) {
  using C = typename std::conditional<KV8, uint8_t, T>::type;  // cache element
  auto kern = pa::attn_simt_kernel<T, D, KV8>;
  constexpr int smem = pa::simt_smem_bytes<D>();
  int occ = 0;
  cudaError_t e = prepare(kern, 128, smem, &occ);
  if (e != cudaSuccess) return cuda_fail(e, "simt kernel set-up");
  long long grid = static_cast<long long>(sm_count()) * occ;
  if (p.max_units < grid) grid = p.max_units;
  if (grid < 1) grid = 1;
  e = launch_pdl(kern, static_cast<unsigned>(grid), 128, smem, a.stream, p.s,
                 static_cast<T*>(a.out), static_cast<const T*>(a.q),
                 static_cast<const C*>(a.k_cache), static_cast<const C*>(a.v_cache),
                 a.block_tables, a.qsl, a.seq_lens, w, static_cast<float>(a.scale * M_LOG2E),
                 a.k_scale, a.v_scale);
  if (e != cudaSuccess) return cuda_fail(e, "simt kernel launch");
  return PA_OK;
}

template <typename T, int D, bool KV8, bool NARROW = false>
pa_status launch_mma(const AttnArgs& a, const Plan& p, const pa::Work& w) {
  // tiles of at most 8 rows on an FP8 cache at head_dim 128: the transposed
  // P.V form of the kernel
  if constexpr (KV8 && D == 128 && !NARROW) {
    if (p.s.gs * p.s.qpt <= 8) return launch_mma<T, D, KV8, true>(a, p, w);
  }
  // FP8 stages are half as large: at head_dim 128 twice as many keep the same
  // bytes in flight; at 64 the per-warp f16 staging tiles take that room.  The
  // NARROW form runs four CTAs per SM of three consumer warps and 9 stages
  // (three per warp; its 8-row query slots leave the room for them): its
  // throughput follows the number of CTAs (each with its own TMA thread) and
  // the tiles each warp has in flight.
  constexpr int kN = NARROW ? 3 : kNcw;
  constexpr int kS = NARROW ? 9 : (KV8 && D == 128 ? 2 * kStages : kStages);
  using L = pa::MmaLayout<D, kN, kS, KV8, NARROW>;
  auto kern = pa::attn_mma_kernel<T, D, kN, kS, KV8, NARROW>;
  int occ = 0;
  cudaError_t e = prepare(kern, L::kThreads, L::kSmem, &occ);
  if (e != cudaSuccess) return cuda_fail(e, "mma kernel set-up");
  CUtensorMap tk, tv, tq;
  // one box = 16 cache rows, or one whole 8-token block
  const uint64_t rows = static_cast<uint64_t>(a.num_blocks) * a.num_kv_heads * a.block_size;
  const int box_rows = a.block_size < pa::kBlock ? a.block_size : pa::kBlock;
  pa_status st = KV8 ? make_map_2d_u8(&tk, a.k_cache, D, rows, box_rows)
                     : make_map_kv(&tk, a.k_cache, a.dtype, D, rows, box_rows / 8);
  if (st != PA_OK) return st;
  st = KV8 ? make_map_2d_u8(&tv, a.v_cache, D, rows, box_rows)
           : make_map_kv(&tv, a.v_cache, a.dtype, D, rows, box_rows / 8);
  if (st != PA_OK) return st;
  st = make_map_3d(&tq, a.q, a.dtype, D, a.num_q_heads, a.total_q, p.s.gs, p.s.qpt);
  if (st != PA_OK) return st;
  long long grid = static_cast<long long>(sm_count()) * occ;
  if (p.max_units < grid) grid = p.max_units;
  if (grid < 1) grid = 1;
  e = launch_pdl(kern, static_cast<unsigned>(grid), L::kThreads, L::kSmem, a.stream, tk, tv, tq,
                 p.s, static_cast<T*>(a.out), a.block_tables, a.qsl, a.seq_lens, w,
                 static_cast<float>(a.scale * M_LOG2E), a.k_scale, a.v_scale);
  if (e != cudaSuccess) return cuda_fail(e, "mma kernel launch");
  return PA_OK;
}

// The tcgen05 chunk kernel: two query tiles per item up to head_dim 128,
// one per item (64-key tiles) at 256.
template <typename T, int D>
pa_status launch_chunk(const AttnArgs& a, const Plan& p, const pa::Work& w) {
  using L = typename std::conditional<D == 256, pa::Tc1Layout<256>, pa::Tc2Layout<D>>::type;
  auto kern = D == 256 ? pa::chunk_tc1_kernel<T, 256> : pa::chunk_tc2_kernel<T, D == 256 ? 128 : D>;
  int occ = 0;
  cudaError_t e = prepare(kern, L::kThreads, L::kSmem, &occ);
  if (e != cudaSuccess) return cuda_fail(e, "chunk kernel set-up");
  CUtensorMap tk, tv, tq;
  // one box = 16 cache rows, or one whole 8-token block
  const uint64_t rows = static_cast<uint64_t>(a.num_blocks) * a.num_kv_heads * a.block_size;
  const int box_rows = a.block_size < pa::kBlock ? a.block_size : pa::kBlock;
  pa_status st = make_map_kv(&tk, a.k_cache, a.dtype, D, rows, box_rows / 8);
  if (st != PA_OK) return st;
  st = make_map_kv(&tv, a.v_cache, a.dtype, D, rows, box_rows / 8);
  if (st != PA_OK) return st;
  st = make_map_3d(&tq, a.q, a.dtype, D, a.num_q_heads, a.total_q, p.s.gs, p.s.chunk_qt);
  if (st != PA_OK) return st;
  long long grid = sm_count();
  const long long items = p.chunk_cap * a.num_kv_heads * p.s.ns;
  if (items < grid) grid = items;
  if (grid < 1) grid = 1;
  e = launch_pdl(kern, static_cast<unsigned>(grid), L::kThreads, L::kSmem, a.stream, tk, tv, tq,
                 p.s, static_cast<T*>(a.out), a.block_tables, a.qsl, a.seq_lens, w,
                 static_cast<float>(a.scale * M_LOG2E));
  if (e != cudaSuccess) return cuda_fail(e, "chunk kernel launch");
  return PA_OK;
}

// The CUDA-core kernel for the call's head_dim and cache type.
template <typename T>
pa_status simt_for_dim(const AttnArgs& a, const Plan& p, const pa::Work& w) {
  switch (a.head_dim) {
    case 64: return a.kv8() ? launch_simt<T, 64, true>(a, p, w) : launch_simt<T, 64, false>(a, p, w);
    case 128:
      return a.kv8() ? launch_simt<T, 128, true>(a, p, w) : launch_simt<T, 128, false>(a, p, w);
    default:
      return a.kv8() ? launch_simt<T, 256, true>(a, p, w) : launch_simt<T, 256, false>(a, p, w);
  }
}

template <typename T>
pa_status run_typed(const AttnArgs& a, const Plan& p, bool use_mma) {
  const pa::Work w = carve(a.workspace, p);
  cudaError_t e = launch_pdl(pa::schedule_kernel<T>, 1, 1024, 0, a.stream, p.s, a.qsl,
                             a.seq_lens, w, static_cast<T*>(a.out));
  if (e != cudaSuccess) return cuda_fail(e, "schedule kernel launch");
  pa_status st;
  const bool d128 = a.head_dim == 128;
  if constexpr (sizeof(T) == 2) {
    if (a.head_dim == 256)
      st = a.kv8() ? launch_mma<T, 256, true>(a, p, w) : launch_mma<T, 256, false>(a, p, w);
    else if (use_mma)
      st = a.kv8() ? (d128 ? launch_mma<T, 128, true>(a, p, w) : launch_mma<T, 64, true>(a, p, w))
                   : (d128 ? launch_mma<T, 128, false>(a, p, w)
                           : launch_mma<T, 64, false>(a, p, w));
    else
      st = simt_for_dim<T>(a, p, w);
  } else {
    st = simt_for_dim<T>(a, p, w);
  }
  if (st != PA_OK) return st;
  if constexpr (sizeof(T) == 2) {
    if (p.s.chunk_qt > 0) {
      st = a.head_dim == 128   ? launch_chunk<T, 128>(a, p, w)
           : a.head_dim == 256 ? launch_chunk<T, 256>(a, p, w)
                               : launch_chunk<T, 64>(a, p, w);
      if (st != PA_OK) return st;
    }
  }
  if (p.s.p_stride <= 1) return PA_OK;
  // one CTA per (request, 16-token slice, 8 heads) of the rows the attention
  // kernels split; with 16 or more partitions per row, one per query head
  const bool wide = p.s.p_stride >= 16;
  int max_q = a.qsl ? a.max_query_len : 1;
  if (p.s.chunk_qt > 0 && max_q >= p.s.chunk_qt) max_q = p.s.chunk_qt - 1;
  const int slices = (max_q + pa::kReduceTokens - 1) / pa::kReduceTokens;
  const dim3 grid(static_cast<unsigned>(a.num_seqs),
                  static_cast<unsigned>(slices < 65535 ? slices : 65535),
                  static_cast<unsigned>(wide ? a.num_q_heads : (a.num_q_heads + 7) / 8));
  if (grid.y == 0) return PA_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto launch = [&](auto kern) {
    return cudaLaunchKernelEx(&cfg, kern, p.s, a.qsl, a.seq_lens, w, static_cast<T*>(a.out));
  };
  if (wide)
    e = a.head_dim == 256   ? launch(pa::reduce_wide_kernel<T, 256>)
        : a.head_dim == 128 ? launch(pa::reduce_wide_kernel<T, 128>)
                            : launch(pa::reduce_wide_kernel<T, 64>);
  else
    e = a.head_dim == 256   ? launch(pa::reduce_kernel<T, 256>)
        : a.head_dim == 128 ? launch(pa::reduce_kernel<T, 128>)
                            : launch(pa::reduce_kernel<T, 64>);
  if (e != cudaSuccess) return cuda_fail(e, "reduce kernel launch");
  return PA_OK;
}

pa_status run_attention(const AttnArgs& a, bool varlen) {
  pa_status st = check_common(a);
  if (st != PA_OK) return st;
  if (a.total_q == 0 || a.num_seqs == 0) return PA_OK;
  const int max_len = a.max_seq_len;
  Plan p = make_plan(a.num_seqs, a.total_q, a.num_q_heads, a.num_kv_heads, a.head_dim, max_len,
                     varlen);
  p.s.table_stride = a.table_stride;
  p.s.block_size = a.block_size;
  p.s.num_blocks = a.num_blocks;
  p.s.max_seq_len = a.max_seq_len;
  p.s.max_query_len = varlen ? a.max_query_len : 1;
  if (!a.workspace) return fail(PA_ERR_WORKSPACE, "null workspace (%zu bytes needed)", p.bytes);
  if (!aligned(a.workspace, 256)) return fail(PA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (a.workspace_bytes < p.bytes)
    return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", a.workspace_bytes, p.bytes);
  if (varlen) {
    if (!a.qsl || !aligned(a.qsl, 4)) return fail(PA_ERR_INVALID_ARG, "bad query_start_loc");
  }
  if (a.kv8() && (!a.v_scale || !aligned(a.k_scale, 4) || !aligned(a.v_scale, 4)))
    return fail(PA_ERR_INVALID_ARG, "bad k_scale / v_scale pointer");
  const int path = g_path.load();
  const bool sixteen = a.dtype != PA_F32;
  if (path == PA_PATH_MMA || path == PA_PATH_TCGEN05) {
    if (!sixteen)
      return fail(PA_ERR_UNSUPPORTED, "tensor-core path needs bf16 or f16 (got fp32)");
  }
  const bool use_mma = sixteen && path != PA_PATH_SIMT;
  // Prefill-chunk rows (q_len >= one 128-row tile) go to the tcgen05 kernel
  // unless a family without it was forced.
  p.s.chunk_qt = (use_mma && !a.kv8() && path != PA_PATH_MMA &&
                  p.chunk_qt > 0 &&
                  a.max_query_len >= p.chunk_qt)
                     ? p.chunk_qt
                     : 0;
  p.s.chunk_cap = static_cast<int>(p.chunk_cap);
  // a chunk item holds two query tiles (one at head_dim 256)
  p.s.chunk_span = a.head_dim == 256 ? p.s.chunk_qt : 2 * p.s.chunk_qt;
  switch (a.dtype) {
    case PA_BF16: return run_typed<__nv_bfloat16>(a, p, use_mma);
    case PA_F16: return run_typed<__half>(a, p, use_mma);
    default: return run_typed<float>(a, p, false);
  }
}

// Scratch for pa_decode_static: a fixed array in the library's device image,
// for callers that cannot allocate (see include/pa.h).  Host code may not use
// the symbol itself as a device address; static_workspace() looks the address
// up, with the device current, once per (device, context): after a
// cudaDeviceReset the primary context is new and the module may load
// elsewhere, so a new context gets a new lookup.
static __device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

pa_status static_workspace(void** ptr) {
  static std::mutex mu;
  static std::map<std::pair<int, CUcontext>, void*> addr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  CUcontext ctx = nullptr;
  const CtxGetCurrentFn get = ctx_get_current_fn();
  if (!get || get(&ctx) != CUDA_SUCCESS) ctx = nullptr;  // keyed on the device alone
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_pair(dev, ctx);
  auto it = addr.find(key);
  if (it == addr.end()) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
    it = addr.emplace(key, p).first;
  }
  *ptr = it->second;
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                               const int32_t* slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                               void* stream) {
  if (!valid_dtype(dtype)) return fail(PA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks < 0)
    return fail(PA_ERR_INVALID_ARG, "bad sizes");
  if (head_dim != 64 && head_dim != 128 && head_dim != 256)
    return fail(PA_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128, 256)", head_dim);
  if (!supported_block_size(block_size))
    return fail(PA_ERR_UNSUPPORTED, "block_size %d (supported: 8, 16, 32)", block_size);
  if (num_tokens == 0) return PA_OK;
  const void* ptrs[] = {k, v, k_cache, v_cache};
  for (const void* p : ptrs) {
    if (!p) return fail(PA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(p, 16)) return fail(PA_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  }
  if (!slot_mapping || !aligned(slot_mapping, 4))
    return fail(PA_ERR_INVALID_ARG, "bad slot_mapping pointer");
  const int row_vecs = head_dim * elem_bytes(dtype) / 16;
  const long long warps = static_cast<long long>(num_tokens) * num_kv_heads;
  const long long blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "too many tokens");
  const cudaError_t e = launch_pdl(
      pa::reshape_and_cache_kernel, static_cast<unsigned>(blocks), 256, 0,
      static_cast<cudaStream_t>(stream), static_cast<const uint4*>(k),
      static_cast<const uint4*>(v), static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
      slot_mapping, num_tokens, num_kv_heads, row_vecs, block_size,
      static_cast<long long>(num_blocks) * block_size);
  if (e != cudaSuccess) return cuda_fail(e, "reshape_and_cache launch");
  return PA_OK;
}

pa_status pa_reshape_and_cache_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                                   const int32_t* slot_mapping, const float* k_scale,
                                   const float* v_scale, int num_tokens, int num_kv_heads,
                                   int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                                   void* stream) {
  if (!valid_dtype(dtype)) return fail(PA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks < 0)
    return fail(PA_ERR_INVALID_ARG, "bad sizes");
  if (head_dim != 64 && head_dim != 128 && head_dim != 256)
    return fail(PA_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128, 256)", head_dim);
  if (!supported_block_size(block_size))
    return fail(PA_ERR_UNSUPPORTED, "block_size %d (supported: 8, 16, 32)", block_size);
  if (num_tokens == 0) return PA_OK;
  const void* ptrs[] = {k, v, k_cache, v_cache};
  for (const void* p : ptrs) {
    if (!p) return fail(PA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(p, 16)) return fail(PA_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  }
  if (!slot_mapping || !aligned(slot_mapping, 4))
    return fail(PA_ERR_INVALID_ARG, "bad slot_mapping pointer");
  if (!k_scale || !v_scale || !aligned(k_scale, 4) || !aligned(v_scale, 4))
    return fail(PA_ERR_INVALID_ARG, "bad k_scale / v_scale pointer");
  const long long warps = static_cast<long long>(num_tokens) * num_kv_heads;
  const long long blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "too many tokens");
  const auto st = static_cast<cudaStream_t>(stream);
  const long long slots = static_cast<long long>(num_blocks) * block_size;
  const unsigned g = static_cast<unsigned>(blocks);
  auto* kc = static_cast<uint8_t*>(k_cache);
  auto* vc = static_cast<uint8_t*>(v_cache);
  auto launch = [&](auto* tag) {
    using T = std::remove_pointer_t<decltype(tag)>;
    return launch_pdl(pa::reshape_and_cache_fp8_kernel<T>, g, 256, 0, st,
                      static_cast<const T*>(k), static_cast<const T*>(v), kc, vc, slot_mapping,
                      k_scale, v_scale, num_tokens, num_kv_heads, head_dim, block_size, slots);
  };
  const cudaError_t e = dtype == PA_BF16 ? launch(static_cast<__nv_bfloat16*>(nullptr))
                        : dtype == PA_F16 ? launch(static_cast<__half*>(nullptr))
                                          : launch(static_cast<float*>(nullptr));
  if (e != cudaSuccess) return cuda_fail(e, "reshape_and_cache_fp8 launch");
  return PA_OK;
}

pa_status pa_rope_reshape_and_cache(void* q, const void* k, const void* v, void* k_cache,
                                    void* v_cache, const int32_t* slot_mapping,
                                    const int32_t* positions, const float* cos_sin,
                                    int max_position, int rot_dim, int neox, int num_tokens,
                                    int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int num_blocks, pa_dtype dtype,
                                    void* stream) {
  if (!valid_dtype(dtype)) return fail(PA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (num_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks < 0 ||
      max_position <= 0)
    return fail(PA_ERR_INVALID_ARG, "bad sizes");
  if (head_dim != 64 && head_dim != 128 && head_dim != 256)
    return fail(PA_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128, 256)", head_dim);
  if (!supported_block_size(block_size))
    return fail(PA_ERR_UNSUPPORTED, "block_size %d (supported: 8, 16, 32)", block_size);
  if (rot_dim < 2 || rot_dim > head_dim || rot_dim % 2 != 0)
    return fail(PA_ERR_INVALID_ARG, "rot_dim %d must be even and in [2, head_dim]", rot_dim);
  if (num_tokens == 0) return PA_OK;
  const void* ptrs[] = {q, k, v, k_cache, v_cache};
  for (const void* p : ptrs) {
    if (!p) return fail(PA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(p, 16)) return fail(PA_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  }
  if (!slot_mapping || !positions || !cos_sin || !aligned(slot_mapping, 4) ||
      !aligned(positions, 4) || !aligned(cos_sin, 4))
    return fail(PA_ERR_INVALID_ARG, "bad slot_mapping / positions / cos_sin pointer");
  // quads of four elements line up with both pair layouts when rot_dim is a
  // multiple of 8; the table rows then start 16-byte aligned if the base is
  const bool vec = rot_dim % 8 == 0 && aligned(cos_sin, 16);
  constexpr int kH = pa::kRopeHeads;
  const long long parts = vec ? (num_q_heads + kH - 1) / kH + (num_kv_heads + kH - 1) / kH
                              : static_cast<long long>(num_q_heads) + num_kv_heads;
  const long long warps = static_cast<long long>(num_tokens) * parts;
  const long long blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "too many tokens");
  const auto st = static_cast<cudaStream_t>(stream);
  const unsigned g = static_cast<unsigned>(blocks);
  const long long slots = static_cast<long long>(num_blocks) * block_size;
  auto launch = [&](auto* tag) {
    using T = std::remove_pointer_t<decltype(tag)>;
    auto kern = vec ? pa::rope_reshape_and_cache_vec_kernel<T> : pa::rope_reshape_and_cache_kernel<T>;
    return launch_pdl(kern, g, 256, 0, st, static_cast<T*>(q), static_cast<const T*>(k),
                      static_cast<const T*>(v), static_cast<T*>(k_cache),
                      static_cast<T*>(v_cache), slot_mapping, positions, cos_sin, max_position,
                      rot_dim, neox != 0, num_tokens, num_q_heads, num_kv_heads, head_dim,
                      block_size, slots);
  };
  const cudaError_t e = dtype == PA_BF16 ? launch(static_cast<__nv_bfloat16*>(nullptr))
                        : dtype == PA_F16 ? launch(static_cast<__half*>(nullptr))
                                          : launch(static_cast<float*>(nullptr));
  if (e != cudaSuccess) return cuda_fail(e, "rope_reshape_and_cache launch");
  return PA_OK;
}

// Device-visible address of a pointer the kernels may dereference: device
// memory as is, page-locked host memory through its mapped address.  Pageable
// host memory is refused.
static pa_status device_address(const void* p, const void** out, const char* what) {
  cudaPointerAttributes at{};
  const cudaError_t e = cudaPointerGetAttributes(&at, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(PA_ERR_INVALID_ARG, "%s: not a CUDA-visible pointer", what);
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) {
    *out = p;
    return PA_OK;
  }
  if (at.type == cudaMemoryTypeHost && at.devicePointer) {
    *out = at.devicePointer;
    return PA_OK;
  }
  return fail(PA_ERR_INVALID_ARG, "%s: host memory must be page-locked (cudaHostAlloc/Register)",
              what);
}

static pa_status launch_block_copy(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                                   const int32_t* block_mapping, int num_pairs, int num_kv_heads,
                                   int head_dim, int block_size, int src_num_blocks,
                                   int dst_num_blocks, pa_dtype dtype, void* stream,
                                   bool allow_host) {
  if (!valid_dtype(dtype) && dtype != PA_E4M3)
    return fail(PA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || src_num_blocks < 0 ||
      dst_num_blocks < 0)
    return fail(PA_ERR_INVALID_ARG, "bad sizes");
  if (head_dim != 64 && head_dim != 128 && head_dim != 256)
    return fail(PA_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128, 256)", head_dim);
  if (!supported_block_size(block_size))
    return fail(PA_ERR_UNSUPPORTED, "block_size %d (supported: 8, 16, 32)", block_size);
  if (num_pairs == 0) return PA_OK;
  const void* in[] = {src_k, src_v, dst_k, dst_v, block_mapping};
  const char* names[] = {"src_k", "src_v", "dst_k", "dst_v", "block_mapping"};
  const void* dev[5];
  for (int i = 0; i < 5; ++i) {
    if (!in[i]) return fail(PA_ERR_INVALID_ARG, "%s is null", names[i]);
    if (!aligned(in[i], i < 4 ? 16 : 4))
      return fail(PA_ERR_INVALID_ARG, "%s is not %d-byte aligned", names[i], i < 4 ? 16 : 4);
    if (allow_host) {
      const pa_status st = device_address(in[i], &dev[i], names[i]);
      if (st != PA_OK) return st;
    } else {
      dev[i] = in[i];
    }
  }
  const long long block_bytes =
      static_cast<long long>(num_kv_heads) * block_size * head_dim * elem_bytes(dtype);
  if (block_bytes / 16 > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "block too large");
  const int block_vecs = static_cast<int>(block_bytes / 16);
  const int chunks = (block_vecs + pa::kCopyThreads * pa::kCopyUnroll - 1) /
                     (pa::kCopyThreads * pa::kCopyUnroll);
  const long long grid = static_cast<long long>(num_pairs) * chunks;
  if (grid > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "too many pairs");
  pa::copy_blocks_kernel<<<dim3(static_cast<unsigned>(grid), 2), pa::kCopyThreads, 0,
                           static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(dev[0]), static_cast<const uint4*>(dev[1]),
      static_cast<uint4*>(const_cast<void*>(dev[2])), static_cast<uint4*>(const_cast<void*>(dev[3])),
      static_cast<const int*>(dev[4]), src_num_blocks, dst_num_blocks, block_vecs, chunks);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "block copy launch");
  return PA_OK;
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* block_mapping,
                         int num_pairs, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype dtype, void* stream) {
  return launch_block_copy(k_cache, v_cache, k_cache, v_cache, block_mapping, num_pairs,
                           num_kv_heads, head_dim, block_size, num_blocks, num_blocks, dtype,
                           stream, false);
}

pa_status pa_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                         const int32_t* block_mapping, int num_pairs, int num_kv_heads,
                         int head_dim, int block_size, int src_num_blocks, int dst_num_blocks,
                         pa_dtype dtype, void* stream) {
  return launch_block_copy(src_k, src_v, dst_k, dst_v, block_mapping, num_pairs, num_kv_heads,
                           head_dim, block_size, src_num_blocks, dst_num_blocks, dtype, stream,
                           true);
}

size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                int max_context_len) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0) return 0;
  return make_plan(num_seqs, num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                   false)
      .bytes;
}

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int block_table_stride,
                    const int32_t* context_lens, int num_seqs, int num_q_heads,
                    int num_kv_heads, int head_dim, int block_size, int num_blocks,
                    int max_context_len, float scale, void* workspace, size_t workspace_bytes,
                    pa_dtype dtype, void* stream) {
  AttnArgs a{out, q, k_cache, v_cache, block_tables, block_table_stride, nullptr, context_lens,
             num_seqs, num_seqs, 1, max_context_len, num_q_heads, num_kv_heads, head_dim,
             block_size, num_blocks, scale, workspace, workspace_bytes, dtype,
             static_cast<cudaStream_t>(stream)};
  return run_attention(a, false);
}

pa_status pa_decode_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int block_table_stride,
                           const int32_t* context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           int max_context_len, float scale, pa_dtype dtype, void* stream) {
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                               max_context_len);
  if (need > PA_STATIC_WORKSPACE_BYTES)
    return fail(PA_ERR_WORKSPACE,
                "pa_decode_static: these sizes need %zu bytes of scratch; the built-in array "
                "holds %zu (use pa_decode with a workspace)",
                need, static_cast<size_t>(PA_STATIC_WORKSPACE_BYTES));
  void* ws = nullptr;
  if (need > 0) {
    const pa_status st = static_workspace(&ws);
    if (st != PA_OK) return st;
  }
  return pa_decode(out, q, k_cache, v_cache, block_tables, block_table_stride, context_lens,
                   num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                   max_context_len, scale, ws, PA_STATIC_WORKSPACE_BYTES, dtype, stream);
}

size_t pa_varlen_workspace_size(int num_seqs, int total_q, int num_q_heads, int num_kv_heads,
                                int head_dim, int max_query_len, int max_seq_len) {
  (void)max_query_len;
  if (num_seqs <= 0 || total_q <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return 0;
  return make_plan(num_seqs, total_q, num_q_heads, num_kv_heads, head_dim, max_seq_len, true)
      .bytes;
}

pa_status pa_varlen(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int block_table_stride,
                    const int32_t* query_start_loc, const int32_t* seq_lens, int num_seqs,
                    int total_q, int max_query_len, int max_seq_len, int num_q_heads,
                    int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                    void* workspace, size_t workspace_bytes, pa_dtype dtype, void* stream) {
  AttnArgs a{out, q, k_cache, v_cache, block_tables, block_table_stride, query_start_loc,
             seq_lens, num_seqs, total_q, max_query_len, max_seq_len, num_q_heads,
             num_kv_heads, head_dim, block_size, num_blocks, scale, workspace, workspace_bytes,
             dtype, static_cast<cudaStream_t>(stream)};
  return run_attention(a, true);
}

pa_status pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const float* k_scale, const float* v_scale,
                        const int32_t* block_tables, int block_table_stride,
                        const int32_t* context_lens, int num_seqs, int num_q_heads,
                        int num_kv_heads, int head_dim, int block_size, int num_blocks,
                        int max_context_len, float scale, void* workspace,
                        size_t workspace_bytes, pa_dtype dtype, void* stream) {
  if (!k_scale) return fail(PA_ERR_INVALID_ARG, "null k_scale");
  AttnArgs a{out, q, k_cache, v_cache, block_tables, block_table_stride, nullptr, context_lens,
             num_seqs, num_seqs, 1, max_context_len, num_q_heads, num_kv_heads, head_dim,
             block_size, num_blocks, scale, workspace, workspace_bytes, dtype,
             static_cast<cudaStream_t>(stream), k_scale, v_scale};
  return run_attention(a, false);
}

pa_status pa_varlen_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const float* k_scale, const float* v_scale,
                        const int32_t* block_tables, int block_table_stride,
                        const int32_t* query_start_loc, const int32_t* seq_lens, int num_seqs,
                        int total_q, int max_query_len, int max_seq_len, int num_q_heads,
                        int num_kv_heads, int head_dim, int block_size, int num_blocks,
                        float scale, void* workspace, size_t workspace_bytes, pa_dtype dtype,
                        void* stream) {
  if (!k_scale) return fail(PA_ERR_INVALID_ARG, "null k_scale");
  AttnArgs a{out, q, k_cache, v_cache, block_tables, block_table_stride, query_start_loc,
             seq_lens, num_seqs, total_q, max_query_len, max_seq_len, num_q_heads,
             num_kv_heads, head_dim, block_size, num_blocks, scale, workspace, workspace_bytes,
             dtype, static_cast<cudaStream_t>(stream), k_scale, v_scale};
  return run_attention(a, true);
}

pa_status pa_get_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  pa::DeviceError rec{};
  e = cudaMemcpyFromSymbol(&rec, pa::g_device_error, sizeof(rec));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (rec.code == 0) return PA_OK;
  const pa::DeviceError zero{};
  e = cudaMemcpyToSymbol(pa::g_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  static const char* where[] = {"?", "reshape_and_cache slot", "block-table entry",
                                "row metadata", "wait for K/V tile", "wait for free stage",
                                "wait for query tile", "tensor memory", "wait for MMA/barrier",
                                "block copy pair", "rope position"};
  const int w = rec.where >= 0 && rec.where <= 10 ? rec.where : 0;
  return fail(static_cast<pa_status>(rec.code), "device: %s (%s; a=%lld b=%lld)",
              pa_status_string(static_cast<pa_status>(rec.code)), where[w], rec.a, rec.b);
}

pa_path pa_set_path(pa_path path) {
  return static_cast<pa_path>(g_path.exchange(static_cast<int>(path)));
}

const char* pa_status_string(pa_status status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_DEVICE_BOUNDS: return "PA_ERR_DEVICE_BOUNDS";
    case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT";
  }
  return "PA_ERR_UNKNOWN";
}

const char* pa_last_error_message(void) { return g_msg.c_str(); }

pa_status pa_debug_lost_load(int kernel) {
  if (kernel < 0 || kernel > 2) return fail(PA_ERR_INVALID_ARG, "kernel %d (0, 1 or 2)", kernel);
  // about one millisecond at the top SM clock while the hook is on
  const long long limit = kernel ? 2000000LL : pa::kWaitLimitCycles;
  cudaError_t e = cudaMemcpyToSymbol(pa::g_wait_limit_cycles, &limit, sizeof(limit));
  if (e != cudaSuccess) return cuda_fail(e, "set wait limit");
  e = cudaMemcpyToSymbol(pa::g_debug_lost_load, &kernel, sizeof(kernel));
  if (e != cudaSuccess) return cuda_fail(e, "set lost-load hook");
  return PA_OK;
}

int pa_binary_version(void) {
  cudaFuncAttributes at{};
  if (cudaFuncGetAttributes(&at, pa::reshape_and_cache_kernel) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return at.binaryVersion;
}

int pa_version(void) { return 100; }

}  // extern "C"
