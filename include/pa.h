/*
 * pa.h -- paged KV-cache attention for NVIDIA B200 (sm_100a), C ABI.
 *
 * The hot path of a paged-KV serving engine's attention layer:
 *
 *   1. pa_reshape_and_cache  -- scatter this step's new K/V rows into
 *      physical blocks (8, 16 or 32 tokens) through a per-token slot mapping
 *      ("vLLM 架构源码解析 | 第 1 篇" §3.3.3: reshape_and_cache(k, v, kv_cache,
 *      slot_mapping) runs before paged_attention in every attention layer).
 *   2. pa_decode             -- one query row per request attends to its
 *      cached context through its block-table row
 *      ("vLLM 深度拆解：当 KV Cache 学会「分页」" §3.3 and §6.2;
 *      "vLLM 架构源码解析" §3.3.3 paged_attention(q, kv_cache, block_tables,
 *      context_lens)).
 *   3. pa_varlen             -- the scheduler's mixed batch: decode rows next
 *      to causal chunked-prefill chunks whose earlier context is cached
 *      ("vLLM 深度拆解" §4.3 chunked prefill; "vLLM 架构源码解析" §3.2 unified
 *      token budget and §3.3.2 query_start_loc / positions / seq_lens).
 *
 * and the block operations next to it: pa_copy_blocks (copy-on-write) and
 * pa_swap_blocks (swap-out / swap-in between the device and a host pool).
 *
 * Attention is softmax(q . K^T * scale) . V ("vLLM 深度拆解" §2.2).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer argument except the returned strings is a DEVICE pointer on
 *   the current CUDA device, owned by the caller (pa_swap_blocks also takes
 *   page-locked host memory).  The library keeps no
 *   pointer after the call returns and allocates no device memory: scratch
 *   space is the caller's `workspace`, sized by the *_workspace_size query
 *   (pa_decode_static uses a fixed array built into the library instead).
 * - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *   NULL = the legacy default stream).  No call synchronises, except
 *   pa_get_device_error.  Order pa_reshape_and_cache before the attention call
 *   that must see its rows on the same stream.
 * - All tensors are dense and row-major with the shapes given below; base
 *   pointers must be 16-byte aligned.
 * - KV cache layout: k_cache and v_cache are each
 *   [num_blocks, num_kv_heads, block_size, head_dim].  Each (block, head)
 *   holds block_size consecutive tokens of one request as a contiguous
 *   block_size x head_dim row-major tile.  (The pages print two layouts,
 *   [blocks, heads, head_size, block_size] in "vLLM 深度拆解" §6.2 and
 *   [blocks, block_size, d_k] in "vLLM 架构源码解析" §4.2; this one keeps a
 *   token's head_dim values contiguous so that one 16-byte load carries eight
 *   16-bit values of one token.)
 * - block_size is 8, 16 or 32 tokens ("vLLM 架构源码解析" §5.1 weighs 8, 16
 *   and 32 and passes block_size=32; 16 is the default of §1.1).
 * - block_tables is int32 [num_seqs, block_table_stride]: entry [r][j] is the
 *   physical block holding tokens j*block_size .. (j+1)*block_size-1 of
 *   request r ("vLLM 深度拆解" §3.3: block_tables[seq_id * stride +
 *   block_idx]).  Entries past ceil(len/block_size) are never read.
 * - Grouped-query attention: query head h reads KV head
 *   h / (num_q_heads / num_kv_heads).  num_q_heads % num_kv_heads == 0.
 * - head_dim is 64, 128 or 256, for every dtype, cache type and block size.
 *   dtype: PA_F32, PA_BF16 or PA_F16; q, k, v, the caches and out all have
 *   that dtype (an FP8 cache holds e4m3 codes instead).  Arithmetic is fp32
 *   with one round-to-nearest-even conversion of the output.
 * - Errors: a status other than PA_OK returned by a call means nothing was
 *   launched (argument checks are done on the host before any launch) or a
 *   launch failed (PA_ERR_CUDA).  Checks that need device data (a block id
 *   outside [0, num_blocks), a slot outside the pool, a length above the
 *   host-given maximum, a bounded wait that ran out) are made inside the
 *   kernels: the offending access is skipped, the first such event is
 *   recorded in a per-device error word, and pa_get_device_error reports it.
 *   No kernel faults, traps or waits without bound on bad metadata.
 * - Thread safety: calls may be made from several host threads; the device
 *   error word is shared per device.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* a null/misaligned pointer, a negative size, Hq % Hkv != 0, ... */
  PA_ERR_UNSUPPORTED = 2,   /* a valid but unimplemented shape: head_dim, block_size, dtype */
  PA_ERR_WORKSPACE = 3,     /* workspace_bytes below the size query's answer */
  PA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  PA_ERR_DEVICE_BOUNDS = 5, /* (device) bad metadata: block id, slot or length out of range */
  PA_ERR_TIMEOUT = 6        /* (device) a bounded wait inside a kernel gave up */
} pa_status;

typedef enum {
  PA_F32 = 0,
  PA_BF16 = 1,
  PA_F16 = 2,
  PA_E4M3 = 3  /* FP8 cache codes: only the element type of a pool in the block copies */
} pa_dtype;

/*
 * Kernel family selection, for tests and measurements.  PA_PATH_AUTO picks
 * the fastest family that supports the shape: the TMA + tensor-core kernel for
 * 16-bit types, the CUDA-core kernel for fp32, and the tcgen05 (TMEM) tile
 * kernel for the prefill chunks of pa_varlen.  The other values force one
 * family; forcing a family that does not support the call's shape makes the
 * call return PA_ERR_UNSUPPORTED.  The setting is process-wide.
 */
typedef enum {
  PA_PATH_AUTO = 0,
  PA_PATH_SIMT = 1,     /* CUDA-core kernel, plain vector loads (any dtype) */
  PA_PATH_MMA = 2,      /* TMA bulk-tensor loads + warp-level bf16/f16 tensor-core MMA */
  PA_PATH_TCGEN05 = 3   /* as PA_PATH_MMA, with prefill chunks on tcgen05/TMEM tiles */
} pa_path;

/*
 * pa_reshape_and_cache -- write this step's new K/V rows into the cache.
 *
 * "vLLM 架构源码解析" §3.3.3 (LlamaAttention.forward calls
 * cache_ops.reshape_and_cache(k, v, kv_cache, slot_mapping) before
 * paged_attention) and §3.3.2 (_prepare_inputs builds the slot mapping).
 *
 *   k, v          [num_tokens, num_kv_heads, head_dim]   this step's rows
 *   k_cache,      [num_blocks, num_kv_heads, block_size, head_dim], updated
 *   v_cache         in place
 *   slot_mapping  int32 [num_tokens]: token t goes to physical block
 *                 slot/block_size, offset slot%block_size.  slot < 0 marks a
 *                 padding token: it is skipped.  A slot >= num_blocks *
 *                 block_size is skipped and recorded as PA_ERR_DEVICE_BOUNDS.
 *
 * Bytes are copied exactly.  Two tokens naming the same slot in one call
 * leave an unspecified one of the two rows.  num_tokens == 0 is a no-op.
 */
pa_status pa_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                               const int32_t* slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                               void* stream);

/*
 * pa_rope_reshape_and_cache -- pa_reshape_and_cache with the rotary position
 * embedding fused in (the kernel-fusion theme of "vLLM 深度拆解" §6.1: the
 * elementwise work rides along with the neighbouring kernel, so q and k make
 * one trip through HBM).  The pages do not define a position encoding; the
 * rotation is RoFormer's: the first rot_dim dims of each head form rot_dim/2
 * pairs -- (2i, 2i+1) when neox == 0, (i, i + rot_dim/2) when neox != 0 --
 * and the pair (x1, x2) of token t becomes (x1 c - x2 s, x2 c + x1 s) with
 * c = cos_sin[positions[t]][i] and s = cos_sin[positions[t]][rot_dim/2 + i].
 * Dims from rot_dim on pass through.
 *
 *   q             [num_tokens, num_q_heads, head_dim], rotated IN PLACE
 *   k, v          [num_tokens, num_kv_heads, head_dim], read only
 *   k_cache,      as for pa_reshape_and_cache: token t's rotated k row and
 *   v_cache         its v row go to slot slot_mapping[t] (slot < 0: padding,
 *                   skipped; q is rotated all the same)
 *   positions     int32 [num_tokens], each in [0, max_position)
 *   cos_sin       fp32 [max_position, rot_dim]: cosines then sines
 *
 * Each result is computed in fp32 and rounded once to `dtype`.  A position
 * outside [0, max_position) leaves that token's q and cache rows untouched
 * and is recorded as PA_ERR_DEVICE_BOUNDS; slots as for pa_reshape_and_cache.
 * rot_dim must be even and at most head_dim (else PA_ERR_INVALID_ARG).  With
 * rot_dim a multiple of 8 and cos_sin 16-byte aligned the call runs a
 * vectorised kernel; other shapes run a per-element one with the same
 * arithmetic.
 */
pa_status pa_rope_reshape_and_cache(void* q, const void* k, const void* v, void* k_cache,
                                    void* v_cache, const int32_t* slot_mapping,
                                    const int32_t* positions, const float* cos_sin,
                                    int max_position, int rot_dim, int neox, int num_tokens,
                                    int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int num_blocks, pa_dtype dtype,
                                    void* stream);

/*
 * FP8 KV cache ("vLLM 深度拆解" §10.1: native FP8 with calibrated scales is
 * the engine's next step).  The reading implemented: k_cache and v_cache hold
 * FP8 e4m3 codes (one byte per element, the OCP E4M3 "fn" format: bias 7, no
 * infinity, largest finite 448) in the layout above, and each KV head h has an
 * fp32 scale for K, k_scale[h], and for V, v_scale[h] (device arrays
 * [num_kv_heads], chosen by the caller's calibration).  A cached element
 * stands for decode(code) * scale.  Halving the KV bytes halves what decode
 * attention streams.
 *
 * pa_reshape_and_cache_fp8 -- the quantising write: element x (of `dtype`) of
 * KV head h becomes the e4m3 code of float(x) / scale[h], the quotient
 * correctly rounded in fp32, then rounded to nearest even and saturated to
 * +-448.  Slots and errors as for pa_reshape_and_cache.
 */
pa_status pa_reshape_and_cache_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                                   const int32_t* slot_mapping, const float* k_scale,
                                   const float* v_scale, int num_tokens, int num_kv_heads,
                                   int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                                   void* stream);

/*
 * pa_decode_fp8 / pa_varlen_fp8 -- pa_decode / pa_varlen over an FP8 cache:
 * the same arguments plus k_scale and v_scale; q and out have `dtype`
 * (PA_BF16, PA_F16 or PA_F32).  The result is attention over the dequantized
 * cache.  On the tensor-core path the codes become f16 (every e4m3 value is
 * exact in f16) and q is converted to f16 for the MMAs; the K scale folds into
 * the softmax scale and the V scale into the output.  Workspace sizes are
 * those of pa_decode_workspace_size / pa_varlen_workspace_size.
 */
pa_status pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const float* k_scale, const float* v_scale,
                        const int32_t* block_tables, int block_table_stride,
                        const int32_t* context_lens, int num_seqs, int num_q_heads,
                        int num_kv_heads, int head_dim, int block_size, int num_blocks,
                        int max_context_len, float scale, void* workspace,
                        size_t workspace_bytes, pa_dtype dtype, void* stream);

pa_status pa_varlen_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const float* k_scale, const float* v_scale,
                        const int32_t* block_tables, int block_table_stride,
                        const int32_t* query_start_loc, const int32_t* seq_lens, int num_seqs,
                        int total_q, int max_query_len, int max_seq_len, int num_q_heads,
                        int num_kv_heads, int head_dim, int block_size, int num_blocks,
                        float scale, void* workspace, size_t workspace_bytes, pa_dtype dtype,
                        void* stream);

/*
 * pa_copy_blocks -- copy-on-write block copies inside one pool.
 *
 * Blocks are shared by reference count ("2. 核心思想" §核心抽象: ref_cnt
 * supports copy-on-write and sharing across requests; "vLLM 架构源码解析"
 * §4.3.2: parallel samples share the prompt's blocks).  Before a request
 * writes into a block that another request still references, the engine
 * gives it a private copy; this call makes those copies.
 *
 *   k_cache, v_cache  [num_blocks, num_kv_heads, block_size, head_dim]
 *   block_mapping     int32 [num_pairs][2] = (src, dst), device memory: block
 *                     dst of both caches becomes a byte copy of block src
 *                     (every KV head, every slot)
 *
 * Pairs must be independent: no dst may be another pair's src or dst (the
 * order among pairs is unspecified).  src == dst is a no-op.  A pair with an
 * id outside [0, num_blocks) is skipped and recorded as PA_ERR_DEVICE_BOUNDS.
 * num_pairs == 0 is a no-op.
 */
pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* block_mapping,
                         int num_pairs, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype dtype, void* stream);

/*
 * pa_swap_blocks -- move blocks between two pools, e.g. the device pool and
 * a pool in host memory.
 *
 * The v0 scheduler preempts a request by swapping its KV cache out to CPU
 * memory and swaps it back into the GPU pool when the request resumes
 * ("vLLM 架构源码解析" §1, the preemption table: v0 (Swap)).
 *
 *   src_k, src_v  [src_num_blocks, num_kv_heads, block_size, head_dim]
 *   dst_k, dst_v  [dst_num_blocks, num_kv_heads, block_size, head_dim]
 *   block_mapping int32 [num_pairs][2] = (src, dst): block dst of (dst_k,
 *                 dst_v) becomes a byte copy of block src of (src_k, src_v)
 *
 * Unlike every other call, the pools and block_mapping may each be device
 * memory or page-locked host memory (cudaHostAlloc / cudaHostRegister, e.g.
 * torch's pin_memory()); the kernel reads and writes host memory through
 * its device-visible address, so a swap is one launch however many blocks
 * it moves.  Pageable host memory is refused (PA_ERR_INVALID_ARG).  The
 * caller keeps the host buffers alive and unmodified until the stream has
 * passed the call.  Pair rules and errors as for pa_copy_blocks (ids are
 * checked against the pool each side of the pair belongs to).
 */
pa_status pa_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                         const int32_t* block_mapping, int num_pairs, int num_kv_heads,
                         int head_dim, int block_size, int src_num_blocks, int dst_num_blocks,
                         pa_dtype dtype, void* stream);

/*
 * Workspace (bytes) pa_decode needs for these sizes.  Includes the split-K
 * partial results (contexts longer than one 512-token partition are split
 * and reduced by log-sum-exp) and the schedule.  Returns 0 only for empty
 * batches.
 */
size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                int max_context_len);

/*
 * pa_decode -- decode attention over the paged cache.
 *
 * "vLLM 深度拆解" §3.3 (the block-table walk, padding past context_len
 * skipped) and §6.2 (the kernel's arguments); "vLLM 架构源码解析" §3.3.3.
 *
 *   out           [num_seqs, num_q_heads, head_dim], written
 *   q             [num_seqs, num_q_heads, head_dim]  one query row per request
 *   block_tables  int32 [num_seqs, block_table_stride]
 *   context_lens  int32 [num_seqs]: cached tokens of each request, including
 *                 the one written this step by pa_reshape_and_cache.  The
 *                 query attends to tokens 0 .. context_lens[r]-1.  A zero
 *                 length gives a zero output row.  A length above
 *                 max_context_len or above block_table_stride*block_size is
 *                 a device-side bounds error (row left unwritten).
 *   max_context_len  host-side upper bound on context_lens (sizes the grid
 *                 and workspace without reading device memory).
 *   scale         multiplies q.k before the softmax (1/sqrt(head_dim) for
 *                 the pages' formula).
 *   workspace     device scratch of at least pa_decode_workspace_size(...)
 *                 bytes, 256-byte aligned, owned by the caller; its contents
 *                 are not preserved.  Concurrent calls need separate workspaces.
 */
pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int block_table_stride,
                    const int32_t* context_lens, int num_seqs, int num_q_heads,
                    int num_kv_heads, int head_dim, int block_size, int num_blocks,
                    int max_context_len, float scale, void* workspace, size_t workspace_bytes,
                    pa_dtype dtype, void* stream);

/*
 * pa_decode_static -- pa_decode for callers that cannot allocate device memory.
 *
 * The pages have no counterpart: this is a convenience of this library.
 * Some callers are handed only their input and output buffers and have no
 * way to obtain scratch memory -- a plugin inside a host runtime that owns
 * every device allocation, or a hot loop that must not call cudaMalloc
 * because cudaMalloc can synchronise the whole device.  This entry point
 * takes the same arguments as pa_decode minus the workspace, and uses a
 * fixed scratch array built into the library instead.
 *
 * - The scratch is PA_STATIC_WORKSPACE_BYTES (32 MiB) of device memory that
 *   every GPU which loads the library holds until the process exits.  A call
 *   whose pa_decode_workspace_size(...) exceeds it is rejected with
 *   PA_ERR_WORKSPACE and launches nothing.
 * - The first call on each device looks up the scratch's device address
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 * - All calls on a device share the one array: calls that may overlap on the
 *   GPU (different streams without ordering) race and corrupt each other's
 *   results.  Order them on one stream.  The array keeps the last call's
 *   contents; each call rewrites everything it reads before reading it.
 * - It allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *   routine.  Everything else -- arguments, layouts, errors -- is pa_decode's.
 */
#define PA_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)

pa_status pa_decode_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int block_table_stride,
                           const int32_t* context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           int max_context_len, float scale, pa_dtype dtype, void* stream);

/* Workspace (bytes) pa_varlen needs for these sizes. */
size_t pa_varlen_workspace_size(int num_seqs, int total_q, int num_q_heads, int num_kv_heads,
                                int head_dim, int max_query_len, int max_seq_len);

/*
 * pa_varlen -- attention for a mixed scheduler batch.
 *
 * "vLLM 架构源码解析" §3.2 (one token budget shared by prefill and decode;
 * num_new_tokens == 1 is a decode row) and §3.3.2 (query_start_loc is
 * [0, L1, L1+L2, ...]; positions run from num_computed_tokens);
 * "vLLM 深度拆解" §4.3 (chunked prefill).
 *
 *   out              [total_q, num_q_heads, head_dim], written
 *   q                [total_q, num_q_heads, head_dim]
 *   query_start_loc  int32 [num_seqs + 1]: request r owns query rows
 *                    query_start_loc[r] .. query_start_loc[r+1]-1;
 *                    query_start_loc[num_seqs] == total_q.
 *   seq_lens         int32 [num_seqs]: cached plus new tokens of request r
 *                    (the new rows already written by pa_reshape_and_cache).
 *   Query row i of request r sits at position seq_lens[r] - q_len_r + i and
 *   attends causally to keys 0 .. that position.
 *   max_query_len, max_seq_len  host-side upper bounds.
 *   workspace        as for pa_decode, sized by pa_varlen_workspace_size.
 */
pa_status pa_varlen(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int block_table_stride,
                    const int32_t* query_start_loc, const int32_t* seq_lens, int num_seqs,
                    int total_q, int max_query_len, int max_seq_len, int num_q_heads,
                    int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                    void* workspace, size_t workspace_bytes, pa_dtype dtype, void* stream);

/*
 * Synchronise `stream`, then return and clear the current device's error
 * word: PA_OK, PA_ERR_DEVICE_BOUNDS or PA_ERR_TIMEOUT (PA_ERR_CUDA if the
 * synchronisation itself failed).  Details go to pa_last_error_message.
 */
pa_status pa_get_device_error(void* stream);

/* Select the kernel family (process-wide).  Returns the previous value. */
pa_path pa_set_path(pa_path path);

/* Static, human-readable name of a status code. */
const char* pa_status_string(pa_status status);

/* Detail of the last non-OK status produced on the calling host thread. */
const char* pa_last_error_message(void);

/* Library version, major*10000 + minor*100 + patch. */
int pa_version(void);

/*
 * SM version the loaded kernels were built for, as the CUDA runtime reports
 * it for this library's code on the current device (100 = sm_100a), or -1
 * when no kernel image can be loaded there.
 */
int pa_binary_version(void);

/*
 * Test hook for the bounded waits (no counterpart in the pages).  Every wait
 * inside the kernels gives up after a limit (about one second), records
 * PA_ERR_TIMEOUT for pa_get_device_error and lets its CTA leave cleanly
 * (copies already issued land first; tensor memory is freed).  With
 * `kernel` = 1 (the decode/varlen attention kernel) or 2 (the tcgen05 chunk
 * kernel), every CTA of that kernel leaves its first K/V tile unissued in
 * every later call -- no copy, no arrival -- and the limit drops to about one
 * millisecond, so the wait for that tile runs out.  0 restores normal
 * operation.  Process-wide on the current device; synchronous.  Never set
 * in production.
 */
pa_status pa_debug_lost_load(int kernel);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
