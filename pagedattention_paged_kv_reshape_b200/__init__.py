"""Paged KV-cache attention for NVIDIA B200 (sm_100a).

The hot path of a paged-KV serving engine's attention layer as a C-ABI
library (``libpa.so``, declared in ``include/pa.h``) with hand-written CUDA
kernels, and this thin Python binding of it:

* :func:`pa_reshape_and_cache` -- scatter new K/V rows into 8-, 16- or 32-token
  blocks;
* :func:`pa_decode` -- block-table-indirected decode attention (GQA, online
  softmax, split-K with a log-sum-exp reduce);
* :func:`pa_varlen` -- mixed batches of decode rows and causal prefill chunks
  (the chunks on tcgen05 tensor cores with TMEM accumulators);
* :func:`pa_copy_blocks` / :func:`pa_swap_blocks` -- copy-on-write copies
  inside a pool, swap-out / swap-in between the device and a host pool;
* :func:`pa_reshape_and_cache_fp8`, :func:`pa_decode_fp8`,
  :func:`pa_varlen_fp8` -- the same path over an FP8 (e4m3) cache with
  per-KV-head scales;
* :func:`pa_rope_reshape_and_cache` -- the cache write with the rotary
  position embedding of q and k fused in.

PyTorch provides device memory and streams only.  The seeded workload
generator lives in :mod:`.workload`; byte/flop accounting in :mod:`.accounting`.
"""

from ._binding import (  # noqa: F401
    LIBRARY_PATH,
    PaError,
    Path,
    Status,
    alloc_workspace,
    lib,
    STATIC_WORKSPACE_BYTES,
    pa_binary_version,
    pa_copy_blocks,
    pa_debug_lost_load,
    pa_decode,
    pa_decode_fp8,
    pa_decode_static,
    pa_decode_workspace_size,
    pa_get_device_error,
    pa_reshape_and_cache,
    pa_reshape_and_cache_fp8,
    pa_rope_reshape_and_cache,
    pa_set_path,
    pa_status_string,
    pa_swap_blocks,
    pa_varlen,
    pa_varlen_fp8,
    pa_varlen_workspace_size,
    pa_version,
)
