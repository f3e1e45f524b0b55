"""ctypes binding of ``libpa.so`` (the C ABI in ``include/pa.h``).

Argument marshalling only: each function checks that tensors have the shape,
dtype and device the C call documents, passes their ``data_ptr()`` and the
current CUDA stream, and turns a non-OK status into :class:`PaError`.  Every
step of the computation runs in the library's CUDA kernels; there is no
fallback of any kind.  If the library is missing, the first call raises.
"""

from __future__ import annotations

import ctypes
import enum
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_PKG, "libpa.so")

_c_int, _c_float, _c_size, _vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p


class Status(enum.IntEnum):
    OK = 0
    INVALID_ARG = 1
    UNSUPPORTED = 2
    WORKSPACE = 3
    CUDA = 4
    DEVICE_BOUNDS = 5
    TIMEOUT = 6


class Path(enum.IntEnum):
    AUTO = 0
    SIMT = 1
    MMA = 2
    TCGEN05 = 3


DTYPE_CODES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
E4M3 = 3  # FP8 cache codes (torch.uint8 or torch.float8_e4m3fn pools)
FP8_CACHE_DTYPES = (torch.uint8, torch.float8_e4m3fn)

# name -> (restype, argtypes); mirrors include/pa.h
_SIGNATURES = {
    "pa_reshape_and_cache": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int,
                                      _c_int, _c_int, _vp]),
    "pa_reshape_and_cache_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int,
                                          _c_int, _c_int, _c_int, _c_int, _vp]),
    "pa_decode_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int,
                               _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _vp, _c_size,
                               _c_int, _vp]),
    "pa_varlen_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _c_int,
                               _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                               _c_float, _vp, _c_size, _c_int, _vp]),
    "pa_rope_reshape_and_cache": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int,
                                           _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                           _c_int, _c_int, _c_int, _vp]),
    "pa_copy_blocks": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                _vp]),
    "pa_swap_blocks": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                _c_int, _c_int, _vp]),
    "pa_decode_workspace_size": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "pa_decode": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int, _c_int,
                           _c_int, _c_int, _c_int, _c_float, _vp, _c_size, _c_int, _vp]),
    "pa_decode_static": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int,
                                  _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _vp]),
    "pa_varlen_workspace_size": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                           _c_int]),
    "pa_varlen": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _c_int, _c_int, _c_int,
                           _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _vp, _c_size,
                           _c_int, _vp]),
    "pa_get_device_error": (_c_int, [_vp]),
    "pa_set_path": (_c_int, [_c_int]),
    "pa_status_string": (ctypes.c_char_p, [_c_int]),
    "pa_last_error_message": (ctypes.c_char_p, []),
    "pa_version": (_c_int, []),
    "pa_binary_version": (_c_int, []),
    "pa_debug_lost_load": (_c_int, [_c_int]),
}

_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded on first use; raises if it was not built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIBRARY_PATH):
                    raise RuntimeError(
                        f"{LIBRARY_PATH} is missing: build it with "
                        "`python -m pagedattention_paged_kv_reshape_b200.build`")
                handle = ctypes.CDLL(LIBRARY_PATH)
                for name, (res, args) in _SIGNATURES.items():
                    fn = getattr(handle, name)
                    fn.restype, fn.argtypes = res, args
                _lib = handle
    return _lib


class PaError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = Status(status) if status in Status._value2member_map_ else status
        super().__init__(f"{getattr(self.status, 'name', status)}: {message}")


def _check(status: int) -> None:
    if status != 0:
        msg = lib().pa_last_error_message()
        raise PaError(status, msg.decode() if msg else "")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _require(cond: bool, what: str) -> None:
    if not cond:
        raise ValueError(what)


def _dtype_code(t: torch.Tensor) -> int:
    _require(t.dtype in DTYPE_CODES, f"unsupported dtype {t.dtype}")
    return DTYPE_CODES[t.dtype]


def _dense(*ts):
    for t in ts:
        _require(t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors")


def pa_reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """Write ``k``, ``v`` ``[T, Hkv, D]`` into ``k_cache``/``v_cache``
    ``[num_blocks, Hkv, 16, D]`` at the slots of ``slot_mapping`` (int32 ``[T]``)."""
    _dense(k, v, k_cache, v_cache, slot_mapping)
    _require(k.shape == v.shape and k.dim() == 3, "k, v must be [T, Hkv, D]")
    _require(k_cache.shape == v_cache.shape and k_cache.dim() == 4, "caches must be 4-D")
    _require(k_cache.shape[1] == k.shape[1] and k_cache.shape[3] == k.shape[2],
             "cache heads/head_dim must match k")
    _require(k.dtype == v.dtype == k_cache.dtype == v_cache.dtype, "dtypes must match")
    _require(slot_mapping.dtype == torch.int32 and slot_mapping.numel() == k.shape[0],
             "slot_mapping must be int32 [T]")
    _check(lib().pa_reshape_and_cache(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), k.shape[0],
        k.shape[1], k.shape[2], k_cache.shape[2], k_cache.shape[0], _dtype_code(k),
        _stream(stream)))


def pa_rope_reshape_and_cache(q, k, v, k_cache, v_cache, slot_mapping, positions, cos_sin,
                              neox: bool = True, stream=None) -> None:
    """Rotate ``q`` ``[T, Hq, D]`` in place and write the rotated ``k`` and the
    ``v`` rows ``[T, Hkv, D]`` into the caches at ``slot_mapping``; angles from
    ``cos_sin`` fp32 ``[max_position, rot_dim]`` at int32 ``positions``."""
    _dense(q, k, v, k_cache, v_cache, slot_mapping, positions, cos_sin)
    _require(q.dim() == 3 and k.shape == v.shape and k.dim() == 3 and q.shape[0] == k.shape[0]
             and q.shape[2] == k.shape[2], "q [T, Hq, D], k/v [T, Hkv, D]")
    _require(k_cache.shape == v_cache.shape and k_cache.dim() == 4
             and k_cache.shape[1] == k.shape[1] and k_cache.shape[3] == k.shape[2],
             "caches [num_blocks, Hkv, block_size, D]")
    _require(q.dtype == k.dtype == v.dtype == k_cache.dtype == v_cache.dtype, "dtypes must match")
    _require(slot_mapping.dtype == torch.int32 and positions.dtype == torch.int32
             and slot_mapping.numel() == positions.numel() == q.shape[0],
             "slot_mapping and positions must be int32 [T]")
    _require(cos_sin.dtype == torch.float32 and cos_sin.dim() == 2, "cos_sin fp32 [P, rot_dim]")
    _check(lib().pa_rope_reshape_and_cache(
        _ptr(q), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
        _ptr(positions), _ptr(cos_sin), cos_sin.shape[0], cos_sin.shape[1], int(bool(neox)),
        q.shape[0], q.shape[1], k.shape[1], q.shape[2], k_cache.shape[2], k_cache.shape[0],
        _dtype_code(q), _stream(stream)))


def _pool_code(t) -> int:
    return E4M3 if t.dtype in FP8_CACHE_DTYPES else _dtype_code(t)


def _pool_pair(k_pool, v_pool, what: str):
    _require(k_pool.shape == v_pool.shape and k_pool.dim() == 4, f"{what} pools must be 4-D")
    _require(k_pool.dtype == v_pool.dtype, f"{what} dtypes must match")
    _require(k_pool.is_contiguous() and v_pool.is_contiguous(), f"{what} pools must be dense")


def _block_mapping(block_mapping) -> int:
    _require(block_mapping.dtype == torch.int32 and block_mapping.dim() == 2
             and block_mapping.shape[1] == 2 and block_mapping.is_contiguous(),
             "block_mapping must be a dense int32 [num_pairs, 2]")
    return block_mapping.shape[0]


def pa_copy_blocks(k_cache, v_cache, block_mapping, stream=None) -> None:
    """Copy-on-write: for each row (src, dst) of ``block_mapping``, block ``dst``
    of both caches becomes a copy of block ``src``."""
    _dense(k_cache, v_cache, block_mapping)
    _pool_pair(k_cache, v_cache, "cache")
    n = _block_mapping(block_mapping)
    nb, hkv, bs, d = k_cache.shape
    _check(lib().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_mapping), n, hkv, d, bs,
                                nb, _pool_code(k_cache), _stream(stream)))


def pa_swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping, stream=None) -> None:
    """Swap out / in: for each row (src, dst) of ``block_mapping``, block ``dst``
    of (``dst_k``, ``dst_v``) becomes a copy of block ``src`` of (``src_k``,
    ``src_v``).  Each pool and the mapping may be on the device or in pinned
    host memory."""
    for t in (src_k, src_v, dst_k, dst_v, block_mapping):
        _require(t.is_cuda or t.is_pinned(), "host tensors must be pinned (pin_memory())")
    _pool_pair(src_k, src_v, "source")
    _pool_pair(dst_k, dst_v, "destination")
    _require(src_k.shape[1:] == dst_k.shape[1:] and src_k.dtype == dst_k.dtype,
             "source and destination blocks must have the same shape and dtype")
    n = _block_mapping(block_mapping)
    _, hkv, bs, d = src_k.shape
    _check(lib().pa_swap_blocks(_ptr(src_k), _ptr(src_v), _ptr(dst_k), _ptr(dst_v),
                                _ptr(block_mapping), n, hkv, d, bs, src_k.shape[0],
                                dst_k.shape[0], _pool_code(src_k), _stream(stream)))


def pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                             max_context_len) -> int:
    return int(lib().pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              max_context_len))


def pa_varlen_workspace_size(num_seqs, total_q, num_q_heads, num_kv_heads, head_dim,
                             max_query_len, max_seq_len) -> int:
    return int(lib().pa_varlen_workspace_size(num_seqs, total_q, num_q_heads, num_kv_heads,
                                              head_dim, max_query_len, max_seq_len))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned uint8 buffer of at least ``nbytes`` (torch's caching
    allocator returns 512-byte aligned blocks)."""
    buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    assert buf.data_ptr() % 256 == 0
    return buf


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
              scale: float, workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """Decode attention.  ``q``/``out``: ``[S, Hq, D]``; ``block_tables`` int32
    ``[S, stride]``; ``context_lens`` int32 ``[S]``."""
    _dense(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    _require(q.shape == out.shape and q.dim() == 3 and q.dtype == out.dtype, "q/out shape")
    _require(block_tables.dtype == torch.int32 and context_lens.dtype == torch.int32,
             "metadata must be int32")
    S, hq, d = q.shape
    _check(lib().pa_decode(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), S, hq, k_cache.shape[1], d, k_cache.shape[2],
        k_cache.shape[0], int(max_context_len), float(scale), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _dtype_code(q), _stream(stream)))
    return out


STATIC_WORKSPACE_BYTES = 32 << 20


def pa_decode_static(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
                     scale: float, stream=None) -> torch.Tensor:
    """:func:`pa_decode` for callers that cannot allocate device memory: the
    split-K scratch is a fixed 32 MiB array built into the library.  Calls on
    one device share it, so calls that may overlap on the GPU race; the first
    call on a device should come before any stream capture."""
    _dense(out, q, k_cache, v_cache, block_tables, context_lens)
    _require(q.shape == out.shape and q.dim() == 3 and q.dtype == out.dtype, "q/out shape")
    _require(block_tables.dtype == torch.int32 and context_lens.dtype == torch.int32,
             "metadata must be int32")
    S, hq, d = q.shape
    _check(lib().pa_decode_static(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), S, hq, k_cache.shape[1], d, k_cache.shape[2],
        k_cache.shape[0], int(max_context_len), float(scale), _dtype_code(q), _stream(stream)))
    return out


def pa_varlen(out, q, k_cache, v_cache, block_tables, query_start_loc, seq_lens,
              max_query_len: int, max_seq_len: int, scale: float, workspace: torch.Tensor,
              stream=None) -> torch.Tensor:
    """Mixed decode/prefill-chunk attention.  ``q``/``out``: ``[total_q, Hq, D]``;
    ``query_start_loc`` int32 ``[S+1]``; ``seq_lens`` int32 ``[S]``."""
    _dense(out, q, k_cache, v_cache, block_tables, query_start_loc, seq_lens, workspace)
    _require(q.shape == out.shape and q.dim() == 3 and q.dtype == out.dtype, "q/out shape")
    _require(query_start_loc.dtype == torch.int32 and seq_lens.dtype == torch.int32 and
             block_tables.dtype == torch.int32, "metadata must be int32")
    _require(query_start_loc.numel() == seq_lens.numel() + 1, "query_start_loc must be [S+1]")
    total_q, hq, d = q.shape
    _check(lib().pa_varlen(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(query_start_loc), _ptr(seq_lens), seq_lens.numel(), total_q,
        int(max_query_len), int(max_seq_len), hq, k_cache.shape[1], d, k_cache.shape[2],
        k_cache.shape[0], float(scale), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _dtype_code(q), _stream(stream)))
    return out


def _fp8_pools(k_cache, v_cache, k_scale, v_scale):
    _require(k_cache.dtype in FP8_CACHE_DTYPES and v_cache.dtype == k_cache.dtype,
             "FP8 caches must be uint8 or float8_e4m3fn")
    _require(k_scale.dtype == torch.float32 and v_scale.dtype == torch.float32
             and k_scale.numel() == k_cache.shape[1] == v_scale.numel(),
             "k_scale / v_scale must be float32 [num_kv_heads]")
    _dense(k_cache, v_cache, k_scale, v_scale)


def pa_reshape_and_cache_fp8(k, v, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                             stream=None) -> None:
    """Quantising write of ``k``, ``v`` ``[T, Hkv, D]`` into the FP8 (e4m3) caches
    at ``slot_mapping``: code = e4m3(float(x) / scale[head])."""
    _dense(k, v, slot_mapping)
    _fp8_pools(k_cache, v_cache, k_scale, v_scale)
    _require(k.shape == v.shape and k.dim() == 3, "k, v must be [T, Hkv, D]")
    _require(k_cache.shape[1] == k.shape[1] and k_cache.shape[3] == k.shape[2],
             "cache heads/head_dim must match k")
    _require(slot_mapping.dtype == torch.int32 and slot_mapping.numel() == k.shape[0],
             "slot_mapping must be int32 [T]")
    _check(lib().pa_reshape_and_cache_fp8(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), _ptr(k_scale),
        _ptr(v_scale), k.shape[0], k.shape[1], k.shape[2], k_cache.shape[2], k_cache.shape[0],
        _dtype_code(k), _stream(stream)))


def pa_decode_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                  max_context_len: int, scale: float, workspace: torch.Tensor,
                  stream=None) -> torch.Tensor:
    """Decode attention over an FP8 cache (workspace: ``pa_decode_workspace_size``)."""
    _dense(out, q, block_tables, context_lens, workspace)
    _fp8_pools(k_cache, v_cache, k_scale, v_scale)
    _require(q.shape == out.shape and q.dim() == 3 and q.dtype == out.dtype, "q/out shape")
    _require(block_tables.dtype == torch.int32 and context_lens.dtype == torch.int32,
             "metadata must be int32")
    S, hq, d = q.shape
    _check(lib().pa_decode_fp8(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
        _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S, hq, k_cache.shape[1],
        d, k_cache.shape[2], k_cache.shape[0], int(max_context_len), float(scale),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _dtype_code(q),
        _stream(stream)))
    return out


def pa_varlen_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, query_start_loc,
                  seq_lens, max_query_len: int, max_seq_len: int, scale: float,
                  workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """Mixed batch over an FP8 cache (workspace: ``pa_varlen_workspace_size``)."""
    _dense(out, q, block_tables, query_start_loc, seq_lens, workspace)
    _fp8_pools(k_cache, v_cache, k_scale, v_scale)
    _require(q.shape == out.shape and q.dim() == 3 and q.dtype == out.dtype, "q/out shape")
    _require(block_tables.dtype == torch.int32 and query_start_loc.dtype == torch.int32
             and seq_lens.dtype == torch.int32, "metadata must be int32")
    T, hq, d = q.shape
    S = seq_lens.numel()
    _check(lib().pa_varlen_fp8(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
        _ptr(block_tables), block_tables.shape[1], _ptr(query_start_loc), _ptr(seq_lens), S, T,
        int(max_query_len), int(max_seq_len), hq, k_cache.shape[1], d, k_cache.shape[2],
        k_cache.shape[0], float(scale), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _dtype_code(q), _stream(stream)))
    return out


def pa_get_device_error(stream=None) -> None:
    """Synchronise ``stream``; raise :class:`PaError` if a kernel recorded an error."""
    _check(lib().pa_get_device_error(_stream(stream)))


def pa_set_path(path: Path | int) -> Path:
    """Select the kernel family (process-wide); returns the previous one."""
    return Path(lib().pa_set_path(int(path)))


def pa_status_string(status: int) -> str:
    return lib().pa_status_string(int(status)).decode()


def pa_version() -> int:
    return int(lib().pa_version())


def pa_binary_version() -> int:
    """SM version of the loaded kernel image on the current device (100 = sm_100a)."""
    return int(lib().pa_binary_version())


def pa_debug_lost_load(kernel: int) -> None:
    """Test hook of the bounded waits (see include/pa.h): 1 or 2 makes every CTA
    of the attention or chunk kernel leave its first K/V tile unissued, with a
    wait limit of about a millisecond; 0 restores normal operation."""
    _check(lib().pa_debug_lost_load(int(kernel)))
