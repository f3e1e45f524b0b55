"""Test plumbing: run the CUDA path and the oracle on the same seeded batch.

The oracle only ever sees host copies of the generator's tensors (never a
value the CUDA path produced).  Full-size batches go to ``oracle_full``: the
batch's tensors are copied once into shared host memory and the plain oracle
runs on every (request, KV head) sub-problem on all host cores.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle as O
import pagedattention_paged_kv_reshape_b200 as pa
from pagedattention_paged_kv_reshape_b200.workload import PagedBatch

# max-abs and mean-abs bounds: bf16/f16 inputs with fp32 accumulation, and fp32 inputs
TOL = {"bf16": (1e-2, 1e-3), "f16": (1e-2, 1e-3), "f32": (1e-5, 1e-5)}


def host(t: torch.Tensor) -> np.ndarray:
    """A tensor in the oracle's encoding (bf16 as uint16 bit patterns)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().double().numpy()


# ---------------------------------------------------------------------------
# CUDA path
# ---------------------------------------------------------------------------

def gpu_cache_write(b: PagedBatch):
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    if b.fp8:
        pa.pa_reshape_and_cache_fp8(b.k_new, b.v_new, kc, vc, b.slot_mapping, b.k_scale,
                                    b.v_scale)
    else:
        pa.pa_reshape_and_cache(b.k_new, b.v_new, kc, vc, b.slot_mapping)
    return kc, vc


def poisoned_workspace(nbytes: int, device) -> torch.Tensor:
    """A workspace whose every byte is 0xFF (NaN as fp32, -1 as int32), so a
    kernel that reads scratch before writing it in the same call shows it."""
    ws = pa.alloc_workspace(nbytes, device)
    ws.fill_(0xFF)
    return ws


def gpu_attention(b: PagedBatch, kc, vc, varlen: bool | None = None, out=None):
    varlen = (not b.is_decode) if varlen is None else varlen
    if out is None:
        out = torch.full_like(b.q, float("nan"))
    if varlen:
        ws = poisoned_workspace(pa.pa_varlen_workspace_size(
            b.num_seqs, b.total_q, b.num_q_heads, b.num_kv_heads, b.head_dim, b.max_query_len,
            b.max_seq_len), b.q.device)
        if b.fp8:
            pa.pa_varlen_fp8(out, b.q, kc, vc, b.k_scale, b.v_scale, b.block_tables,
                             b.query_start_loc, b.seq_lens, b.max_query_len, b.max_seq_len,
                             b.scale, ws)
        else:
            pa.pa_varlen(out, b.q, kc, vc, b.block_tables, b.query_start_loc, b.seq_lens,
                         b.max_query_len, b.max_seq_len, b.scale, ws)
    else:
        ws = poisoned_workspace(pa.pa_decode_workspace_size(
            b.num_seqs, b.num_q_heads, b.num_kv_heads, b.head_dim, b.max_seq_len), b.q.device)
        if b.fp8:
            pa.pa_decode_fp8(out, b.q, kc, vc, b.k_scale, b.v_scale, b.block_tables, b.seq_lens,
                             b.max_seq_len, b.scale, ws)
        else:
            pa.pa_decode(out, b.q, kc, vc, b.block_tables, b.seq_lens, b.max_seq_len, b.scale, ws)
    pa.pa_get_device_error()
    return out


def gpu_step(b: PagedBatch, varlen: bool | None = None):
    kc, vc = gpu_cache_write(b)
    return gpu_attention(b, kc, vc, varlen), kc, vc


# ---------------------------------------------------------------------------
# oracle
# ---------------------------------------------------------------------------

def oracle_step(b: PagedBatch, varlen: bool | None = None, seqs=None):
    """Oracle cache write then attention, on host copies of the batch."""
    varlen = (not b.is_decode) if varlen is None else varlen
    bs = b.block_size
    q = host(b.q)
    if b.fp8:
        ks, vs = host(b.k_scale), host(b.v_scale)
        kc, vc = O.reshape_and_cache_fp8(host(b.k_cache), host(b.v_cache), host(b.k_new),
                                         host(b.v_new), b.host_slots, ks, vs, b.dtype,
                                         block_size=bs)
        if varlen:
            out = O.paged_varlen_fp8(q, kc, vc, ks, vs, b.host_tables, b.host_qsl,
                                     b.host_seq_lens, b.scale, b.dtype, block_size=bs, seqs=seqs)
        else:
            out = O.paged_decode_fp8(q, kc, vc, ks, vs, b.host_tables, b.host_seq_lens, b.scale,
                                     b.dtype, block_size=bs, seqs=seqs)
        return out, kc, vc
    kc, vc = O.reshape_and_cache(host(b.k_cache), host(b.v_cache), host(b.k_new),
                                 host(b.v_new), b.host_slots, block_size=bs)
    if varlen:
        out = O.paged_varlen(q, kc, vc, b.host_tables, b.host_qsl, b.host_seq_lens, b.scale,
                             b.dtype, block_size=bs, seqs=seqs)
    else:
        out = O.paged_decode(q, kc, vc, b.host_tables, b.host_seq_lens, b.scale, b.dtype,
                             block_size=bs, seqs=seqs)
    return out, kc, vc


def assert_close(gpu_out: torch.Tensor, ref: np.ndarray, dtype: str, what: str = ""):
    got = f64(gpu_out)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    max_tol, mean_tol = TOL[dtype]
    assert err.max() <= max_tol, f"{what}: max abs err {err.max():.3e} > {max_tol}"
    assert err.mean() <= mean_tol, f"{what}: mean abs err {err.mean():.3e} > {mean_tol}"
    return float(err.max()), float(err.mean())


# ---------------------------------------------------------------------------
# the oracle on every row of a (full-size) batch, on all host cores
# ---------------------------------------------------------------------------

_NP_OF = {torch.bfloat16: np.int16, torch.float16: np.float16, torch.float32: np.float32,
          torch.uint8: np.uint8}


def _fill_shared(pool, name: str, t: torch.Tensor) -> None:
    """Copy tensor ``t`` into the pool's shared array ``name`` (bf16 as its
    16-bit patterns, the oracle's encoding)."""
    npdt = _NP_OF[t.dtype]
    arr = pool.array(name, tuple(t.shape), np.uint16 if t.dtype == torch.bfloat16 else npdt)
    view = arr.view(npdt) if t.dtype == torch.bfloat16 else arr
    src = t.view(torch.int16) if t.dtype == torch.bfloat16 else t
    torch.from_numpy(view).copy_(src)


def oracle_full(b: PagedBatch, varlen: bool | None = None, workers: int | None = None):
    """Oracle output (float64, ``[total_q, Hq, D]``) for every query row of
    ``b``: the batch's input tensors go to shared host memory once and
    ``oracle.parallel`` solves its (request, KV head) sub-problems on all host
    cores with the plain oracle functions."""
    from oracle.parallel import OraclePool

    varlen = (not b.is_decode) if varlen is None else varlen
    with OraclePool(workers) as pool:
        for name in ("k_cache", "v_cache", "q", "k_new", "v_new"):
            _fill_shared(pool, name, getattr(b, name))
        pool.start(tables=b.host_tables, seq_lens=b.host_seq_lens, qsl=b.host_qsl,
                   slots=b.host_slots, num_q_heads=b.num_q_heads,
                   num_kv_heads=b.num_kv_heads, block_size=b.block_size, dtype=b.dtype,
                   scale=b.scale, varlen=varlen, fp8=b.fp8,
                   k_scale=None if not b.fp8 else host(b.k_scale),
                   v_scale=None if not b.fp8 else host(b.v_scale))
        return pool.solve_batch()
