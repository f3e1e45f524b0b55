"""Test plumbing: run the CUDA path and the oracle on the same seeded batch.

The oracle only ever sees host copies of the generator's tensors (never a
value the CUDA path produced).  For full-size batches the oracle runs on a
compact copy of a few sampled requests: their blocks are copied out of the
pool (an exact byte copy) and their block ids renumbered; nothing else moves.
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


def compact(b: PagedBatch, rows) -> dict:
    """Host copy of requests ``rows`` of a (large) batch with renumbered blocks."""
    rows = list(rows)
    tables = b.host_tables[rows]
    lens = b.host_seq_lens[rows]
    used = sorted({int(tables[i, j]) for i in range(len(rows))
                   for j in range(-(-int(lens[i]) // b.block_size))})
    remap = {old: new for new, old in enumerate(used)}
    idx = torch.tensor(used, dtype=torch.long, device=b.k_cache.device)
    kc = host(b.k_cache.index_select(0, idx)) if used else host(b.k_cache[:0])
    vc = host(b.v_cache.index_select(0, idx)) if used else host(b.v_cache[:0])
    new_tables = np.zeros_like(tables)
    for i in range(len(rows)):
        for j in range(-(-int(lens[i]) // b.block_size)):
            new_tables[i, j] = remap[int(tables[i, j])]
    tok = np.concatenate([np.arange(b.host_qsl[r], b.host_qsl[r + 1]) for r in rows]) \
        if rows else np.zeros(0, np.int64)
    qsl = np.zeros(len(rows) + 1, np.int32)
    qsl[1:] = np.cumsum([b.host_qsl[r + 1] - b.host_qsl[r] for r in rows])
    slots = b.host_slots[tok]
    new_slots = np.array([remap[int(s) // b.block_size] * b.block_size + int(s) % b.block_size
                          for s in slots], dtype=np.int32)
    ti = torch.from_numpy(tok.astype(np.int64)).to(b.q.device)
    return dict(tokens=tok, tables=new_tables, lens=lens, qsl=qsl, slots=new_slots, kc=kc, vc=vc,
                q=host(b.q.index_select(0, ti)), k_new=host(b.k_new.index_select(0, ti)),
                v_new=host(b.v_new.index_select(0, ti)))


def oracle_rows(b: PagedBatch, rows, varlen: bool | None = None):
    """Oracle output (float64) for the query tokens of requests ``rows``."""
    varlen = (not b.is_decode) if varlen is None else varlen
    c = compact(b, rows)
    bs = b.block_size
    if b.fp8:
        ks, vs = host(b.k_scale), host(b.v_scale)
        kc, vc = O.reshape_and_cache_fp8(c["kc"], c["vc"], c["k_new"], c["v_new"], c["slots"],
                                         ks, vs, b.dtype, block_size=bs)
        if varlen:
            out = O.paged_varlen_fp8(c["q"], kc, vc, ks, vs, c["tables"], c["qsl"], c["lens"],
                                     b.scale, b.dtype, block_size=bs)
        else:
            out = O.paged_decode_fp8(c["q"], kc, vc, ks, vs, c["tables"], c["lens"], b.scale,
                                     b.dtype, block_size=bs)
        return c["tokens"], out
    kc, vc = O.reshape_and_cache(c["kc"], c["vc"], c["k_new"], c["v_new"], c["slots"],
                                 block_size=bs)
    if varlen:
        out = O.paged_varlen(c["q"], kc, vc, c["tables"], c["qsl"], c["lens"], b.scale, b.dtype,
                             block_size=bs)
    else:
        out = O.paged_decode(c["q"], kc, vc, c["tables"], c["lens"], b.scale, b.dtype,
                             block_size=bs)
    return c["tokens"], out


def assert_close(gpu_out: torch.Tensor, ref: np.ndarray, dtype: str, what: str = ""):
    got = f64(gpu_out)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    max_tol, mean_tol = TOL[dtype]
    assert err.max() <= max_tol, f"{what}: max abs err {err.max():.3e} > {max_tol}"
    assert err.mean() <= mean_tol, f"{what}: mean abs err {err.mean():.3e} > {mean_tol}"
    return float(err.max()), float(err.mean())
