"""Run the oracle over a whole batch on every host core.

TEST INFRASTRUCTURE ONLY (see the package header): only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` / reference
legs use it.

Requests, and the KV heads inside a request, are independent sub-problems of
paged attention (each query head reads one KV head, [DEEP] §3.3 walks one
request's block table at a time).  This module only splits a batch into
(request, KV head) sub-problems, hands them to a pool of worker processes and
puts the answers back in place; every number is computed by the plain
functions of this package -- ``reshape_and_cache`` (or its FP8 form) on the
request's own blocks, then ``paged_decode`` or ``paged_varlen`` -- unchanged.

A sub-problem for request r and KV head g holds:
* r's physical blocks, in logical order, restricted to KV head g (a byte
  copy); the block table becomes 0 .. nb-1;
* every new token of the batch whose slot lies in one of those blocks, with
  its slot renumbered to the copy (so a write by another request into a block
  r reads would still be seen);
* r's query rows for the query heads that read KV head g
  (``kv_head_of(h) == g``).

The large arrays (the cache pool, q and the new rows) live in shared memory,
filled once by the caller; workers attach to them by name.  The pool uses the
``spawn`` start method (no fork after a CUDA context exists), and each worker
is limited to one BLAS thread, so ``workers`` is the number of cores in use.
"""

from __future__ import annotations

import math
import multiprocessing as mp
import os
import time
from multiprocessing import shared_memory

import numpy as np

from .fp8 import paged_decode_fp8, paged_varlen_fp8, reshape_and_cache_fp8
from .paged_attention import kv_head_of, paged_decode, paged_varlen, reshape_and_cache

_BIG = ("k_cache", "v_cache", "q", "k_new", "v_new")
_STATE: dict = {}


def _attach(segments: dict, small: dict) -> None:
    """Worker initializer: map the shared arrays, keep the scalars."""
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    _STATE.clear()
    _STATE["shm"] = []
    for name, (shm_name, shape, dtype) in segments.items():
        seg = shared_memory.SharedMemory(name=shm_name)
        _STATE["shm"].append(seg)
        _STATE[name] = np.ndarray(shape, dtype=np.dtype(dtype), buffer=seg.buf)
    _STATE.update(small)


def _sub_problem(r: int, g: int) -> dict:
    """The arrays of the (request r, KV head g) sub-problem."""
    s = _STATE
    bs = s["block_size"]
    length = int(s["seq_lens"][r])
    nb = -(-length // bs)
    blocks = np.asarray(s["tables"][r, :nb], dtype=np.int64)
    where = {int(b): i for i, b in enumerate(blocks)}
    slots = np.asarray(s["slots"], dtype=np.int64)
    writes = np.nonzero((slots >= 0) & np.isin(slots // bs, blocks))[0]
    new_slots = np.array([where[int(slots[t]) // bs] * bs + int(slots[t]) % bs for t in writes],
                         dtype=np.int32)
    t0, t1 = int(s["qsl"][r]), int(s["qsl"][r + 1])
    hq, hkv = s["num_q_heads"], s["num_kv_heads"]
    heads = [h for h in range(hq) if kv_head_of(h, hq, hkv) == g]
    return dict(
        length=length,
        kc=s["k_cache"][blocks, g:g + 1], vc=s["v_cache"][blocks, g:g + 1],
        kn=s["k_new"][writes, g:g + 1], vn=s["v_new"][writes, g:g + 1],
        slots=new_slots, table=np.arange(max(nb, 1), dtype=np.int32)[None, :],
        q=s["q"][t0:t1][:, heads], t0=t0, t1=t1, heads=heads)


def _solve(unit):
    t_start = time.perf_counter()
    r, g = unit
    s = _STATE
    p = _sub_problem(r, g)
    bs, dt, scale = s["block_size"], s["dtype"], s["scale"]
    lens = np.array([p["length"]], dtype=np.int32)
    qsl = np.array([0, p["t1"] - p["t0"]], dtype=np.int32)
    if s["fp8"]:
        ks, vs = s["k_scale"][g:g + 1], s["v_scale"][g:g + 1]
        kc, vc = reshape_and_cache_fp8(p["kc"], p["vc"], p["kn"], p["vn"], p["slots"], ks, vs,
                                       dt, block_size=bs)
        if s["varlen"]:
            out = paged_varlen_fp8(p["q"], kc, vc, ks, vs, p["table"], qsl, lens, scale, dt,
                                   block_size=bs)
        else:
            out = paged_decode_fp8(p["q"], kc, vc, ks, vs, p["table"], lens, scale, dt,
                                   block_size=bs)
    else:
        kc, vc = reshape_and_cache(p["kc"], p["vc"], p["kn"], p["vn"], p["slots"],
                                   block_size=bs)
        if s["varlen"]:
            out = paged_varlen(p["q"], kc, vc, p["table"], qsl, lens, scale, dt, block_size=bs)
        else:
            out = paged_decode(p["q"], kc, vc, p["table"], lens, scale, dt, block_size=bs)
    algorithmic = p["length"] * 2 * p["kc"].shape[-1] * p["kc"].itemsize \
        + 2 * p["q"].size * p["q"].itemsize + 4 * p["table"].shape[1]
    return r, g, p["t0"], p["heads"], out, algorithmic, time.perf_counter() - t_start


def units_of(num_seqs: int, num_kv_heads: int, order: str = "interleaved"):
    """Every (request, KV head) pair; 'interleaved' spreads long requests."""
    return [(r, g) for g in range(num_kv_heads) for r in range(num_seqs)] \
        if order == "interleaved" else [(r, g) for r in range(num_seqs)
                                        for g in range(num_kv_heads)]


class OraclePool:
    """Shared batch arrays plus a pool of oracle workers.

    Usage: ``p = OraclePool(); a = p.array("k_cache", shape, dtype)`` for each
    of k_cache, v_cache, q, k_new, v_new (fill them), then ``p.start(**small)``
    and ``p.solve_batch()`` (or ``p.map(units)``); ``p.close()`` at the end
    (also on ``with``).
    """

    def __init__(self, workers: int | None = None):
        self.workers = workers or os.cpu_count() or 1
        self._segs: dict = {}
        self._arrays: dict = {}
        self._pool = None
        self._small: dict = {}

    def array(self, name: str, shape, dtype) -> np.ndarray:
        if name not in _BIG:
            raise ValueError(f"unknown shared array {name!r}")
        dtype = np.dtype(dtype)
        nbytes = max(1, int(np.prod(shape)) * dtype.itemsize)
        seg = shared_memory.SharedMemory(create=True, size=nbytes)
        self._segs[name] = (seg, tuple(int(x) for x in shape), dtype.str)
        arr = np.ndarray(shape, dtype=dtype, buffer=seg.buf)
        self._arrays[name] = arr
        return arr

    def _share(self, name: str, a) -> np.ndarray:
        """A shared copy of a (small) metadata array."""
        a = np.ascontiguousarray(a)
        seg = shared_memory.SharedMemory(create=True, size=max(1, a.nbytes))
        self._segs[name] = (seg, a.shape, a.dtype.str)
        arr = np.ndarray(a.shape, dtype=a.dtype, buffer=seg.buf)
        arr[...] = a
        self._arrays[name] = arr
        return arr

    def start(self, *, tables, seq_lens, qsl, slots, num_q_heads: int, num_kv_heads: int,
              block_size: int, dtype: str, scale: float, varlen: bool, fp8: bool = False,
              k_scale=None, v_scale=None) -> None:
        missing = [n for n in _BIG if n not in self._segs]
        if missing:
            raise ValueError(f"shared arrays not created: {missing}")
        # Metadata goes to shared memory too: the spawn start method pickles
        # the initializer's arguments through a pipe that each new process
        # drains only after its start-up imports, so they must stay small.
        for name, a in (("tables", tables), ("seq_lens", seq_lens), ("qsl", qsl),
                        ("slots", slots)):
            self._share(name, a)
        self._small = dict(num_q_heads=int(num_q_heads), num_kv_heads=int(num_kv_heads),
                           block_size=int(block_size), dtype=dtype, scale=float(scale),
                           varlen=bool(varlen), fp8=bool(fp8),
                           k_scale=None if k_scale is None else np.asarray(k_scale, np.float32),
                           v_scale=None if v_scale is None else np.asarray(v_scale, np.float32))
        segments = {n: (seg.name, shape, dt) for n, (seg, shape, dt) in self._segs.items()}
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS",
                                                 "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        try:
            ctx = mp.get_context("spawn")
            self._pool = ctx.Pool(self.workers, initializer=_attach,
                                  initargs=(segments, self._small))
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v

    def map(self, units, chunksize: int | None = None):
        """Results ``(r, g, t0, heads, out, algorithmic_bytes, seconds)`` of
        ``units`` (``seconds``: the worker's time on that sub-problem)."""
        units = list(units)
        if chunksize is None:
            chunksize = max(1, min(16, math.ceil(len(units) / (8 * self.workers))))
        return list(self._pool.imap_unordered(_solve, units, chunksize=chunksize))

    def solve_batch(self) -> np.ndarray:
        """The oracle's output for every query row of the batch (float64)."""
        q = self._arrays["q"]
        out = np.zeros(q.shape, dtype=np.float64)
        n = len(self._arrays["seq_lens"])
        for r, g, t0, heads, o, _, _ in self.map(units_of(n, self._small["num_kv_heads"])):
            out[t0:t0 + o.shape[0], heads] = o
        return out

    def close(self) -> None:
        if self._pool is not None:
            self._pool.terminate()
            self._pool.join()
            self._pool = None
        for seg, _, _ in self._segs.values():
            seg.close()
            try:
                seg.unlink()
            except FileNotFoundError:
                pass
        self._segs.clear()
        self._arrays.clear()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
