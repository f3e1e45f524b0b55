#!/usr/bin/env python
"""Benchmark of the paged-attention hot path on B200.

One step = one pass of the whole hot path over one seeded synthetic batch:
``pa_reshape_and_cache`` of the step's new K/V rows, then paged attention
(``pa_varlen`` for mixed batches, ``pa_decode`` for decode batches), all
through the C ABI.  The KV cache is resident in HBM (it is the engine's state);
``value`` is the step's algorithmic bytes (every visible K/V row once, a
shared prefix once, q, out, block-table entries, the cache write) over the
device time of the step, in GB/s.  The headline workload is the mixed
scheduler iteration (a 512-token causal prefill chunk next to 1536 decode
rows, half of them sharing a 512-token prefix): the largest batch, and the
one that runs both halves of the path.

``roofline`` times the attention call alone in a loop of back-to-back calls
(events around the loop only), so its duration is at most a step's.  ``e2e``
repeats the step with each step's inputs copied from pinned host memory and
its output copied back inside the timed region.

Usage:  python bench.py [--gpus N --steps K --warmup W] [--workload NAME]
        python bench.py --impl reference ...   (the fp64 oracle on host cores)
Multi-GPU: launch under torchrun; every rank runs its own batch (data-parallel
replicas, no collective on the data path) and rank 0 prints the JSON line.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("paged-attn decode KV-read GB/s (% of B200 HBM peak); decode tokens/s per config")
HEADLINE = "mixed_2048"
PER_CONFIG = ("mha_bs64", "gqa_bs256", "long_32k", "mixed_2048", "prefill_16x512",
              "gqa_bs256_b8", "gqa_bs256_b32", "gqa_bs256_fp8", "gqa_bs256_d256",
              "prefill_16x512_d256")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--per-config-steps", type=int, default=100)
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU-seconds of oracle work in the cpu_baseline sample")
    ap.add_argument("--requests", type=int, default=0,
                    help="keep only the first N decode requests of the workload (its chunk rows "
                         "stay): a smaller case of the same recipe, e.g. for profiler captures")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s, kind): MEASURED_PEAKS.json, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# Sources the attention kernels are compiled from (traffic records are keyed to them).
ATTENTION_SOURCES = ("pa_common.cuh", "pa_sched.cuh", "pa_attn_mma.cuh",
                     "pa_chunk_tc2.cuh", "pa_tcgen05.cuh", "pa_reduce.cuh", "pa_api.cu")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in ATTENTION_SOURCES:
        with open(os.path.join(ROOT, "pagedattention_paged_kv_reshape_b200", "csrc", name),
                  "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes of one attention call from the committed ncu summary, if it
    was taken on the current kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            e = json.load(f).get(workload)
        if e and e.get("source_hash") == kernel_source_hash():
            return e.get("dram_bytes_per_call")
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# clocks: nvidia-smi sampled from the first warm-up step to the end of the run
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("timestamp,uuid,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    INTERVAL_MS = 20

    def __init__(self, uuid: str):
        self.uuid = uuid.lower().replace("gpu-", "")
        self.marks = {}
        self.lines = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.INTERVAL_MS)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def mark(self, name: str) -> None:
        self.marks[name] = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.reader.join(timeout=5)
        rows = []
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10 or f[1].lower().replace("gpu-", "") != self.uuid:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[2]), float(f[3]), float(f[5]),
                             {n for n, v in zip(self.REASONS, f[6:10])
                              if v.lower().startswith("active")}))
            except ValueError:
                continue
        load = [r for r in rows if r[3] >= 30.0]
        t0, t1 = self.marks.get("timed_start"), self.marks.get("timed_end")
        timed = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        reasons = sorted(set().union(*[r[4] for r in load])) if load else []
        return {"sm_mhz": statistics.median(r[1] for r in load) if load else None,
                "sm_max_mhz": max(r[2] for r in rows) if rows else None,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "samples_in_timed_region": len(timed),
                "timed_region_sm_mhz": statistics.median(r[1] for r in timed) if timed else None,
                "interval_ms": self.INTERVAL_MS,
                "note": "nvidia-smi from the first warm-up step to the end of the run "
                        "(per_config and e2e included); 'under load' = utilization >= 30%"}


# ---------------------------------------------------------------------------
# the fp64 oracle on host cores (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def host_sample_batch(W, workload: str, seed: int, max_requests: int):
    """A host (CPU) batch of the workload's recipe holding its first requests
    (the chunk rows of a mixed batch are kept): the oracle's sample."""
    spec = dict(W.CONFIGS[workload])
    reqs = spec.pop("requests")(seed)
    spec.pop("kind")
    spec.pop("about")
    chunks = [r for r in reqs if r.q_len > 1]
    decode = [r for r in reqs if r.q_len <= 1]
    keep = decode[:max(0, max_requests - len(chunks[:2]))] + chunks[:2]
    if not any(r.shares_prefix for r in keep):
        spec.pop("shared_prefix_len", None)
    return W.build_batch(keep, seed=seed, device="cpu", name=workload, **spec)


def oracle_pool_for(batch, workers=None):
    """An oracle.parallel pool over the host batch (its tensors in shared memory)."""
    import numpy as np
    import torch

    from oracle.parallel import OraclePool

    pool = OraclePool(workers)
    for name in ("k_cache", "v_cache", "q", "k_new", "v_new"):
        t = getattr(batch, name)
        if t.dtype == torch.bfloat16:
            arr = pool.array(name, tuple(t.shape), np.uint16)
            torch.from_numpy(arr.view(np.int16)).copy_(t.view(torch.int16))
        else:
            arr = pool.array(name, tuple(t.shape), t.numpy().dtype)
            arr[...] = t.numpy()
    pool.start(tables=batch.host_tables, seq_lens=batch.host_seq_lens, qsl=batch.host_qsl,
               slots=batch.host_slots, num_q_heads=batch.num_q_heads,
               num_kv_heads=batch.num_kv_heads, block_size=batch.block_size, dtype=batch.dtype,
               scale=batch.scale, varlen=not batch.is_decode, fp8=batch.fp8,
               k_scale=None if not batch.fp8 else batch.k_scale.numpy(),
               v_scale=None if not batch.fp8 else batch.v_scale.numpy())
    return pool


def run_oracle_units(pool, units):
    """(wall seconds, algorithmic bytes, CPU seconds) of the oracle on ``units``."""
    t0 = time.perf_counter()
    res = pool.map(units)
    wall = time.perf_counter() - t0
    return wall, sum(r[5] for r in res), sum(r[6] for r in res)


def cpu_baseline(W, workload: str, seed: int, cpu_seconds: float) -> dict:
    """The oracle, as it stands, on every host core over a bounded sample of
    the workload's (request, KV head) sub-problems."""
    from oracle.parallel import units_of

    batch = host_sample_batch(W, workload, seed, max_requests=48)
    pool = oracle_pool_for(batch)
    try:
        units = units_of(batch.num_seqs, batch.num_kv_heads)
        run_oracle_units(pool, units[:pool.workers])          # workers warm
        wall = nbytes = cpu = 0.0
        rounds = 0
        while cpu < cpu_seconds and rounds < 50:
            w_, b_, c_ = run_oracle_units(pool, units)
            wall, nbytes, cpu, rounds = wall + w_, nbytes + b_, cpu + c_, rounds + 1
        return {"value": round(nbytes / wall / 1e9, 5), "unit": "GB/s", "cores": pool.workers,
                "kind": "oracle",
                "sample": f"{rounds} pass(es) over the {len(units)} (request, KV head) "
                          f"sub-problems of a host batch of {batch.num_seqs} requests of "
                          f"{workload}'s recipe ({nbytes / 1e6:.1f} MB of algorithmic bytes, "
                          f"{cpu:.1f} CPU-s in {wall:.2f} s on {pool.workers} worker processes)"}
    finally:
        pool.close()


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def cache_write(pa, b, k_new, v_new, slots):
    """pa_reshape_and_cache (or its quantising FP8 form) into ``b``'s pool."""
    if b.fp8:
        pa.pa_reshape_and_cache_fp8(k_new, v_new, b.k_cache, b.v_cache, slots, b.k_scale,
                                    b.v_scale)
    else:
        pa.pa_reshape_and_cache(k_new, v_new, b.k_cache, b.v_cache, slots)


def attention(pa, b, out, q, tables, lens, qsl, ws):
    """pa_decode / pa_varlen (or the FP8 forms) over ``b``'s pool."""
    if not b.is_decode:
        if b.fp8:
            pa.pa_varlen_fp8(out, q, b.k_cache, b.v_cache, b.k_scale, b.v_scale, tables, qsl,
                             lens, b.max_query_len, b.max_seq_len, b.scale, ws)
        else:
            pa.pa_varlen(out, q, b.k_cache, b.v_cache, tables, qsl, lens, b.max_query_len,
                         b.max_seq_len, b.scale, ws)
    elif b.fp8:
        pa.pa_decode_fp8(out, q, b.k_cache, b.v_cache, b.k_scale, b.v_scale, tables, lens,
                         b.max_seq_len, b.scale, ws)
    else:
        pa.pa_decode(out, q, b.k_cache, b.v_cache, tables, lens, b.max_seq_len, b.scale, ws)


def workspace_for(pa, b):
    if b.is_decode:
        n = pa.pa_decode_workspace_size(b.num_seqs, b.num_q_heads, b.num_kv_heads, b.head_dim,
                                        b.max_seq_len)
    else:
        n = pa.pa_varlen_workspace_size(b.num_seqs, b.total_q, b.num_q_heads, b.num_kv_heads,
                                        b.head_dim, b.max_query_len, b.max_seq_len)
    return pa.alloc_workspace(n, b.q.device)


def launches_per_step(b) -> int:
    """Our kernels per step: cache write, schedule, attention, then the
    tcgen05 chunk kernel (rows of >= one 128-row tile of new tokens) and the
    split-K reduce (contexts over one 512-key partition) when the batch has them."""
    group = b.num_q_heads // b.num_kv_heads
    gs = min(group, 16)
    chunk_qt = 128 // gs if gs in (1, 2, 4, 8, 16) else 0
    chunk = (not b.is_decode and not b.fp8 and b.head_dim != 256 and chunk_qt > 0
             and b.max_query_len >= chunk_qt)
    split = math.ceil(b.max_seq_len / 512) > 1
    return 3 + int(chunk) + int(split)


def timed_loop(torch, fn, n: int, warmup: int = 3) -> float:
    """Mean ms of ``fn`` over ``n`` back-to-back calls, CUDA events on the
    launching stream around the loop only."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(n):
        fn()
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e) / n


# Idle time before each timed loop.  Under a sustained full-bandwidth load the
# B200 reaches its power cap within about 50 ms and slows by a few percent
# (the largest batch's back-to-back calls went from 1.96 to 2.2 ms over 0.7 s);
# a short rest before every loop gives each the same starting point, so the
# attention call and the whole step are timed under the same conditions.
REST_S = 1.0


def measure_workload(torch, pa, b, steps: int, warmup: int, sampler=None):
    """(step ms, attention-call ms, cache-write ms): K steps (cache write +
    attention) between two events after W warm-up steps, then the attention
    call alone and the cache write alone, each in its own loop of K calls,
    each loop after REST_S of idle time.  Every input is larger than the L2
    except the cache write's few MB."""
    out = torch.empty_like(b.q)
    ws = workspace_for(pa, b)

    def write():
        cache_write(pa, b, b.k_new, b.v_new, b.slot_mapping)

    def attend():
        attention(pa, b, out, b.q, b.block_tables, b.seq_lens, b.query_start_loc, ws)

    def step():
        write()
        attend()

    for _ in range(warmup):
        step()
    pa.pa_get_device_error()
    torch.cuda.synchronize()
    time.sleep(REST_S)
    if sampler:
        sampler.mark("timed_start")
    step_ms = timed_loop(torch, step, steps, warmup=0)
    if sampler:
        sampler.mark("timed_end")
    time.sleep(REST_S)
    attn_ms = timed_loop(torch, attend, steps, warmup=1)
    time.sleep(REST_S)
    write_ms = timed_loop(torch, write, steps)
    pa.pa_get_device_error()
    return step_ms, attn_ms, write_ms


def time_e2e(torch, pa, b, steps):
    """Each step copies its inputs from pinned host memory to the device and its
    output back, all inside the timed region.  The copies run on their own
    streams with two sets of device buffers, so step i+1's inputs move while
    step i computes and step i's output returns while step i+1 computes (a
    serving loop's overlap); events order every reuse of a buffer."""
    names = ["q", "k_new", "v_new", "slot_mapping", "block_tables", "seq_lens", "query_start_loc"]
    host = {n: getattr(b, n).cpu().pin_memory() for n in names}
    comp = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = []
    for _ in range(2):
        bufs.append({"dev": {n: torch.empty_like(getattr(b, n)) for n in names},
                     "out": torch.empty_like(b.q),
                     "out_host": torch.empty(b.q.shape, dtype=b.q.dtype, pin_memory=True),
                     "ready": torch.cuda.Event(), "computed": torch.cuda.Event(),
                     "returned": torch.cuda.Event(), "used": False})
    ws = workspace_for(pa, b)

    def step(i):
        buf = bufs[i % 2]
        dev = buf["dev"]
        with torch.cuda.stream(h2d_s):
            if buf["used"]:
                h2d_s.wait_event(buf["computed"])     # step i-2 has read these inputs
            for n in names:
                dev[n].copy_(host[n], non_blocking=True)
            buf["ready"].record(h2d_s)
        comp.wait_event(buf["ready"])
        if buf["used"]:
            comp.wait_event(buf["returned"])          # step i-2's output has left
        cache_write(pa, b, dev["k_new"], dev["v_new"], dev["slot_mapping"])
        attention(pa, b, buf["out"], dev["q"], dev["block_tables"], dev["seq_lens"],
                  dev["query_start_loc"], ws)
        buf["computed"].record(comp)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(buf["computed"])
            buf["out_host"].copy_(buf["out"], non_blocking=True)
            buf["returned"].record(d2h_s)
        buf["used"] = True

    for i in range(5):
        step(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    h2d_s.wait_event(start)
    for i in range(steps):
        step(i)
    for buf in bufs:
        comp.wait_event(buf["returned"])
    end.record(comp)
    torch.cuda.synchronize()
    pa.pa_get_device_error()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = bufs[0]["out_host"].numel() * bufs[0]["out_host"].element_size()
    return start.elapsed_time(end) / steps, h2d, d2h


def combine_over_ranks(local_ms: float, local_bytes: float, local_tokens: float, device):
    """Whole-job throughput: the slowest rank's time, every rank's bytes and
    tokens.  Returns (max_ms, GB/s, tokens/s); works on any process group
    backend (NCCL on GPUs, gloo in the CPU tests) or with none."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    nb = torch.tensor([float(local_bytes)], dtype=torch.float64, device=device)
    tok = torch.tensor([float(local_tokens)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(nb, op=dist.ReduceOp.SUM)
        dist.all_reduce(tok, op=dist.ReduceOp.SUM)
    max_ms = float(t.item())
    return max_ms, nb.item() / (max_ms / 1e3) / 1e9, tok.item() / (max_ms / 1e3)


def measure_device_copy(torch, dev) -> float:
    """Context for the peak: torch's device-to-device copy of a 2 GiB buffer
    (read + write bytes over time), on this machine, in this run."""
    n = 1 << 31
    src = torch.empty(n, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    time.sleep(REST_S)
    ms = timed_loop(torch, lambda: dst.copy_(src), 10)
    del src, dst
    torch.cuda.empty_cache()
    return round(2 * n / (ms * 1e-3) / 1e9, 1)


def measure_block_ops(torch, pa, dev, peak) -> dict:
    """Copy-on-write copies inside the device pool and swaps to / from a pinned
    host pool, each on 2048 / 1024 blocks of 8 KV heads x 16 x 128 bf16
    (64 KB of K+V per block; 256 MB of HBM traffic per copy call, more than
    the L2).  GB/s count the bytes each call reads plus writes (copy) or
    moves (swap)."""
    nb, hkv, d = 6144, 8, 128
    g = torch.Generator(device=dev).manual_seed(1234)
    k = torch.randn(nb, hkv, 16, d, generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn(nb, hkv, 16, d, generator=g, device=dev).to(torch.bfloat16)
    block_bytes = 2 * hkv * 16 * d * 2
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(1234))
    n_copy, n_swap = 2048, 1024
    cmap = torch.stack([perm[:n_copy], perm[n_copy:2 * n_copy]], 1).int().to(dev)
    host_k = torch.empty(n_swap, hkv, 16, d, dtype=torch.bfloat16).pin_memory()
    host_v = torch.empty_like(host_k).pin_memory()
    omap = torch.stack([perm[:n_swap], torch.arange(n_swap)], 1).int().to(dev)
    imap = torch.stack([torch.arange(n_swap), perm[2 * n_copy:2 * n_copy + n_swap]], 1).int().to(dev)
    copy_ms = timed_loop(torch, lambda: pa.pa_copy_blocks(k, v, cmap), 10)
    out_ms = timed_loop(torch, lambda: pa.pa_swap_blocks(k, v, host_k, host_v, omap), 10)
    in_ms = timed_loop(torch, lambda: pa.pa_swap_blocks(host_k, host_v, k, v, imap), 10)
    pa.pa_get_device_error()
    copy_gbs = 2 * n_copy * block_bytes / (copy_ms / 1e3) / 1e9
    return {"copy_blocks": {"pairs": n_copy, "ms": round(copy_ms, 4),
                            "gbs_read_plus_write": round(copy_gbs, 1),
                            "pct_of_hbm_peak": round(100 * copy_gbs / peak, 1)},
            "swap_out": {"blocks": n_swap, "ms": round(out_ms, 4),
                         "gbs": round(n_swap * block_bytes / (out_ms / 1e3) / 1e9, 1)},
            "swap_in": {"blocks": n_swap, "ms": round(in_ms, 4),
                        "gbs": round(n_swap * block_bytes / (in_ms / 1e3) / 1e9, 1)},
            "blocks": "8 KV heads x 16 tokens x 128 dims, bf16, K and V"}


def measure_rope_write(torch, pa, dev, peak) -> dict:
    """pa_rope_reshape_and_cache on 16384 new tokens (32 query / 8 KV heads,
    head_dim 128, bf16, full rotation, NeoX pairs): q is read and written, k and
    v read, both cache rows written, plus one table row, position and slot per
    token -- about 410 MB per call, more than the L2."""
    T, hq, hkv, d, bs = 16384, 32, 8, 128, 16
    g = torch.Generator(device=dev).manual_seed(77)
    q = torch.randn(T, hq, d, generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn(T, hkv, d, generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn(T, hkv, d, generator=g, device=dev).to(torch.bfloat16)
    nb = T // bs + 64
    kc = torch.zeros(nb, hkv, bs, d, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(77))[:T // bs]
    slots = (perm.repeat_interleave(bs) * bs + torch.arange(T) % bs).int().to(dev)
    positions = (torch.arange(T) % 8192).int().to(dev)
    inv = 10000.0 ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)
    ang = torch.arange(8192, dtype=torch.float64)[:, None] * inv[None, :]
    table = torch.cat([ang.cos(), ang.sin()], 1).float().to(dev)
    ms = timed_loop(torch, lambda: pa.pa_rope_reshape_and_cache(q, k, v, kc, vc, slots,
                                                                positions, table), 20)
    pa.pa_get_device_error()
    nbytes = (2 * T * hq * d * 2 + 2 * T * hkv * d * 2 + 2 * T * hkv * d * 2 + T * d * 4
              + 8 * T)
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"tokens": T, "ms": round(ms, 4), "algorithmic_bytes": nbytes, "gbs": round(gbs, 1),
            "pct_of_hbm_peak": round(100 * gbs / peak, 1)}


def per_config_entry(A, b, step_ms, attn_ms, write_ms, peak, tensor_peak) -> dict:
    acc = A.attention_bytes(b)
    sb = acc["total"] + A.reshape_bytes(b)
    attn_gbs = acc["total"] / (attn_ms / 1e3) / 1e9
    ent = {"step_gbs": round(sb / (step_ms / 1e3) / 1e9, 1),
           "attention_gbs": round(attn_gbs, 1),
           "pct_of_hbm_peak": round(100 * attn_gbs / peak, 1),
           "ms_per_step": round(step_ms, 4), "attention_ms": round(attn_ms, 4),
           "cache_write_ms": round(write_ms, 4),
           "tokens_per_s": round(b.total_q / (step_ms / 1e3), 1)}
    if A.chunk_flops(b):
        ent["chunk_gflop"] = round(A.chunk_flops(b) / 1e9, 2)
    if any(r.shares_prefix for r in b.requests):
        ent["unique_vs_logical_kv"] = [acc["kv_unique"], acc["kv_logical"]]
    if all(r.q_len > 1 for r in b.requests):   # dense causal chunks: a tensor-core roofline
        tflops = A.chunk_flops(b) / (attn_ms / 1e3) / 1e12
        ent.update({"chunk_tflops": round(tflops, 1),
                    "pct_of_bf16_peak": round(100 * tflops / tensor_peak, 1),
                    "tokens_per_s": round(b.total_q / (attn_ms / 1e3), 1)})
    return ent


def make_batch(W, workload: str, seed: int, device, requests: int = 0):
    """The named workload, or (requests > 0) a smaller case of its recipe: its
    first `requests` decode requests plus all its chunk rows."""
    if requests <= 0:
        return W.make_config(workload, seed=seed, device=device)
    spec = dict(W.CONFIGS[workload])
    reqs = spec.pop("requests")(seed)
    spec.pop("kind")
    spec.pop("about")
    keep = [r for r in reqs if r.q_len <= 1][:requests] + [r for r in reqs if r.q_len > 1]
    return W.build_batch(keep, seed=seed, device=device, name=f"{workload}[:{requests}]", **spec)


def run_ours(args):
    import torch
    import torch.distributed as dist

    import pagedattention_paged_kv_reshape_b200 as pa
    from pagedattention_paged_kv_reshape_b200 import accounting as A
    from pagedattention_paged_kv_reshape_b200 import build as pa_build
    from pagedattention_paged_kv_reshape_b200 import workload as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        pa_build.build(quiet=True)
    if world > 1:
        dist.barrier()
    pa.lib()

    dev = torch.device("cuda", local)
    peak, tensor_peak, peak_kind = measured_peaks()
    b = make_batch(W, args.workload, args.seed + rank, dev, args.requests)
    acc = A.attention_bytes(b)
    step_bytes = acc["total"] + A.reshape_bytes(b)

    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(str(props.uuid)) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms, attn_ms, write_ms = measure_workload(torch, pa, b, args.steps, args.warmup,
                                                  sampler)
    max_ms, value, tok_per_s = combine_over_ranks(step_ms * args.steps,
                                                  step_bytes * args.steps,
                                                  b.total_q * args.steps, dev)
    attn_t = torch.tensor([attn_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(attn_t, op=dist.ReduceOp.MAX)
    attn_ms = attn_t.item()

    time.sleep(REST_S)
    e2e_ms, h2d, d2h = (float("nan"), 0, 0) if args.no_e2e else time_e2e(torch, pa, b,
                                                                       args.e2e_steps)
    e2e = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e, op=dist.ReduceOp.MAX)
    e2e_value = step_bytes * world / (e2e.item() / 1e3) / 1e9

    achieved = acc["total"] / (attn_ms / 1e3) / 1e9
    peak_note = ("of measured (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                 else f"of fallback ({FALLBACK_HBM_GBS:.0f} GB/s; MEASURED_PEAKS.json absent)")
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(max_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": b.dtype,
        "data": "synthetic (seeded N(0,1) q/k/v, shuffled block pool, NaN-poisoned padding)",
        "config": {"workload": args.workload if args.requests <= 0 else
                   f"{args.workload} (first {args.requests} decode requests)",
                   "about": W.CONFIGS[args.workload]["about"],
                   "num_seqs": b.num_seqs, "total_q": b.total_q,
                   "kv_tokens": int(b.host_seq_lens.sum()),
                   "pool_bytes": 2 * b.k_cache.numel() * b.k_cache.element_size(),
                   "l2": "inputs larger than L2 (KV read per step "
                         f"{acc['kv_unique'] / 1e6:.0f} MB vs 126 MB L2); no flush",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "seed": args.seed},
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "tokens_per_s": round(tok_per_s, 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": recorded_traffic(args.workload),
                     "kernel": ("one pa_varlen call (schedule_kernel + attn_mma_kernel + "
                                "chunk_tc2_kernel + reduce_kernel)" if not b.is_decode else
                                "one pa_decode call (schedule_kernel + attn_mma_kernel "
                                "[+ reduce_kernel])"),
                     "timing": f"CUDA events on the launching stream around a loop of "
                               f"{args.steps} back-to-back calls (mean {attn_ms:.4f} ms)",
                     "algorithmic_bytes_per_launch": acc["total"],
                     "peak_kind": peak_note},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e.item(), 5)},
        "cache_write": {"ms": round(write_ms, 5), "bytes": A.reshape_bytes(b),
                        "note": "pa_reshape_and_cache alone, a loop of back-to-back calls; "
                                "launch-latency bound (a few MB), not a bandwidth figure"},
        "gpu_launches": launches_per_step(b) * args.steps,
    }

    if not args.no_per_config:
        per = {args.workload: per_config_entry(A, b, step_ms, attn_ms, write_ms, peak,
                                               tensor_peak)}
        for name in PER_CONFIG:
            if name == args.workload:
                continue
            del b
            torch.cuda.empty_cache()
            b = W.make_config(name, seed=args.seed + rank, device=dev)
            s_ms, a_ms, w_ms = measure_workload(torch, pa, b, args.per_config_steps,
                                                max(3, args.warmup // 4))
            per[name] = per_config_entry(A, b, s_ms, a_ms, w_ms, peak, tensor_peak)
        result["per_config"] = per
        result["block_ops"] = measure_block_ops(torch, pa, dev, peak)
        result["rope_cache_write"] = measure_rope_write(torch, pa, dev, peak)
        result["peaks"] = {"hbm_gbs": peak, "bf16_tflops": tensor_peak, "kind": peak_kind,
                           "device_copy_gbs": measure_device_copy(torch, dev)}
    result["clocks"] = sampler.stop() if sampler else None

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(W, args.workload, args.seed, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on host cores
# ---------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from oracle.parallel import units_of
    from pagedattention_paged_kv_reshape_b200 import workload as W

    # the same recipe on the host (values differ from the GPU draw; shapes match)
    b = host_sample_batch(W, args.workload, args.seed, max_requests=64)
    pool = oracle_pool_for(b)
    try:
        units = units_of(b.num_seqs, b.num_kv_heads)
        # calibrate the sub-problems per step so the whole run takes ~2-3 minutes
        w_, _, _ = run_oracle_units(pool, units)
        per_unit = max(w_ / len(units), 1e-5)
        budget = min(6.0, 150.0 / max(1, args.steps + args.warmup))
        per_step = max(pool.workers, int(budget / per_unit))
        cursor = 0

        def next_units():
            nonlocal cursor
            out = [units[(cursor + i) % len(units)] for i in range(per_step)]
            cursor += per_step
            return out

        for _ in range(args.warmup):
            run_oracle_units(pool, next_units())
        s = nb = cpu = 0.0
        for _ in range(args.steps):
            w_, b_, c_ = run_oracle_units(pool, next_units())
            s, nb, cpu = s + w_, nb + b_, cpu + c_
        cores = pool.workers
    finally:
        pool.close()
    value = nb / s / 1e9
    sample = (f"{per_step} (request, KV head) sub-problems per step, cycling over a host batch "
              f"of {b.num_seqs} requests of {args.workload}'s recipe; {cpu:.1f} CPU-s over "
              f"{cores} worker processes")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": b.dtype,
        "data": "synthetic (seeded N(0,1))",
        "config": {"workload": args.workload, "about": W.CONFIGS[args.workload]["about"]},
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
