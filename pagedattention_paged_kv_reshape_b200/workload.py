"""Seeded synthetic batches shaped like the pages' decode and mixed-batch workloads.

This module holds none of the attention arithmetic.  It draws values and lays
out the metadata a scheduler hands to the attention layer (block tables, the
per-token slot mapping, ``query_start_loc``, sequence lengths), and nothing
else.  Both the CUDA library and the fp64 oracle read the tensors it returns.

Recipe (all of it seeded):

* Metadata comes from ``numpy.random.default_rng(seed)``: lengths, which
  requests share a prefix, and a Fisher-Yates permutation of the physical pool
  (``Generator.permutation``) from which blocks are handed out in order -- the
  free-list allocator of "vLLM 深度拆解" §3.2 fed with shuffled ids, so a
  request's blocks are scattered over the pool.
* Values come from ``torch.Generator(device).manual_seed(seed)``: q, the new
  k/v rows and every cached row are N(0, 1) drawn in float32 and rounded to the
  storage dtype (round-to-nearest-even).
* Poison: every cache slot that no query may read -- the padding past each
  request's last token, blocks no request owns, the reserved poison block that
  fills unused block-table entries, and the slots this step's new tokens will
  be written to -- holds NaN.  A kernel that reads padding, reads a table entry
  past the last logical block, or attends before the cache write lands,
  produces NaN in its output.
* A request with ``shares_prefix`` uses the common prefix run of blocks as its
  first logical blocks (ref_cnt > 1, as in "vLLM 架构源码解析" §2.3 (4) and
  §4.3.1), so several block-table rows name the same physical ids.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK_SIZE = 16

TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
ELEMENT_BYTES = {"f32": 4, "bf16": 2, "f16": 2}


@dataclass
class Request:
    """One scheduled request: ``seq_len`` tokens after this step, ``q_len`` of them new."""

    seq_len: int
    q_len: int = 1
    shares_prefix: bool = False


@dataclass
class PagedBatch:
    """Device (or host) tensors for one attention call plus its host metadata."""

    name: str
    dtype: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    requests: list
    q: torch.Tensor              # [total_q, Hq, D]
    k_new: torch.Tensor          # [total_q, Hkv, D]  rows written by reshape_and_cache
    v_new: torch.Tensor          # [total_q, Hkv, D]
    slot_mapping: torch.Tensor   # int32 [total_q]
    k_cache: torch.Tensor        # [num_blocks, Hkv, block_size, D], before the write
    v_cache: torch.Tensor
    block_tables: torch.Tensor   # int32 [num_seqs, table_width]
    seq_lens: torch.Tensor       # int32 [num_seqs]  (context_lens for decode batches)
    query_start_loc: torch.Tensor  # int32 [num_seqs + 1]
    scale: float
    poison_block: int
    shared_blocks: list = field(default_factory=list)
    # host copies of the metadata (numpy) for the test harness and accounting
    host_tables: np.ndarray | None = None
    host_seq_lens: np.ndarray | None = None
    host_qsl: np.ndarray | None = None
    host_slots: np.ndarray | None = None
    # FP8 (e4m3) cache: k_cache / v_cache hold uint8 codes; per-KV-head fp32 scales
    kv_dtype: str = "same"
    k_scale: torch.Tensor | None = None
    v_scale: torch.Tensor | None = None

    @property
    def fp8(self) -> bool:
        return self.kv_dtype == "fp8"

    @property
    def num_seqs(self) -> int:
        return len(self.requests)

    @property
    def total_q(self) -> int:
        return int(self.host_qsl[-1])

    @property
    def max_query_len(self) -> int:
        return max((r.q_len for r in self.requests), default=0)

    @property
    def max_seq_len(self) -> int:
        return max((r.seq_len for r in self.requests), default=0)

    @property
    def is_decode(self) -> bool:
        return all(r.q_len == 1 for r in self.requests)

    @property
    def table_stride(self) -> int:
        return int(self.block_tables.shape[1])


def _randn_into(dst: torch.Tensor, gen: torch.Generator, chunk_rows: int = 8192) -> None:
    """Fill ``dst`` (any float dtype) with N(0,1) drawn in float32, chunk by chunk."""
    flat = dst.view(dst.shape[0], -1)
    for lo in range(0, flat.shape[0], chunk_rows):
        hi = min(lo + chunk_rows, flat.shape[0])
        tmp = torch.randn((hi - lo, flat.shape[1]), generator=gen, device=dst.device,
                          dtype=torch.float32)
        flat[lo:hi].copy_(tmp)


def build_batch(requests, *, num_q_heads: int, num_kv_heads: int, head_dim: int, dtype: str,
                seed: int, device="cpu", name: str = "custom", pool_factor: float = 1.0,
                pool_blocks: int | None = None, shared_prefix_len: int = 0,
                extra_table_cols: int = 1, poison: bool = True,
                block_size: int = BLOCK_SIZE, kv_dtype: str = "same") -> PagedBatch:
    """Lay out ``requests`` in a shuffled block pool and draw all values.

    ``pool_factor`` sizes the pool to that multiple of the blocks the batch
    needs (plus the poison block); ``pool_blocks`` fixes it instead.
    ``shared_prefix_len`` (a multiple of ``block_size``) is the length of the
    common prefix run used by requests with ``shares_prefix``.
    ``kv_dtype="fp8"`` makes an FP8 (e4m3) cache: uint8 codes drawn as the e4m3
    rounding of N(0,1) * 48 (torch's float8 conversion), per-KV-head scales
    drawn from U[0.012, 0.024], and the NaN code 0x7F in unowned slots.
    """
    if kv_dtype not in ("same", "fp8"):
        raise ValueError(f"unknown kv_dtype {kv_dtype!r}")
    if dtype not in TORCH_DTYPES:
        raise ValueError(f"unknown dtype {dtype!r}")
    if shared_prefix_len % block_size:
        raise ValueError("shared_prefix_len must be a whole number of blocks")
    rng = np.random.default_rng(seed)
    device = torch.device(device)
    n_shared = shared_prefix_len // block_size
    uses_shared = any(r.shares_prefix for r in requests)
    for r in requests:
        if r.q_len > r.seq_len or r.q_len < 0:
            raise ValueError("each request needs 0 <= q_len <= seq_len")
        if r.shares_prefix and r.seq_len - r.q_len < shared_prefix_len:
            raise ValueError("a sharing request's new tokens must lie past the shared prefix")

    logical = [-(-r.seq_len // block_size) for r in requests]
    private = [nb - (n_shared if r.shares_prefix else 0) for nb, r in zip(logical, requests)]
    need = (n_shared if uses_shared else 0) + sum(private)
    if pool_blocks is None:
        pool_blocks = max(need + 1, int(math.ceil(pool_factor * need)) + 1)
    if pool_blocks < need + 1:
        raise ValueError(f"pool of {pool_blocks} blocks cannot hold {need} + 1 poison block")

    perm = rng.permutation(pool_blocks)
    cursor = 0

    def take(n):
        nonlocal cursor
        out = perm[cursor:cursor + n]
        cursor += n
        return out

    poison_block = int(take(1)[0])
    shared = take(n_shared) if uses_shared else np.zeros(0, dtype=np.int64)
    width = max(logical, default=0) + extra_table_cols
    width = max(width, 1)
    tables = np.full((len(requests), width), poison_block, dtype=np.int32)
    for i, r in enumerate(requests):
        row = list(shared) if r.shares_prefix else []
        row += list(take(private[i]))
        tables[i, :len(row)] = row

    seq_lens = np.array([r.seq_len for r in requests], dtype=np.int32)
    qsl = np.zeros(len(requests) + 1, dtype=np.int32)
    qsl[1:] = np.cumsum([r.q_len for r in requests])
    total_q = int(qsl[-1])
    slots = np.empty(total_q, dtype=np.int32)
    for i, r in enumerate(requests):
        for j in range(r.q_len):
            pos = r.seq_len - r.q_len + j
            slots[qsl[i] + j] = tables[i, pos // block_size] * block_size + pos % block_size

    tdt = TORCH_DTYPES[dtype]
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = torch.empty((total_q, num_q_heads, head_dim), dtype=tdt, device=device)
    k_new = torch.empty((total_q, num_kv_heads, head_dim), dtype=tdt, device=device)
    v_new = torch.empty_like(k_new)
    fp8 = kv_dtype == "fp8"
    cdt = torch.float32 if fp8 else tdt
    k_cache = torch.empty((pool_blocks, num_kv_heads, block_size, head_dim), dtype=cdt,
                          device=device)
    v_cache = torch.empty_like(k_cache)
    for t in (q, k_new, v_new, k_cache, v_cache):
        if t.numel():
            _randn_into(t, gen)
    k_scale = v_scale = None
    if fp8:
        k_cache = (k_cache * 48.0).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
        v_cache = (v_cache * 48.0).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
        k_scale = torch.from_numpy(rng.uniform(0.012, 0.024, num_kv_heads).astype(np.float32))
        v_scale = torch.from_numpy(rng.uniform(0.012, 0.024, num_kv_heads).astype(np.float32))
        k_scale, v_scale = k_scale.to(device), v_scale.to(device)

    if poison and pool_blocks:
        live = np.zeros((pool_blocks, block_size), dtype=bool)
        for i, r in enumerate(requests):
            cached = r.seq_len - r.q_len      # rows already in the cache before this step
            for pos in range(0, cached, block_size):
                n = min(block_size, cached - pos)
                live[tables[i, pos // block_size], :n] = True
        dead = torch.from_numpy(~live).to(device)
        nan = 0x7F if fp8 else float("nan")   # the e4m3 NaN code for an FP8 cache
        k_cache.masked_fill_(dead[:, None, :, None], nan)
        v_cache.masked_fill_(dead[:, None, :, None], nan)

    return PagedBatch(
        name=name, dtype=dtype, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size, num_blocks=pool_blocks,
        requests=list(requests), q=q, k_new=k_new, v_new=v_new,
        slot_mapping=torch.from_numpy(slots).to(device),
        k_cache=k_cache, v_cache=v_cache,
        block_tables=torch.from_numpy(tables).to(device),
        seq_lens=torch.from_numpy(seq_lens).to(device),
        query_start_loc=torch.from_numpy(qsl).to(device),
        scale=1.0 / math.sqrt(head_dim), poison_block=poison_block,
        shared_blocks=[int(b) for b in shared],
        host_tables=tables, host_seq_lens=seq_lens, host_qsl=qsl, host_slots=slots,
        kv_dtype=kv_dtype, k_scale=k_scale, v_scale=v_scale,
    )


# ---------------------------------------------------------------------------
# The five named workloads.  Sizes follow the decode and mixed-batch shapes the
# pages discuss (Llama-2-7B-like MHA, Llama-3-8B-like GQA, 32K-token context,
# a 2048-token scheduler budget with a 512-token chunk and a shared 512-token
# system prompt).
# ---------------------------------------------------------------------------

def _log_uniform_ints(rng, n, lo, hi):
    return np.rint(np.exp(rng.uniform(math.log(lo), math.log(hi), size=n))).astype(int)


def tiny_requests(seed):
    return [Request(c) for c in (1, 17, 33, 100)]


def mha_requests(seed, batch=64, lo=256, hi=2048):
    rng = np.random.default_rng(seed + 1)
    return [Request(int(c)) for c in rng.integers(lo, hi + 1, size=batch)]


def gqa_requests(seed, batch=256, lo=128, hi=8192):
    rng = np.random.default_rng(seed + 1)
    return [Request(int(c)) for c in _log_uniform_ints(rng, batch, lo, hi)]


def long_requests(seed, batch=8, ctx=32768):
    return [Request(ctx) for _ in range(batch)]


def mixed_requests(seed, decode_rows=1536, chunk_q=512, chunk_cached=1536, lo=64, hi=4096,
                   prefix_len=512, chunk_first=False):
    """2048-token budget: one 512-token causal chunk on 1536 cached tokens plus
    1536 decode rows, half of which share the ``prefix_len``-token prefix."""
    rng = np.random.default_rng(seed + 1)
    sharing = np.zeros(decode_rows, dtype=bool)
    sharing[rng.choice(decode_rows, size=decode_rows // 2, replace=False)] = True
    reqs = []
    for s in sharing:
        if s:   # the new token lands in a private block past the shared run
            reqs.append(Request(int(rng.integers(prefix_len + 1, hi + 1)), 1, True))
        else:
            reqs.append(Request(int(rng.integers(lo, hi + 1)), 1, False))
    chunk = Request(chunk_cached + chunk_q, chunk_q, False)
    return [chunk] + reqs if chunk_first else reqs + [chunk]


def prefill_requests(seed, rows=16, chunk_q=512, cached=1536):
    """A prefill-heavy scheduler iteration: ``rows`` requests each running a
    512-token causal chunk on 1536 cached tokens (chunked prefill of long
    prompts); every row goes to the tensor-core chunk path."""
    return [Request(cached + chunk_q, chunk_q) for _ in range(rows)]


CONFIGS = {
    "tiny": dict(requests=tiny_requests, num_q_heads=4, num_kv_heads=4, head_dim=64,
                 dtype="f32", pool_blocks=64, kind="decode",
                 about="4 requests, context_lens {1,17,33,100}, 4/4 heads, head_dim 64, fp32, "
                       "64-block pool"),
    "mha_bs64": dict(requests=mha_requests, num_q_heads=32, num_kv_heads=32, head_dim=128,
                     dtype="bf16", pool_factor=1.25, kind="decode",
                     about="Llama-2-7B-shaped MHA decode, batch 64, ctx U[256,2048], 32/32 heads, "
                           "head_dim 128, bf16, pool 1.25x need"),
    "gqa_bs256": dict(requests=gqa_requests, num_q_heads=32, num_kv_heads=8, head_dim=128,
                      dtype="bf16", pool_factor=1.25, kind="decode",
                      about="Llama-3-8B-shaped GQA decode, batch 256, ctx log-uniform [128,8192], "
                            "32/8 heads, head_dim 128, bf16, 256 new tokens cached"),
    "long_32k": dict(requests=long_requests, num_q_heads=64, num_kv_heads=8, head_dim=128,
                     dtype="bf16", pool_factor=1.25, kind="decode",
                     about="long-context GQA decode, batch 8 x 32768, 64/8 heads, head_dim 128, "
                           "bf16, split-K partitions of 512"),
    "mixed_2048": dict(requests=mixed_requests, num_q_heads=32, num_kv_heads=8, head_dim=128,
                       dtype="bf16", pool_factor=1.0, shared_prefix_len=512, kind="varlen",
                       about="2048-token budget: 512-query causal chunk on 1536 cached tokens + "
                             "1536 decode rows (ctx U[64,4096], half share a 512-token prefix), "
                             "32/8 heads, head_dim 128, bf16"),
    "gqa_bs256_b8": dict(requests=gqa_requests, num_q_heads=32, num_kv_heads=8, head_dim=128,
                         dtype="bf16", pool_factor=1.25, kind="decode", block_size=8,
                         about="gqa_bs256 with 8-token blocks (\"vLLM 架构源码解析\" §5.1)"),
    "gqa_bs256_b32": dict(requests=gqa_requests, num_q_heads=32, num_kv_heads=8, head_dim=128,
                          dtype="bf16", pool_factor=1.25, kind="decode", block_size=32,
                          about="gqa_bs256 with 32-token blocks (\"vLLM 架构源码解析\" §5.1)"),
    "gqa_bs256_fp8": dict(requests=gqa_requests, num_q_heads=32, num_kv_heads=8, head_dim=128,
                          dtype="bf16", pool_factor=1.25, kind="decode", kv_dtype="fp8",
                          about="gqa_bs256 over an FP8 (e4m3) cache with per-KV-head scales "
                                "(\"vLLM 深度拆解\" §10.1)"),
    "gqa_bs256_d256": dict(requests=gqa_requests, num_q_heads=16, num_kv_heads=4,
                           head_dim=256, dtype="bf16", pool_factor=1.25, kind="decode",
                           about="gqa_bs256's lengths with head_dim 256, 16/4 heads (the same "
                                 "KV bytes per token)"),
    "prefill_16x512": dict(requests=prefill_requests, num_q_heads=32, num_kv_heads=8,
                           head_dim=128, dtype="bf16", pool_factor=1.0, kind="varlen",
                           about="16 causal prefill chunks of 512 tokens on 1536 cached tokens, "
                                 "32/8 heads, head_dim 128, bf16 (tensor-core chunk kernel)"),
    "prefill_16x512_d256": dict(requests=prefill_requests, num_q_heads=16, num_kv_heads=4,
                                head_dim=256, dtype="bf16", pool_factor=1.0, kind="varlen",
                                about="prefill_16x512's chunks with head_dim 256, 16/4 heads "
                                      "(the same KV bytes per token and FLOPs per query token)"),
}


def make_config(name: str, *, seed: int = 0, device="cpu", poison: bool = True) -> PagedBatch:
    """Build one of the named workloads (``CONFIGS``) on ``device``."""
    spec = dict(CONFIGS[name])
    reqs = spec.pop("requests")(seed)
    spec.pop("kind")
    spec.pop("about")
    return build_batch(reqs, seed=seed, device=device, name=name, poison=poison, **spec)
