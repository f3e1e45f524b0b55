"""Algorithmic byte and FLOP counts for the roofline.

Algorithmic bytes are what the operation must move at least once, whatever
the kernel does:

* attention: every cached K and V row a query may see, read once per KV head
  (``seq_len * 2 * Hkv * D * elem`` per request; a run of prefix blocks shared
  by several requests counts once), plus q and out (``total_q * Hq * D *
  elem`` each), plus the block-table entries walked (4 bytes per logical
  block) and the per-request lengths;
* reshape_and_cache: each new K and V row read once and written once, plus
  the slot mapping.

``kv_bytes_per_block`` and ``kv_bytes_per_token`` restate the pages' own
block accounting ("vLLM 架构源码解析 | 第 1 篇" §4.2; "vLLM 深度拆解" §2.1);
``tests/test_accounting.py`` pins them to the numbers printed there.
"""

from __future__ import annotations

from .workload import ELEMENT_BYTES, PagedBatch


def kv_bytes_per_block(block_size: int, num_layers: int, num_kv_heads: int, head_dim: int,
                       elem_bytes: int) -> int:
    """Bytes of one block across all layers, K and V."""
    return block_size * num_layers * 2 * num_kv_heads * head_dim * elem_bytes


def kv_bytes_per_token(num_kv_heads: int, head_dim: int, elem_bytes: int, kv: int = 2) -> int:
    """Bytes one token occupies in one layer's cache (``kv=1``: K or V alone)."""
    return kv * num_kv_heads * head_dim * elem_bytes


def blocks_that_fit(cache_bytes: int, block_bytes: int) -> int:
    return cache_bytes // block_bytes


def _logical_blocks(length: int, block_size: int) -> int:
    return -(-length // block_size)


def kv_elem_bytes(b: PagedBatch) -> int:
    """Bytes of one cached K or V element: 1 for an FP8 (e4m3) cache."""
    return 1 if b.fp8 else ELEMENT_BYTES[b.dtype]


def attention_bytes(b: PagedBatch) -> dict:
    """Algorithmic bytes of one attention call over batch ``b`` (an FP8 cache
    adds its 2 x Hkv fp32 scales)."""
    elem = ELEMENT_BYTES[b.dtype]
    per_tok = kv_bytes_per_token(b.num_kv_heads, b.head_dim, kv_elem_bytes(b))
    lens = [int(x) for x in b.host_seq_lens]
    logical_kv = sum(lens) * per_tok
    sharers = sum(1 for r in b.requests if r.shares_prefix)
    shared_tokens = len(b.shared_blocks) * b.block_size
    unique_kv = logical_kv - max(0, sharers - 1) * shared_tokens * per_tok
    qo = 2 * b.total_q * b.num_q_heads * b.head_dim * elem
    tables = 4 * sum(_logical_blocks(L, b.block_size) for L in lens)
    meta = 4 * (2 * b.num_seqs + 1) + (8 * b.num_kv_heads if b.fp8 else 0)
    return {"kv_logical": logical_kv, "kv_unique": unique_kv, "q_out": qo, "tables": tables,
            "meta": meta, "total": unique_kv + qo + tables + meta,
            "total_logical": logical_kv + qo + tables + meta}


def reshape_bytes(b: PagedBatch) -> int:
    """Algorithmic bytes of one reshape_and_cache call (read of the new rows,
    write of their cached form) plus the slot mapping."""
    elem = ELEMENT_BYTES[b.dtype]
    read = b.total_q * kv_bytes_per_token(b.num_kv_heads, b.head_dim, elem)
    write = b.total_q * kv_bytes_per_token(b.num_kv_heads, b.head_dim, kv_elem_bytes(b))
    return read + write + 4 * b.total_q


def chunk_flops(b: PagedBatch) -> int:
    """Dense QK^T + PV FLOPs of the prefill-chunk rows (q_len > 1): 4*D*Hq per
    visible (query, key) pair under the causal rule key <= position."""
    pairs = 0
    for r in b.requests:
        if r.q_len > 1:
            first = r.seq_len - r.q_len
            pairs += sum(first + i + 1 for i in range(r.q_len))
    return 4 * b.head_dim * b.num_q_heads * pairs
