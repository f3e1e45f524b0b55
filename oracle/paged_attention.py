"""Plain fp64 definition of reshape_and_cache and paged attention.

TEST INFRASTRUCTURE ONLY (see the package header).  Slow on purpose: a Python
loop over requests, blocks, query rows and heads; numpy does the dot products,
``exp`` and sums of one query row at a time.

Cache layout (the reading taken where the pages disagree, see [DEEP] §6.2 and
[ARCH] §4.2): ``k_cache`` and ``v_cache`` are each ``[num_blocks, num_kv_heads,
block_size, head_dim]``.  A physical block holds ``block_size`` consecutive
tokens of one request ([CORE] §核心抽象 2 "Block"; [ARCH] §1.1, 16 tokens).

Value encodings accepted everywhere (``dtype`` argument):
  "f32"  -> numpy float32 arrays
  "f16"  -> numpy float16 arrays
  "bf16" -> numpy uint16 arrays holding the bfloat16 bit patterns
"""

from __future__ import annotations

import numpy as np

# [CORE] §核心抽象 2 ("常见为 16"); [ARCH] §1.1 ("默认 16 tokens") and §5.1.
BLOCK_SIZE = 16


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact conversion of stored values to float64.

    bfloat16 is the upper half of an IEEE binary32, so its value is the
    binary32 whose high 16 bits are the stored pattern and whose low 16 bits
    are zero; every binary32 and binary16 value is exact in binary64.
    """
    if dtype == "bf16":
        if a.dtype != np.uint16:
            raise TypeError("bf16 values must be passed as uint16 bit patterns")
        wide = a.astype(np.uint32) << np.uint32(16)
        return wide.view(np.float32).astype(np.float64)
    if dtype == "f16":
        return np.asarray(a, dtype=np.float16).astype(np.float64)
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == "f64":  # values already decoded (e.g. a dequantized FP8 cache)
        return np.asarray(a, dtype=np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


def slot_to_block_offset(slot: int, block_size: int = BLOCK_SIZE) -> tuple[int, int]:
    """A flat cache slot names (physical block, offset inside the block).

    [ARCH] §3.3.2 builds a per-token ``slot_mapping`` in ``_prepare_inputs``;
    [DEEP] §3.3 shows logical block ``i`` of a request living in physical block
    ``block_tables[seq*stride + i]``.  The flat slot is therefore
    ``physical_block * block_size + offset``.
    """
    return slot // block_size, slot % block_size


def reshape_and_cache(k_cache, v_cache, k, v, slot_mapping, block_size: int = BLOCK_SIZE):
    """Write this step's new K/V rows into the paged cache.

    [ARCH] §3.3.3: ``cache_ops.reshape_and_cache(k, v, kv_cache, slot_mapping)``
    runs before ``paged_attention`` in every attention layer.  Token ``t``'s
    rows ``k[t]``, ``v[t]`` (``[num_kv_heads, head_dim]``) go to the slot
    ``slot_mapping[t]``; a negative slot marks a padding token and is skipped.

    Returns new arrays (the inputs are not modified).  Values are copied
    bit-for-bit in their stored encoding.
    """
    k_out = np.array(k_cache, copy=True)
    v_out = np.array(v_cache, copy=True)
    for t in range(len(slot_mapping)):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        blk, off = slot_to_block_offset(slot, block_size)
        k_out[blk, :, off, :] = k[t]
        v_out[blk, :, off, :] = v[t]
    return k_out, v_out


def gather_sequence(cache, table_row, length: int, block_size: int = BLOCK_SIZE):
    """Contiguous ``[length, num_kv_heads, head_dim]`` copy of one request.

    Walks the request's logical blocks in order and looks each one up in its
    block-table row, as in the loop of [DEEP] §3.3 ("physical_block_id =
    block_tables[seq_id * stride + block_idx]"); tokens at or past the context
    length are never touched ("跳过 padding token").  Table entries past the
    last logical block are never read.
    """
    num_kv_heads, head_dim = cache.shape[1], cache.shape[3]
    out = np.empty((length, num_kv_heads, head_dim), dtype=cache.dtype)
    num_logical = -(-length // block_size)
    for logical in range(num_logical):
        physical = int(table_row[logical])
        first = logical * block_size
        count = min(block_size, length - first)
        # cache[physical] is [num_kv_heads, block_size, head_dim]; its first
        # ``count`` token rows are the live ones.
        out[first:first + count] = cache[physical, :, :count, :].transpose(1, 0, 2)
    return out


def kv_head_of(q_head: int, num_q_heads: int, num_kv_heads: int) -> int:
    """KV head read by a query head.

    The pages show multi-head attention only ([DEEP] §2.1, §6.2 use one
    ``num_heads``).  Reading taken for grouped-query attention: query heads are
    split into ``num_kv_heads`` contiguous groups of ``num_q_heads /
    num_kv_heads``; group ``g`` reads KV head ``g``.  With equal head counts
    this is the identity, i.e. plain multi-head attention.
    """
    group = num_q_heads // num_kv_heads
    return q_head // group


def query_positions(seq_len: int, q_len: int) -> list[int]:
    """Absolute positions of a request's query rows in this step.

    [ARCH] §3.3.2 ``_prepare_inputs``: a prefill chunk's positions are
    ``range(num_computed_tokens, num_computed_tokens + num_tokens)`` and a
    decode row's position is ``num_computed_tokens``.  ``seq_len`` counts the
    cached tokens plus this step's new tokens, so the rows sit at
    ``seq_len - q_len + i``.
    """
    return [seq_len - q_len + i for i in range(q_len)]


def softmax_attention(q_row, keys, values, scale: float):
    """``softmax(q · K^T * scale) · V`` for one query row, in float64.

    [DEEP] §2.2: ``Attention(Q, K, V) = softmax(Q · K^T / √d) · V``; §3.3 and
    §6.2 multiply the dot product by a scale (``/ sqrt(head_dim)``).  The
    softmax subtracts the row maximum before ``exp`` (the value is unchanged
    mathematically; it only keeps ``exp`` finite).  An empty key set gives a
    zero row.
    """
    n = keys.shape[0]
    if n == 0:
        return np.zeros(values.shape[1], dtype=np.float64)
    scores = scale * (keys @ q_row)          # s_j = scale * <q, k_j>
    weights = np.exp(scores - scores.max())  # unnormalised softmax weights
    weights /= weights.sum()
    return weights @ values                  # sum_j w_j v_j


def _check_heads(num_q_heads: int, num_kv_heads: int) -> None:
    if num_kv_heads <= 0 or num_q_heads % num_kv_heads != 0:
        raise ValueError("num_q_heads must be a positive multiple of num_kv_heads")


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, dtype: str,
                 block_size: int = BLOCK_SIZE, seqs=None):
    """Decode attention: one query row per request over its cached context.

    ``q``: ``[num_seqs, num_q_heads, head_dim]``; ``context_lens[r]`` counts
    request ``r``'s cached tokens including the one written this step by
    :func:`reshape_and_cache` (decode "needs the K and V of all previous
    tokens", [CORE] §设计理念; the write precedes the read, [ARCH] §3.3.3).
    ``paged_attention(q, kv_cache, block_tables, context_lens)`` of [ARCH]
    §3.3.3 and the kernel signature of [DEEP] §6.2.

    Returns float64 ``[num_seqs, num_q_heads, head_dim]``; rows of requests not
    in ``seqs`` (when given) stay zero.
    """
    num_seqs, num_q_heads, _ = q.shape
    num_kv_heads = k_cache.shape[1]
    _check_heads(num_q_heads, num_kv_heads)
    out = np.zeros(q.shape, dtype=np.float64)
    for r in (range(num_seqs) if seqs is None else seqs):
        length = int(context_lens[r])
        keys = to_f64(gather_sequence(k_cache, block_tables[r], length, block_size), dtype)
        values = to_f64(gather_sequence(v_cache, block_tables[r], length, block_size), dtype)
        q_r = to_f64(q[r], dtype)
        for h in range(num_q_heads):
            g = kv_head_of(h, num_q_heads, num_kv_heads)
            out[r, h] = softmax_attention(q_r[h], keys[:, g, :], values[:, g, :], scale)
    return out


def paged_varlen(q, k_cache, v_cache, block_tables, query_start_loc, seq_lens, scale: float,
                 dtype: str, block_size: int = BLOCK_SIZE, seqs=None):
    """Attention for a scheduler batch that mixes decode rows and prefill chunks.

    ``q``: ``[total_q, num_q_heads, head_dim]``; request ``r`` owns query rows
    ``query_start_loc[r] .. query_start_loc[r+1]`` ([ARCH] §3.3.2 table:
    ``[0, L1, L1+L2, ...]`` for prefill, ``[0, 1, 2, ...]`` for decode).
    ``seq_lens[r]`` counts cached plus new tokens.  Query row ``i`` sits at
    position ``seq_len - q_len + i`` (:func:`query_positions`) and attends to
    keys ``0 .. position`` (causal reading: a token sees itself and every
    earlier token; the pages state no mask, only the positions).  A row with
    ``q_len == 1`` is a decode row ([ARCH] §3.2 "num_new_tokens == 1").
    """
    total_q, num_q_heads, _ = q.shape
    num_kv_heads = k_cache.shape[1]
    _check_heads(num_q_heads, num_kv_heads)
    num_seqs = len(seq_lens)
    out = np.zeros(q.shape, dtype=np.float64)
    for r in (range(num_seqs) if seqs is None else seqs):
        first, last = int(query_start_loc[r]), int(query_start_loc[r + 1])
        q_len, length = last - first, int(seq_lens[r])
        if q_len > length:
            raise ValueError(f"request {r}: {q_len} query rows but seq_len {length}")
        keys = to_f64(gather_sequence(k_cache, block_tables[r], length, block_size), dtype)
        values = to_f64(gather_sequence(v_cache, block_tables[r], length, block_size), dtype)
        for i, pos in enumerate(query_positions(length, q_len)):
            q_i = to_f64(q[first + i], dtype)
            visible = pos + 1
            for h in range(num_q_heads):
                g = kv_head_of(h, num_q_heads, num_kv_heads)
                out[first + i, h] = softmax_attention(
                    q_i[h], keys[:visible, g, :], values[:visible, g, :], scale)
    return out
