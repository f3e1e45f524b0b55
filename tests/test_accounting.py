"""Byte/FLOP accounting used by the roofline, pinned to the pages' printed numbers."""

import json
import os

from pagedattention_paged_kv_reshape_b200 import accounting as A
from pagedattention_paged_kv_reshape_b200 import workload as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "block_bytes.json")


def test_block_bytes_match_the_pages():
    g = json.load(open(GOLDEN))
    blk = g["block_structure"]
    per_block = A.kv_bytes_per_block(blk["block_size"], blk["num_layers"], blk["num_kv_heads"],
                                     blk["head_dim"], blk["elem_bytes"])
    assert per_block == blk["per_block_bytes"]
    n = A.blocks_that_fit(blk["cache_gib"] * 2 ** 30, per_block)
    assert n == blk["num_blocks"]
    assert n * blk["block_size"] == blk["max_tokens"]
    pre = g["static_prealloc"]
    k_only = pre["max_seq_len"] * A.kv_bytes_per_token(pre["num_heads"], pre["head_dim"],
                                                       pre["elem_bytes"], kv=1)
    assert k_only == pre["bytes"]


def test_attention_bytes_count_shared_prefix_once():
    reqs = [W.Request(600, 1, True), W.Request(700, 1, True), W.Request(100)]
    b = W.build_batch(reqs, num_q_heads=8, num_kv_heads=2, head_dim=64, dtype="bf16", seed=0,
                      shared_prefix_len=512, pool_factor=1.0)
    per_tok = 2 * 2 * 64 * 2
    acc = A.attention_bytes(b)
    assert acc["kv_logical"] == (600 + 700 + 100) * per_tok
    assert acc["kv_unique"] == acc["kv_logical"] - 512 * per_tok
    assert acc["q_out"] == 2 * 3 * 8 * 64 * 2
    assert acc["tables"] == 4 * (38 + 44 + 7)


def test_chunk_flops():
    b = W.build_batch([W.Request(10, 4), W.Request(5, 1)], num_q_heads=2, num_kv_heads=1,
                      head_dim=64, dtype="bf16", seed=0)
    # positions 6..9 see 7+8+9+10 keys
    assert A.chunk_flops(b) == 4 * 64 * 2 * (7 + 8 + 9 + 10)
