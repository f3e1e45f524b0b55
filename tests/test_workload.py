"""The seeded workload recipes, CPU only: each named configuration's request
generator and shape spec match the recipe it states (lengths, head counts,
the mixed batch's sharing structure and token budget), draws are reproducible
from the seed, and a small batch is laid out as documented (a shuffled pool,
padding poisoned, new tokens' slots past each request's cached keys).  The
full-size pools are not built here (the mixed batch's alone is 11.5 GB)."""

import math

import numpy as np
import pytest
import torch

from pagedattention_paged_kv_reshape_b200 import workload as W


def reqs(name, seed=0):
    return W.CONFIGS[name]["requests"](seed)


def test_tiny():
    r = reqs("tiny")
    assert [x.seq_len for x in r] == [1, 17, 33, 100] and all(x.q_len == 1 for x in r)
    spec = W.CONFIGS["tiny"]
    assert (spec["num_q_heads"], spec["num_kv_heads"], spec["head_dim"], spec["dtype"]) == \
        (4, 4, 64, "f32") and spec["pool_blocks"] == 64


def test_mha_bs64():
    r = reqs("mha_bs64")
    lens = np.array([x.seq_len for x in r])
    assert len(r) == 64 and all(x.q_len == 1 for x in r)
    assert lens.min() >= 256 and lens.max() <= 2048
    spec = W.CONFIGS["mha_bs64"]
    assert (spec["num_q_heads"], spec["num_kv_heads"], spec["head_dim"], spec["dtype"]) == \
        (32, 32, 128, "bf16") and spec["pool_factor"] == 1.25


def test_gqa_bs256_is_log_uniform():
    lens = np.array([x.seq_len for x in reqs("gqa_bs256")])
    assert len(lens) == 256 and lens.min() >= 128 and lens.max() <= 8192
    # log-uniform on [128, 8192]: the log-lengths spread evenly, median near 1024
    logs = np.log(lens)
    assert abs(np.median(lens) / 1024 - 1) < 0.35
    lo, hi = math.log(128), math.log(8192)
    hist, _ = np.histogram(logs, bins=4, range=(lo, hi))
    assert hist.min() >= 40  # 64 expected per quarter
    spec = W.CONFIGS["gqa_bs256"]
    assert (spec["num_q_heads"], spec["num_kv_heads"], spec["head_dim"]) == (32, 8, 128)


def test_long_32k():
    r = reqs("long_32k")
    assert [x.seq_len for x in r] == [32768] * 8 and all(x.q_len == 1 for x in r)
    spec = W.CONFIGS["long_32k"]
    assert (spec["num_q_heads"], spec["num_kv_heads"]) == (64, 8)


def test_mixed_2048_budget_and_sharing():
    r = reqs("mixed_2048")
    spec = W.CONFIGS["mixed_2048"]
    assert spec["shared_prefix_len"] == 512
    chunk = [x for x in r if x.q_len > 1]
    decode = [x for x in r if x.q_len == 1]
    assert len(chunk) == 1 and (chunk[0].seq_len, chunk[0].q_len) == (2048, 512)
    assert r[-1] is chunk[0]                     # the chunk row comes last
    assert len(decode) == 1536
    assert sum(x.q_len for x in r) == 2048       # the scheduler's token budget
    sharing = [x for x in decode if x.shares_prefix]
    private = [x for x in decode if not x.shares_prefix]
    assert len(sharing) == 768
    # sharing rows' new token lands past the 512-token shared run
    assert min(x.seq_len for x in sharing) >= 513 and max(x.seq_len for x in sharing) <= 4096
    assert min(x.seq_len for x in private) >= 64 and max(x.seq_len for x in private) <= 4096


def test_prefill_and_variants():
    r = reqs("prefill_16x512")
    assert [(x.seq_len, x.q_len) for x in r] == [(2048, 512)] * 16
    assert W.CONFIGS["gqa_bs256_b8"]["block_size"] == 8
    assert W.CONFIGS["gqa_bs256_b32"]["block_size"] == 32
    assert W.CONFIGS["gqa_bs256_fp8"]["kv_dtype"] == "fp8"
    d = W.CONFIGS["gqa_bs256_d256"]
    g = W.CONFIGS["gqa_bs256"]
    # the same KV bytes per token as gqa_bs256
    assert d["num_kv_heads"] * d["head_dim"] == g["num_kv_heads"] * g["head_dim"]
    # every variant draws gqa_bs256's lengths
    base = [x.seq_len for x in reqs("gqa_bs256")]
    for name in ("gqa_bs256_b8", "gqa_bs256_b32", "gqa_bs256_fp8", "gqa_bs256_d256"):
        assert [x.seq_len for x in reqs(name)] == base
    # prefill at head_dim 256: prefill_16x512's rows, the same KV bytes per token
    p = W.CONFIGS["prefill_16x512_d256"]
    q = W.CONFIGS["prefill_16x512"]
    assert p["head_dim"] == 256 and p["kind"] == "varlen"
    assert p["num_kv_heads"] * p["head_dim"] == q["num_kv_heads"] * q["head_dim"]
    assert [(x.seq_len, x.q_len) for x in reqs("prefill_16x512_d256")] == [(2048, 512)] * 16


@pytest.mark.parametrize("name", ["mha_bs64", "gqa_bs256", "mixed_2048"])
def test_draws_follow_the_seed(name):
    a, b, c = reqs(name, 0), reqs(name, 0), reqs(name, 1)
    key = lambda rs: [(x.seq_len, x.q_len, x.shares_prefix) for x in rs]  # noqa: E731
    assert key(a) == key(b) and key(a) != key(c)


def test_small_batch_layout():
    """Shuffled pool, sharing rows map to the same leading blocks, every slot
    no query may read holds NaN, and the new tokens' slots lie in the right
    blocks at the right offsets."""
    rq = [W.Request(600, 1, True), W.Request(40, 7), W.Request(700, 1, True), W.Request(5, 1)]
    b = W.build_batch(rq, num_q_heads=4, num_kv_heads=2, head_dim=64, dtype="f32", seed=3,
                      shared_prefix_len=512, pool_factor=1.3)
    bs = b.block_size
    tables = b.host_tables
    # the shared 512-token run: the same 32 leading blocks for both sharing rows
    assert np.array_equal(tables[0, :512 // bs], tables[2, :512 // bs])
    used = set()
    for r, x in enumerate(rq):
        own = tables[r, :math.ceil(x.seq_len / bs)]
        if not x.shares_prefix:
            assert not (set(own.tolist()) & used)   # private blocks are private
        used |= set(own.tolist())
    # the pool is shuffled: the used ids are not simply 0, 1, 2, ...
    assert sorted(used) != list(range(len(used)))
    # each new token's slot is at (table[pos // bs], pos % bs) of its position
    slots = b.host_slots
    qsl = b.host_qsl
    for r, x in enumerate(rq):
        for i in range(x.q_len):
            pos = x.seq_len - x.q_len + i
            assert slots[qsl[r] + i] == tables[r, pos // bs] * bs + pos % bs
    # before the write, the new tokens' slots and every padding slot hold NaN
    kc = b.k_cache.numpy()
    for r, x in enumerate(rq):
        for pos in range(x.seq_len - x.q_len, math.ceil(x.seq_len / bs) * bs):
            blk, off = tables[r, pos // bs], pos % bs
            assert np.isnan(kc[blk, :, off, :]).all()
        for pos in range(0, x.seq_len - x.q_len):
            blk, off = tables[r, pos // bs], pos % bs
            assert np.isfinite(kc[blk, :, off, :]).all()
    assert torch.isfinite(b.q).all()
