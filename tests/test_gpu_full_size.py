"""Every benchmarked workload at its full size, every output row against the oracle.

Each named workload the benchmark times (the five decode/mixed shapes of the
pages' serving engine plus the prefill, block-size, FP8 and head_dim-256
variants) is built at the size the benchmark uses, run through the C ABI
(cache write, then pa_decode or pa_varlen), and compared with the fp64 oracle
on every element of every output row: max-abs 1e-2 and mean-abs 1e-3 for the
16-bit inputs.  The oracle runs on all host cores (``oracle.parallel``: the
plain oracle functions on each (request, KV head) sub-problem).  The cache
write is checked bit for bit: every new row lands in its slot (its e4m3 code,
as the oracle encodes it, for an FP8 cache) and every other slot of the pool
is unchanged.

A second group repeats full-size calls many times and requires bitwise equal
outputs: the work is claimed dynamically by whichever CTA is free, but each
output depends only on its own inputs, so any difference would be a race.
"""

import numpy as np
import pytest
import torch

import oracle as O
import pagedattention_paged_kv_reshape_b200 as pa
from pagedattention_paged_kv_reshape_b200 import workload as W
from tests._helpers import assert_close, gpu_attention, gpu_cache_write, host, oracle_full

pytestmark = pytest.mark.gpu
DEV = "cuda"

FULL_SIZE = ["mha_bs64", "gqa_bs256", "long_32k", "mixed_2048", "prefill_16x512",
             "gqa_bs256_b8", "gqa_bs256_b32", "gqa_bs256_fp8", "gqa_bs256_d256",
             "prefill_16x512_d256"]


def check_cache_write(b, kc, vc):
    """Bitwise: the written slots hold the new rows (FP8: the oracle's codes of
    them), every other slot equals the pool before the write."""
    bs = b.block_size
    slots = b.slot_mapping.long()
    blk, off = slots // bs, slots % bs
    if b.fp8:
        n = b.total_q
        # the oracle's quantising write into a scratch pool of one block per token
        zeros = np.zeros((n, b.num_kv_heads, bs, b.head_dim), np.uint8)
        ok, ov = O.reshape_and_cache_fp8(zeros, zeros, host(b.k_new), host(b.v_new),
                                         np.arange(n, dtype=np.int32) * bs, host(b.k_scale),
                                         host(b.v_scale), b.dtype, block_size=bs)
        want_k = torch.from_numpy(ok[:, :, 0, :]).to(DEV)
        want_v = torch.from_numpy(ov[:, :, 0, :]).to(DEV)
        assert torch.equal(kc[blk, :, off, :], want_k)
        assert torch.equal(vc[blk, :, off, :], want_v)
        bits = lambda t: t                                        # noqa: E731
    else:
        bits = lambda t: t.view(torch.int16)                      # noqa: E731
        assert torch.equal(bits(kc[blk, :, off, :]), bits(b.k_new))
        assert torch.equal(bits(vc[blk, :, off, :]), bits(b.v_new))
    untouched = torch.ones(b.num_blocks, bs, dtype=torch.bool, device=DEV)
    untouched[blk, off] = False
    for new, old in ((kc, b.k_cache), (vc, b.v_cache)):
        a, o = bits(new).permute(0, 2, 1, 3), bits(old).permute(0, 2, 1, 3)
        assert torch.equal(a[untouched], o[untouched])


@pytest.mark.parametrize("name", FULL_SIZE)
def test_full_size_every_row_matches_oracle(name):
    b = W.make_config(name, seed=0, device=DEV)
    kc, vc = gpu_cache_write(b)
    out = gpu_attention(b, kc, vc)
    check_cache_write(b, kc, vc)
    del kc, vc
    torch.cuda.empty_cache()
    ref = oracle_full(b)
    assert ref.shape == tuple(out.shape)
    assert_close(out, ref, b.dtype, f"{name} (all {b.total_q} x {b.num_q_heads} rows)")


@pytest.mark.parametrize("name,repeats", [("gqa_bs256", 200), ("gqa_bs256_fp8", 200),
                                          ("mixed_2048", 40), ("prefill_16x512", 100),
                                          ("prefill_16x512_d256", 40)])
def test_repeated_full_size_calls_are_bitwise_identical(name, repeats):
    """The same call repeated back to back on one stream and one workspace
    (each call's kernels overlap the previous call's tail through
    programmatic dependent launch), four output buffers in turn."""
    b = W.make_config(name, seed=0, device=DEV)
    kc, vc = gpu_cache_write(b)
    first = gpu_attention(b, kc, vc)
    assert torch.all(torch.isfinite(first))
    if b.is_decode:
        ws = pa.alloc_workspace(pa.pa_decode_workspace_size(
            b.num_seqs, b.num_q_heads, b.num_kv_heads, b.head_dim, b.max_seq_len), DEV)
    else:
        ws = pa.alloc_workspace(pa.pa_varlen_workspace_size(
            b.num_seqs, b.total_q, b.num_q_heads, b.num_kv_heads, b.head_dim, b.max_query_len,
            b.max_seq_len), DEV)
    outs = [torch.full_like(first, float("nan")) for _ in range(4)]
    for i in range(repeats):
        o = outs[i % 4]
        if not b.is_decode:
            pa.pa_varlen(o, b.q, kc, vc, b.block_tables, b.query_start_loc, b.seq_lens,
                         b.max_query_len, b.max_seq_len, b.scale, ws)
        elif b.fp8:
            pa.pa_decode_fp8(o, b.q, kc, vc, b.k_scale, b.v_scale, b.block_tables, b.seq_lens,
                             b.max_seq_len, b.scale, ws)
        else:
            pa.pa_decode(o, b.q, kc, vc, b.block_tables, b.seq_lens, b.max_seq_len, b.scale, ws)
        if i % 4 == 3 or i == repeats - 1:
            pa.pa_get_device_error()
            for j in range(i % 4 + 1):
                assert torch.equal(outs[j].view(torch.int16), first.view(torch.int16)), \
                    f"{name}: call {i - (i % 4) + j} differs from the first"
                outs[j].fill_(float("nan"))
