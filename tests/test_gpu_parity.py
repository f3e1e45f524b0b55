"""GPU parity: the CUDA library against the fp64 oracle on the same seeded inputs.

Bars: cache writes bit-exact; attention within max-abs 1e-2 / mean-abs 1e-3
for bf16 and f16 inputs (fp32 accumulation) and 1e-5 for fp32 inputs.
Small cases span several 16-token blocks and 512-token partitions with ragged
tails; the full-size workloads are checked on every row in
test_gpu_full_size.py.  Every call goes through the C ABI.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
import pagedattention_paged_kv_reshape_b200 as pa
from pagedattention_paged_kv_reshape_b200 import workload as W
from tests._helpers import (assert_close, f64, gpu_attention, gpu_cache_write, gpu_step, host,
                            oracle_step)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _path_reset():
    prev = pa.pa_set_path(pa.Path.AUTO)
    yield
    pa.pa_set_path(prev)


def decode_batch(lengths, hq, hkv, d, dtype, seed=0, **kw):
    return W.build_batch([W.Request(L) for L in lengths], num_q_heads=hq, num_kv_heads=hkv,
                         head_dim=d, dtype=dtype, seed=seed, device=DEV, pool_factor=1.5, **kw)


# ---------------------------------------------------------------------------
# reshape_and_cache: bit-exact against the oracle's copy
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,d,bs", [("f32", 64, 16), ("bf16", 128, 16), ("f16", 64, 16),
                                        ("bf16", 64, 16), ("bf16", 128, 8), ("f32", 64, 32),
                                        ("bf16", 256, 16), ("f32", 256, 8)])
def test_reshape_and_cache_bit_exact(dtype, d, bs):
    b = W.build_batch([W.Request(L, q) for L, q in [(1, 1), (40, 7), (300, 300), (17, 1)]],
                      num_q_heads=4, num_kv_heads=4, head_dim=d, dtype=dtype, seed=3, device=DEV,
                      pool_factor=1.3, block_size=bs)
    slots = b.slot_mapping.clone()
    slots[::5] = -1                      # padding tokens are skipped
    hslots = b.host_slots.copy()
    hslots[::5] = -1
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    pa.pa_reshape_and_cache(b.k_new, b.v_new, kc, vc, slots)
    pa.pa_get_device_error()
    ok, ov = O.reshape_and_cache(host(b.k_cache), host(b.v_cache), host(b.k_new), host(b.v_new),
                                 hslots, block_size=bs)
    # byte-for-byte, NaN payloads included
    assert np.array_equal(host(kc).view(np.uint8), ok.view(np.uint8))
    assert np.array_equal(host(vc).view(np.uint8), ov.view(np.uint8))


def test_reshape_and_cache_bad_slot_is_reported_not_written():
    b = decode_batch([5, 9], 2, 2, 64, "bf16")
    slots = b.slot_mapping.clone()
    slots[1] = b.num_blocks * 16 + 3      # past the pool
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    pa.pa_reshape_and_cache(b.k_new, b.v_new, kc, vc, slots)
    with pytest.raises(pa.PaError) as e:
        pa.pa_get_device_error()
    assert e.value.status == pa.Status.DEVICE_BOUNDS
    hs = b.host_slots.copy()
    hs[1] = -1
    ok, _ = O.reshape_and_cache(host(b.k_cache), host(b.v_cache), host(b.k_new), host(b.v_new), hs)
    assert np.array_equal(host(kc).view(np.uint8), ok.view(np.uint8))
    pa.pa_get_device_error()              # the word was cleared


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

def test_tiny_config_fp32():
    b = W.make_config("tiny", seed=0, device=DEV)
    out, kc, vc = gpu_step(b)
    ref, okc, ovc = oracle_step(b)
    assert np.array_equal(host(kc).view(np.uint8), okc.view(np.uint8))
    assert_close(out, ref, "f32", "tiny")
    # context length 1 returns V exactly
    assert torch.equal(out[0], b.v_new[0].repeat_interleave(1, 0))


DECODE_CASES = [
    # lengths, hq, hkv, d, dtype
    ([1, 15, 16, 17, 513, 1100], 4, 4, 128, "bf16"),          # MHA, block and partition edges
    ([1, 2, 31, 512, 1024, 1537, 3000], 32, 8, 128, "bf16"),  # GQA 4
    ([4999, 700, 33], 16, 2, 128, "bf16"),                    # GQA 8, long
    ([129, 1030, 7], 32, 2, 64, "f16"),                       # GQA 16, head_dim 64
    ([600, 45], 64, 2, 64, "bf16"),                           # group 32: two 16-head slices
    ([800, 20, 1], 6, 2, 128, "f16"),                         # group 3
    ([1, 77, 2048], 8, 8, 64, "f32"),                         # fp32, head_dim 64
    ([300, 1500], 8, 4, 128, "f32"),                          # fp32, head_dim 128, GQA 2
]


@pytest.mark.parametrize("path", ["auto", "simt"])
@pytest.mark.parametrize("case", range(len(DECODE_CASES)))
def test_decode_matches_oracle(case, path):
    lengths, hq, hkv, d, dtype = DECODE_CASES[case]
    if path == "simt":
        pa.pa_set_path(pa.Path.SIMT)
    b = decode_batch(lengths, hq, hkv, d, dtype, seed=case)
    out, _, _ = gpu_step(b)
    ref, _, _ = oracle_step(b)
    assert_close(out, ref, dtype, f"decode case {case} ({path})")


def test_mma_path_forced_matches_auto():
    b = decode_batch([1, 100, 700], 32, 8, 128, "bf16", seed=11)
    kc, vc = gpu_cache_write(b)
    auto = gpu_attention(b, kc, vc)
    pa.pa_set_path(pa.Path.MMA)
    forced = gpu_attention(b, kc, vc)
    assert torch.equal(auto, forced)


def test_decode_empty_context_is_zero_row():
    b = decode_batch([40, 3], 8, 2, 128, "bf16", seed=5)
    kc, vc = gpu_cache_write(b)
    lens = b.seq_lens.clone()
    lens[1] = 0
    out = torch.full_like(b.q, float("nan"))
    ws = pa.alloc_workspace(pa.pa_decode_workspace_size(2, 8, 2, 128, 40), DEV)
    pa.pa_decode(out, b.q, kc, vc, b.block_tables, lens, 40, b.scale, ws)
    pa.pa_get_device_error()
    assert torch.all(out[1] == 0)
    assert torch.all(torch.isfinite(out[0]))


# ---------------------------------------------------------------------------
# varlen: decode rows next to causal prefill chunks
# ---------------------------------------------------------------------------

VARLEN_CASES = [
    # (seq_len, q_len) rows, hq, hkv, d, dtype.  With the default path, rows of
    # at least 128 / min(group, 16) new tokens run on the tcgen05 chunk kernel.
    ([(700, 37), (1, 1), (33, 1), (64, 64), (2000, 1), (530, 0), (1300, 300)], 32, 8, 128, "bf16"),
    ([(1, 1), (600, 600), (90, 5)], 8, 8, 64, "f16"),
    ([(2048, 512), (100, 1), (4096, 1)], 16, 2, 128, "bf16"),
    ([(45, 45), (1100, 13), (3, 1)], 6, 2, 128, "bf16"),          # group 3: no tcgen05 tiles
    ([(520, 20), (17, 17), (2, 1)], 4, 4, 64, "f32"),
    ([(300, 40), (1000, 129), (200, 200), (5, 1)], 32, 8, 64, "bf16"),  # ragged chunk tiles
    ([(1000, 129), (129, 129), (77, 1)], 4, 4, 128, "f16"),        # MHA: 128-token tiles
    ([(600, 70), (64, 1), (900, 9)], 64, 2, 128, "bf16"),          # group 32: 16-head slices
    ([(2500, 256), (300, 1)], 16, 2, 64, "f16"),                   # group 8, head_dim 64
]


@pytest.mark.parametrize("path", ["auto", "mma", "simt"])
@pytest.mark.parametrize("case", range(len(VARLEN_CASES)))
def test_varlen_matches_oracle(case, path):
    rows, hq, hkv, d, dtype = VARLEN_CASES[case]
    if path == "simt":
        pa.pa_set_path(pa.Path.SIMT)
    elif path == "mma":
        if dtype == "f32":
            pytest.skip("tensor-core paths need 16-bit inputs")
        pa.pa_set_path(pa.Path.MMA)
    b = W.build_batch([W.Request(s, q) for s, q in rows], num_q_heads=hq, num_kv_heads=hkv,
                      head_dim=d, dtype=dtype, seed=100 + case, device=DEV, pool_factor=1.2)
    out, _, _ = gpu_step(b, varlen=True)
    ref, _, _ = oracle_step(b, varlen=True)
    assert_close(out, ref, dtype, f"varlen case {case} ({path})")


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("scale", [1.0, -0.3, 0.0])
def test_varlen_other_scales(scale, d):
    """Scales other than 1/sqrt(head_dim).  With 1.0 the scores of N(0,1) data
    have a standard deviation of about 11, so a row's running maximum climbs by
    many powers of two across the context and the chunk kernel has to move the
    reference point of its TMEM accumulator several times; a negative scale
    reverses the order of the scores; zero is the plain mean of the visible
    values.  f16, so that the near one-hot outputs of the large scale (|o| up to
    about 5) still round to within the 1e-2 bound."""
    rows = [(1500, 300), (700, 129), (40, 1), (900, 1)]
    b = W.build_batch([W.Request(s, q) for s, q in rows], num_q_heads=32, num_kv_heads=8,
                      head_dim=d, dtype="f16", seed=55, device=DEV, pool_factor=1.2)
    b.scale = scale
    out, _, _ = gpu_step(b, varlen=True)
    ref, _, _ = oracle_step(b, varlen=True)
    assert_close(out, ref, "f16", f"varlen scale {scale} head_dim {d}")


BLOCK_SIZE_CASES = [
    # (rows (seq_len, q_len), hq, hkv, d, dtype, block_size): 8- and 32-token
    # blocks through decode rows, split-K rows and tcgen05 chunk rows
    ([(700, 37), (1, 1), (33, 1), (2000, 1), (1300, 300), (9, 9)], 32, 8, 128, "bf16", 8),
    ([(700, 37), (1, 1), (33, 1), (2000, 1), (1300, 300), (9, 9)], 32, 8, 128, "bf16", 32),
    ([(600, 600), (90, 5), (1100, 1)], 8, 8, 64, "f16", 8),
    ([(520, 20), (17, 17), (2, 1)], 4, 4, 64, "f32", 32),
    ([(2500, 256), (300, 1), (15, 1)], 16, 2, 64, "f16", 32),
]


@pytest.mark.parametrize("path", ["auto", "mma", "simt"])
@pytest.mark.parametrize("case", range(len(BLOCK_SIZE_CASES)))
def test_block_sizes_match_oracle(case, path):
    rows, hq, hkv, d, dtype, bs = BLOCK_SIZE_CASES[case]
    if path == "simt":
        pa.pa_set_path(pa.Path.SIMT)
    elif path == "mma":
        if dtype == "f32":
            pytest.skip("tensor-core paths need 16-bit inputs")
        pa.pa_set_path(pa.Path.MMA)
    b = W.build_batch([W.Request(s, q) for s, q in rows], num_q_heads=hq, num_kv_heads=hkv,
                      head_dim=d, dtype=dtype, seed=300 + case, device=DEV, pool_factor=1.2,
                      block_size=bs)
    out, kc, vc = gpu_step(b, varlen=True)
    ref, okc, ovc = oracle_step(b, varlen=True)
    assert np.array_equal(host(kc).view(np.uint8), okc.view(np.uint8))
    assert_close(out, ref, dtype, f"block_size {bs} case {case} ({path})")
    dec = [r for r, (s_, q_) in enumerate(rows) if q_ == 1]
    if dec:  # the decode entry point on the same cache, for rows of one new token
        bd = W.build_batch([W.Request(rows[r][0]) for r in dec], num_q_heads=hq,
                           num_kv_heads=hkv, head_dim=d, dtype=dtype, seed=400 + case,
                           device=DEV, pool_factor=1.2, block_size=bs)
        out_d, _, _ = gpu_step(bd, varlen=False)
        ref_d, _, _ = oracle_step(bd, varlen=False)
        assert_close(out_d, ref_d, dtype, f"decode block_size {bs} case {case} ({path})")


HEAD_DIM_256_CASES = [
    # head_dim 256: the tensor-core decode/varlen kernel for 16-bit types, the
    # one-tile tcgen05 chunk kernel for rows of >= 128/gs new tokens, the
    # CUDA-core kernel for fp32 and when it is forced
    ([(700, 37), (1, 1), (2000, 1), (600, 160), (9, 9)], 16, 2, "bf16"),    # group 8
    ([(1300, 1), (33, 1), (4096, 1)], 8, 8, "f16"),                          # MHA, split-K
    ([(520, 20), (17, 17), (1025, 1)], 32, 8, "bf16"),                      # group 4
    ([(700, 1), (40, 9), (1537, 1)], 8, 2, "f32"),                           # fp32
    # chunk rows of several 64-key tiles with ragged last query tiles
    ([(900, 300), (5, 1), (2100, 777), (64, 64)], 32, 8, "bf16"),          # group 4
    ([(640, 200), (130, 130), (3000, 1)], 4, 4, "f16"),                     # MHA: 128-token tiles
    ([(1000, 64), (700, 300), (8, 8)], 16, 1, "bf16"),                      # group 16: 8-token tiles
]


@pytest.mark.parametrize("path", ["auto", "simt"])
@pytest.mark.parametrize("case", range(len(HEAD_DIM_256_CASES)))
def test_head_dim_256_matches_oracle(case, path):
    rows, hq, hkv, dtype = HEAD_DIM_256_CASES[case]
    if path == "simt":
        pa.pa_set_path(pa.Path.SIMT)
    b = W.build_batch([W.Request(s, q) for s, q in rows], num_q_heads=hq, num_kv_heads=hkv,
                      head_dim=256, dtype=dtype, seed=700 + case, device=DEV, pool_factor=1.2)
    varlen = any(q_ != 1 for _, q_ in rows)
    out, kc, vc = gpu_step(b, varlen=varlen)
    ref, okc, _ = oracle_step(b, varlen=varlen)
    assert np.array_equal(host(kc).view(np.uint8), okc.view(np.uint8))
    assert_close(out, ref, dtype, f"head_dim 256 case {case} ({path})")


# Batches whose longest row has 16 or more 512-key partitions take the wide
# split-K reduce (one CTA per query head, warps splitting the partitions);
# short rows of the same batch go through it too.
WIDE_REDUCE_CASES = [
    # (rows (seq_len, q_len), hq, hkv, d, dtype, kv cache dtype, path)
    ([(9000, 1), (17, 1), (8200, 1), (600, 1), (16385, 1)], 8, 2, 128, "bf16", None, "auto"),
    ([(8193, 1), (3, 1), (12000, 1)], 4, 4, 64, "f32", None, "simt"),
    ([(9100, 1), (530, 1)], 8, 4, 256, "bf16", None, "auto"),
    ([(9000, 37), (1, 1), (8300, 1), (700, 200)], 8, 2, 128, "f16", None, "mma"),
    ([(10000, 1), (45, 1), (8500, 9)], 16, 2, 128, "bf16", "fp8", "auto"),
]


@pytest.mark.parametrize("case", range(len(WIDE_REDUCE_CASES)))
def test_wide_split_k_reduce_matches_oracle(case):
    rows, hq, hkv, d, dtype, kv_dtype, path = WIDE_REDUCE_CASES[case]
    if path == "simt":
        pa.pa_set_path(pa.Path.SIMT)
    elif path == "mma":
        pa.pa_set_path(pa.Path.MMA)
    extra = {"kv_dtype": kv_dtype} if kv_dtype else {}
    b = W.build_batch([W.Request(L, q) for L, q in rows], num_q_heads=hq, num_kv_heads=hkv,
                      head_dim=d, dtype=dtype, seed=900 + case, device=DEV, pool_factor=1.2,
                      **extra)
    assert math.ceil(b.max_seq_len / 512) >= 16
    varlen = any(q_ != 1 for _, q_ in rows)
    out, _, _ = gpu_step(b, varlen=varlen)
    ref, _, _ = oracle_step(b, varlen=varlen)
    assert_close(out, ref, dtype, f"wide reduce case {case} ({path})")


@pytest.mark.parametrize("bs", [8, 32])
def test_head_dim_256_chunk_block_sizes(bs):
    """The head_dim-256 chunk kernel's K/V boxes for 8-token blocks (one box
    per block) and 32-token blocks (two boxes per block)."""
    rows = [(1300, 300), (700, 37), (33, 1), (200, 129)]
    b = W.build_batch([W.Request(s, q) for s, q in rows], num_q_heads=16, num_kv_heads=4,
                      head_dim=256, dtype="bf16", seed=1200 + bs, device=DEV, pool_factor=1.2,
                      block_size=bs)
    out, _, _ = gpu_step(b, varlen=True)
    ref, _, _ = oracle_step(b, varlen=True)
    assert_close(out, ref, "bf16", f"head_dim 256 chunk, block_size {bs}")


@pytest.mark.parametrize("d", [128, 256])
def test_chunk_kernel_agrees_with_decode_kernel_tiles(d):
    """The tcgen05 chunk tiles and the decode kernel's 16-row tiles compute the
    same rows; both are within tolerance of each other as well as the oracle."""
    b = W.build_batch([W.Request(s, q) for s, q in [(1536 + 512, 512), (800, 1)]],
                      num_q_heads=32, num_kv_heads=8, head_dim=d, dtype="bf16", seed=7,
                      device=DEV, pool_factor=1.1)
    kc, vc = gpu_cache_write(b)
    tc = gpu_attention(b, kc, vc, varlen=True)
    pa.pa_set_path(pa.Path.MMA)
    mma = gpu_attention(b, kc, vc, varlen=True)
    assert_close(tc, f64(mma), "bf16", "tcgen05 vs mma tiles")
    assert torch.equal(tc[-1], mma[-1])   # the decode row takes the same kernel on both


def test_varlen_decode_rows_equal_decode():
    b = decode_batch([3, 600, 1200, 17], 32, 8, 128, "bf16", seed=21)
    kc, vc = gpu_cache_write(b)
    dec = gpu_attention(b, kc, vc, varlen=False)
    var = gpu_attention(b, kc, vc, varlen=True)
    assert torch.equal(dec, var)


# ---------------------------------------------------------------------------
# invariants the pages fix, on the GPU (bitwise)
# ---------------------------------------------------------------------------

def test_permutation_of_physical_ids_is_invisible():
    b = decode_batch([5, 333, 1700, 64], 32, 8, 128, "bf16", seed=31)
    kc, vc = gpu_cache_write(b)
    base = gpu_attention(b, kc, vc)
    g = torch.Generator().manual_seed(7)
    sigma = torch.randperm(b.num_blocks, generator=g).to(DEV)     # block b -> sigma[b]
    kc2, vc2 = torch.empty_like(kc), torch.empty_like(vc)
    kc2[sigma], vc2[sigma] = kc, vc
    tables = sigma[b.block_tables.long()].int()
    out = torch.full_like(b.q, float("nan"))
    ws = pa.alloc_workspace(pa.pa_decode_workspace_size(b.num_seqs, 32, 8, 128, b.max_seq_len), DEV)
    pa.pa_decode(out, b.q, kc2, vc2, tables, b.seq_lens, b.max_seq_len, b.scale, ws)
    pa.pa_get_device_error()
    assert torch.equal(out, base)


def test_shared_prefix_equals_private_copies():
    reqs = [W.Request(L, 1, True) for L in (600, 1100, 513)] + [W.Request(800)]
    b = W.build_batch(reqs, num_q_heads=32, num_kv_heads=8, head_dim=128, dtype="bf16", seed=41,
                      device=DEV, pool_factor=2.0, shared_prefix_len=512)
    kc, vc = gpu_cache_write(b)
    shared = gpu_attention(b, kc, vc)
    # give request 1 private copies of the 32 shared blocks, in unused pool blocks
    used = set(b.host_tables[:, :].ravel().tolist())
    free = [i for i in range(b.num_blocks) if i not in used][:32]
    assert len(free) == 32
    tables = b.block_tables.clone()
    src = torch.tensor(b.shared_blocks, device=DEV)
    dst = torch.tensor(free, device=DEV)
    kc[dst], vc[dst] = kc[src], vc[src]
    tables[1, :32] = dst.int()
    out = torch.full_like(b.q, float("nan"))
    ws = pa.alloc_workspace(pa.pa_decode_workspace_size(b.num_seqs, 32, 8, 128, b.max_seq_len), DEV)
    pa.pa_decode(out, b.q, kc, vc, tables, b.seq_lens, b.max_seq_len, b.scale, ws)
    pa.pa_get_device_error()
    assert torch.equal(out, shared)


def test_equal_values_give_that_row():
    b = decode_batch([1000, 37], 16, 4, 128, "bf16", seed=51, poison=False)
    row = torch.randn(4, 128, device=DEV).to(torch.bfloat16)
    b.v_cache[:] = row[None, :, None, :]
    b.v_new[:] = row[None]
    out, _, _ = gpu_step(b)
    want = row.float().repeat_interleave(4, 0)
    assert torch.allclose(out.float(), want[None].expand_as(out), atol=8e-3, rtol=0)


# ---------------------------------------------------------------------------
# device-side metadata checks: reported, never a fault
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", ["auto", "simt"])
def test_out_of_range_block_id_is_reported(path):
    if path == "simt":
        pa.pa_set_path(pa.Path.SIMT)
    b = decode_batch([100, 40], 8, 2, 128, "bf16", seed=61)
    kc, vc = gpu_cache_write(b)
    tables = b.block_tables.clone()
    tables[0, 2] = b.num_blocks + 5
    out = torch.zeros_like(b.q)
    ws = pa.alloc_workspace(pa.pa_decode_workspace_size(2, 8, 2, 128, 100), DEV)
    pa.pa_decode(out, b.q, kc, vc, tables, b.seq_lens, b.max_seq_len, b.scale, ws)
    with pytest.raises(pa.PaError) as e:
        pa.pa_get_device_error()
    assert e.value.status == pa.Status.DEVICE_BOUNDS
    # the other request is unaffected
    ref, _, _ = oracle_step(b)
    assert_close(out[1:], ref[1:], "bf16", "untouched request")


def test_context_len_above_host_bound_is_reported():
    b = decode_batch([100, 40], 8, 2, 128, "bf16", seed=62)
    kc, vc = gpu_cache_write(b)
    out = torch.zeros_like(b.q)
    ws = pa.alloc_workspace(pa.pa_decode_workspace_size(2, 8, 2, 128, 64), DEV)
    pa.pa_decode(out, b.q, kc, vc, b.block_tables, b.seq_lens, 64, b.scale, ws)
    with pytest.raises(pa.PaError) as e:
        pa.pa_get_device_error()
    assert e.value.status == pa.Status.DEVICE_BOUNDS
