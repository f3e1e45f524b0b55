"""GPU parity of the FP8 (e4m3) KV cache against the oracle.

* pa_reshape_and_cache_fp8: the codes are bit-exact against
  ``oracle.reshape_and_cache_fp8`` -- random rows, rows that saturate, and rows
  placed exactly on the midpoints between two e4m3 values (round to even).
* pa_decode_fp8 / pa_varlen_fp8: within the attention tolerance of the
  oracle's attention over the dequantized cache, on every path (tensor-core
  MMA with f16 operands, CUDA cores), for GQA groups 1 to 8, head_dim 64,
  128 and 256, 8/16/32-token blocks, split-K rows and causal chunks.
"""

import numpy as np
import pytest
import torch

import oracle as O
import pagedattention_paged_kv_reshape_b200 as pa
from pagedattention_paged_kv_reshape_b200 import workload as W
from tests._helpers import assert_close, gpu_step, host, oracle_step

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _path_reset():
    prev = pa.pa_set_path(pa.Path.AUTO)
    yield
    pa.pa_set_path(prev)


@pytest.mark.parametrize("dtype,d,bs", [("bf16", 128, 16), ("f16", 64, 8), ("f32", 128, 32),
                                        ("bf16", 256, 16)])
def test_quantising_write_bit_exact(dtype, d, bs):
    b = W.build_batch([W.Request(L, q) for L, q in [(1, 1), (40, 7), (300, 300), (17, 1)]],
                      num_q_heads=4, num_kv_heads=4, head_dim=d, dtype=dtype, seed=5, device=DEV,
                      pool_factor=1.3, block_size=bs, kv_dtype="fp8")
    k_new = b.k_new.clone()
    k_new[3] *= 30.0                  # some x / scale beyond 448: saturate
    slots = b.slot_mapping.clone()
    slots[::6] = -1                   # padding tokens are skipped
    hs = b.host_slots.copy()
    hs[::6] = -1
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    pa.pa_reshape_and_cache_fp8(k_new, b.v_new, kc, vc, slots, b.k_scale, b.v_scale)
    pa.pa_get_device_error()
    ok, ov = O.reshape_and_cache_fp8(host(b.k_cache), host(b.v_cache), host(k_new),
                                     host(b.v_new), hs, host(b.k_scale), host(b.v_scale), dtype,
                                     block_size=bs)
    assert np.array_equal(host(kc), ok) and np.array_equal(host(vc), ov)


def test_quantising_write_rounds_midpoints_to_even():
    """Rows on the exact midpoints between adjacent e4m3 values (scale 0.5, a
    power of two, so x / scale is exact): every tie goes to the even code."""
    hkv, d = 2, 128
    codes = np.arange(0, 0x7E, dtype=np.uint8)        # 0 .. 446 (positive finite)
    vals = O.e4m3_decode(codes)
    mids = (vals[:-1] + vals[1:]) / 2                 # 125 midpoints, exact in bf16
    row = np.resize(np.concatenate([mids, -mids]), (hkv, d)).astype(np.float32)
    k = torch.from_numpy(np.stack([row * 0.5, row * 0.5 + 0.0])).to(torch.bfloat16).to(DEV)
    assert torch.equal(k.float().cpu(), torch.from_numpy(np.stack([row * 0.5] * 2)))
    kc = torch.full((4, hkv, 16, d), 0x7F, dtype=torch.uint8, device=DEV)
    vc = kc.clone()
    scale = torch.full((hkv,), 0.5, dtype=torch.float32, device=DEV)
    slots = torch.tensor([16 + 3, 2 * 16 + 9], dtype=torch.int32, device=DEV)
    pa.pa_reshape_and_cache_fp8(k, k, kc, vc, slots, scale, scale)
    pa.pa_get_device_error()
    ok, _ = O.reshape_and_cache_fp8(np.full((4, hkv, 16, d), 0x7F, np.uint8),
                                    np.full((4, hkv, 16, d), 0x7F, np.uint8), host(k), host(k),
                                    host(slots), np.full(hkv, 0.5, np.float32),
                                    np.full(hkv, 0.5, np.float32), "bf16")
    assert np.array_equal(host(kc), ok)
    got = host(kc)[1, :, 3, :]
    assert np.all(got[(got & 0x7F) != 0] & 1 == 0)   # ties landed on even mantissas


FP8_CASES = [
    # (rows (seq_len, q_len), hq, hkv, d, q dtype, block_size)
    ([(700, 37), (1, 1), (33, 1), (2000, 1), (1300, 300), (9, 9)], 32, 8, 128, "bf16", 16),
    ([(600, 600), (90, 5), (1100, 1)], 8, 8, 64, "f16", 8),
    ([(520, 20), (17, 17), (2, 1)], 4, 4, 64, "f32", 32),
    ([(2500, 256), (300, 1), (15, 1)], 16, 2, 128, "bf16", 32),
    ([(1000, 1), (4096, 1), (77, 1)], 32, 4, 128, "f16", 16),
    ([(700, 37), (1, 1), (2000, 1), (600, 160), (9, 9)], 16, 2, 256, "bf16", 16),  # head_dim 256
    ([(1300, 1), (33, 1), (4096, 1)], 8, 8, 256, "f32", 8),
    # decode at head_dim 128 on both sides of the transposed (<= 8 rows) form:
    # group 16 (16-row tiles), MHA with 8-token blocks, group 6 with 32-token
    # blocks, with split-K rows, one-token contexts and ragged last blocks
    ([(3000, 1), (17, 1), (513, 1), (1, 1)], 16, 1, 128, "bf16", 16),
    ([(2049, 1), (5, 1), (700, 1)], 8, 8, 128, "f16", 8),
    ([(1500, 1), (64, 1), (1, 1)], 24, 4, 128, "bf16", 32),
]


@pytest.mark.parametrize("path", ["auto", "mma", "simt"])
@pytest.mark.parametrize("case", range(len(FP8_CASES)))
def test_fp8_attention_matches_oracle(case, path):
    rows, hq, hkv, d, dtype, bs = FP8_CASES[case]
    if path == "simt":
        pa.pa_set_path(pa.Path.SIMT)
    elif path == "mma":
        if dtype == "f32":
            pytest.skip("tensor-core paths need 16-bit q")
        pa.pa_set_path(pa.Path.MMA)
    b = W.build_batch([W.Request(s, q) for s, q in rows], num_q_heads=hq, num_kv_heads=hkv,
                      head_dim=d, dtype=dtype, seed=500 + case, device=DEV, pool_factor=1.2,
                      block_size=bs, kv_dtype="fp8")
    varlen = any(q_ != 1 for _, q_ in rows)
    out, kc, vc = gpu_step(b, varlen=varlen)
    ref, okc, ovc = oracle_step(b, varlen=varlen)
    assert np.array_equal(host(kc), okc) and np.array_equal(host(vc), ovc)
    assert_close(out, ref, dtype, f"fp8 case {case} ({path})")
