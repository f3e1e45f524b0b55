"""GPU parity of the block operations against the oracle: bit-exact.

pa_copy_blocks (copy-on-write inside one pool) and pa_swap_blocks (device
pool <-> page-locked host pool) through the C ABI, compared byte for byte
with ``oracle.copy_blocks`` / ``oracle.swap_blocks`` on host copies of the
same pools; plus the copy-on-write fork of "vLLM 架构源码解析" §4.3.2 end to
end (copy, write the new token into the private copy, decode) against the
oracle within the attention tolerance.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import pagedattention_paged_kv_reshape_b200 as pa
from tests._helpers import assert_close, host

pytestmark = pytest.mark.gpu
DEV = "cuda"
TDT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def pool(nb, hkv, d, dtype, seed, device=DEV):
    g = torch.Generator(device="cpu").manual_seed(seed)
    k = torch.randn(nb, hkv, 16, d, generator=g).to(TDT[dtype])
    v = torch.randn(nb, hkv, 16, d, generator=g).to(TDT[dtype])
    return k.to(device), v.to(device)


def independent_pairs(rng, nb, n):
    ids = rng.permutation(nb)[:2 * n + 1]
    m = np.stack([ids[:n], ids[n:2 * n]], axis=1)
    m = np.concatenate([m, [[ids[2 * n], ids[2 * n]]]])  # src == dst: a no-op
    return m.astype(np.int32)


@pytest.mark.parametrize("dtype,d,hkv,n", [("bf16", 128, 8, 20), ("f32", 64, 4, 7),
                                           ("f16", 128, 2, 1), ("bf16", 64, 32, 300)])
def test_copy_blocks_bit_exact(dtype, d, hkv, n):
    nb = max(64, 2 * n + 8)
    k, v = pool(nb, hkv, d, dtype, seed=n)
    m = independent_pairs(np.random.default_rng(n), nb, n)
    want_k, want_v = O.copy_blocks(host(k), host(v), m)
    pa.pa_copy_blocks(k, v, torch.from_numpy(m).to(DEV))
    pa.pa_get_device_error()
    assert np.array_equal(host(k), want_k)
    assert np.array_equal(host(v), want_v)


def test_copy_blocks_bad_id_is_reported_and_others_copied():
    k, v = pool(32, 4, 128, "bf16", seed=7)
    m = np.array([[1, 2], [3, 40], [-1, 5], [6, 7]], np.int32)
    want_k, want_v = O.copy_blocks(host(k), host(v), m[[0, 3]])
    pa.pa_copy_blocks(k, v, torch.from_numpy(m).to(DEV))
    with pytest.raises(pa.PaError) as e:
        pa.pa_get_device_error()
    assert e.value.status == pa.Status.DEVICE_BOUNDS
    assert np.array_equal(host(k), want_k) and np.array_equal(host(v), want_v)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_swap_out_and_in_bit_exact(dtype, d):
    hkv = 8
    k, v = pool(48, hkv, d, dtype, seed=11)
    hk, hv = pool(20, hkv, d, dtype, seed=12, device="cpu")
    hk, hv = hk.pin_memory(), hv.pin_memory()
    out_map = np.array([[5, 3], [17, 0], [40, 19], [8, 8]], np.int32)
    want_hk, want_hv = O.swap_blocks(host(k), host(v), host(hk), host(hv), out_map)
    # swap out, mapping in device memory
    pa.pa_swap_blocks(k, v, hk, hv, torch.from_numpy(out_map).to(DEV))
    torch.cuda.synchronize()
    pa.pa_get_device_error()
    assert np.array_equal(host(hk), want_hk) and np.array_equal(host(hv), want_hv)
    # swap back in to other device blocks, mapping in page-locked host memory
    in_map = np.array([[3, 30], [0, 2], [19, 47], [8, 11]], np.int32)
    want_k, want_v = O.swap_blocks(host(hk), host(hv), host(k), host(v), in_map)
    pa.pa_swap_blocks(hk, hv, k, v, torch.from_numpy(in_map).pin_memory())
    torch.cuda.synchronize()
    pa.pa_get_device_error()
    assert np.array_equal(host(k), want_k) and np.array_equal(host(v), want_v)


def test_swap_refuses_pageable_host_memory():
    k, v = pool(8, 2, 64, "bf16", seed=3)
    hk = np.zeros((8, 2, 16, 64), np.uint16)
    m = torch.tensor([[0, 1]], dtype=torch.int32, device=DEV)
    p = hk.ctypes.data_as(ctypes.c_void_p)
    st = pa.lib().pa_swap_blocks(k.data_ptr(), v.data_ptr(), p, p, m.data_ptr(), 1, 2, 64, 16,
                                 8, 8, 1, torch.cuda.current_stream().cuda_stream)
    assert st == pa.Status.INVALID_ARG
    assert b"page-locked" in pa.lib().pa_last_error_message()
    assert not hk.any()


def test_cow_fork_then_decode():
    """"vLLM 架构源码解析" §4.3.2: three samples share a 37-token prompt in
    blocks [0, 1, 2]; sample 0 copies block 2 to block 10, writes its next
    token into slot 5 of the copy and decodes; samples 1 and 2 still read the
    unmodified shared block."""
    hkv, hq, d = 8, 32, 128
    k, v = pool(40, hkv, d, "bf16", seed=21)
    g = torch.Generator(device="cpu").manual_seed(22)
    nk = torch.randn(1, hkv, d, generator=g).to(torch.bfloat16).to(DEV)
    nv = torch.randn(1, hkv, d, generator=g).to(torch.bfloat16).to(DEV)
    q = torch.randn(3, hq, d, generator=g).to(torch.bfloat16).to(DEV)
    m = np.array([[2, 10]], np.int32)
    slot = np.array([10 * 16 + 5], np.int32)
    tables = np.array([[0, 1, 10], [0, 1, 2], [0, 1, 2]], np.int32)
    lens = np.array([38, 37, 37], np.int32)
    ok, ov = O.copy_blocks(host(k), host(v), m)
    ok, ov = O.reshape_and_cache(ok, ov, host(nk), host(nv), slot)
    ref = O.paged_decode(host(q), ok, ov, tables, lens, d ** -0.5, "bf16")
    pa.pa_copy_blocks(k, v, torch.from_numpy(m).to(DEV))
    pa.pa_reshape_and_cache(nk, nv, k, v, torch.from_numpy(slot).to(DEV))
    out = torch.full_like(q, float("nan"))
    ws = pa.alloc_workspace(pa.pa_decode_workspace_size(3, hq, hkv, d, 38), DEV)
    pa.pa_decode(out, q, k, v, torch.from_numpy(tables).to(DEV), torch.from_numpy(lens).to(DEV),
                 38, d ** -0.5, ws)
    pa.pa_get_device_error()
    assert np.array_equal(host(k), ok) and np.array_equal(host(v), ov)
    assert_close(out, ref, "bf16", "decode after copy-on-write")
