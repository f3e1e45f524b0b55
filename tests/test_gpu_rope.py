"""GPU parity of pa_rope_reshape_and_cache against the oracle.

The rotated values are floating-point results: each must lie within one unit
in the last place of the storage type of the oracle's exact value (fp32
storage: 2^-21 relative, two fp32 roundings), plus 2^-20 absolute for the
fp32 arithmetic where the two products nearly cancel.  Everything the call only
copies -- dims past rot_dim, the v rows -- and everything it must not touch --
other cache slots, padding tokens' cache rows -- is compared bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle as O
import pagedattention_paged_kv_reshape_b200 as pa
from pagedattention_paged_kv_reshape_b200 import workload as W
from tests._helpers import f64, host

pytestmark = pytest.mark.gpu
DEV = "cuda"
ULP = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11, "f32": 2.0 ** -21}


def within_ulp(got: np.ndarray, ref: np.ndarray, dtype: str, what: str):
    # one ulp of the storage type, plus 2^-20 for the fp32 arithmetic when
    # x1 c and x2 s nearly cancel (inputs are N(0,1)-sized)
    tol = ULP[dtype] * np.abs(ref) + 2.0 ** -20
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{what}: {bad.sum()} values off by more than one ulp"


# (q dtype, head_dim, rot_dim, NeoX pairs, block_size, q heads, KV heads, table
# offset in floats).  rot_dim a multiple of 8 with an aligned table takes the
# vector kernel (16-head parts: 24 q heads make a ragged second part); rot_dim 36 or 62,
# or a table 4 bytes off alignment, take the per-element kernel.
ROPE_CASES = [("bf16", 128, 128, True, 16, 8, 2, 0),
              ("f16", 64, 32, False, 8, 8, 2, 0),
              ("f32", 128, 64, True, 32, 8, 2, 0),
              ("bf16", 64, 64, False, 16, 8, 2, 0),
              ("bf16", 128, 128, False, 16, 24, 12, 0),
              ("f16", 256, 192, True, 32, 24, 12, 0),
              ("f32", 64, 56, False, 16, 4, 4, 0),
              ("bf16", 128, 36, True, 16, 8, 2, 0),
              ("f16", 64, 62, False, 8, 8, 4, 0),
              ("bf16", 128, 128, True, 16, 8, 2, 1),
              ("bf16", 64, 64, True, 16, 20, 20, 0)]


@pytest.mark.parametrize("dtype,d,rot,neox,bs,hq,hkv,offset", ROPE_CASES)
def test_rope_cache_write_matches_oracle(dtype, d, rot, neox, bs, hq, hkv, offset):
    b = W.build_batch([W.Request(L, q) for L, q in [(1, 1), (40, 7), (300, 300), (17, 1)]],
                      num_q_heads=hq, num_kv_heads=hkv, head_dim=d, dtype=dtype, seed=9,
                      device=DEV, pool_factor=1.3, block_size=bs)
    maxp = 512
    host_table = O.rope_table(maxp, rot).astype(np.float32)
    buf = torch.empty(maxp * rot + offset, dtype=torch.float32, device=DEV)
    table = buf[offset:].view(maxp, rot)
    table.copy_(torch.from_numpy(host_table))
    assert (table.data_ptr() % 16 == 0) == (offset == 0)
    positions = torch.from_numpy(np.concatenate(
        [np.arange(r.seq_len - r.q_len, r.seq_len) for r in b.requests]).astype(np.int32)).to(DEV)
    slots = b.slot_mapping.clone()
    slots[::5] = -1
    hs = b.host_slots.copy()
    hs[::5] = -1
    q0, kc0, vc0 = host(b.q), host(b.k_cache), host(b.v_cache)
    q, kc, vc = b.q.clone(), b.k_cache.clone(), b.v_cache.clone()
    pa.pa_rope_reshape_and_cache(q, b.k_new, b.v_new, kc, vc, slots, positions, table, neox)
    pa.pa_get_device_error()
    rq, rk, rv = O.rope_reshape_and_cache(q0, host(b.k_new), host(b.v_new), kc0, vc0, hs,
                                          host(positions), host(table), rot, neox, dtype,
                                          block_size=bs)
    within_ulp(f64(q)[..., :rot], rq[..., :rot], dtype, "rotated q")
    assert np.array_equal(host(q)[..., rot:], q0[..., rot:])
    within_ulp(f64(kc), rk, dtype, "cache after the write")
    written = np.zeros(kc.shape[0] * bs, bool)
    written[hs[hs >= 0]] = True
    written = written.reshape(kc.shape[0], bs)
    # untouched slots keep their bytes (NaN poison included); copied parts are exact
    k_now, v_now = host(kc).transpose(0, 2, 1, 3), host(vc).transpose(0, 2, 1, 3)
    assert np.array_equal(k_now[~written].view(np.uint8), kc0.transpose(0, 2, 1, 3)[~written]
                          .view(np.uint8))
    assert np.array_equal(v_now[~written].view(np.uint8), vc0.transpose(0, 2, 1, 3)[~written]
                          .view(np.uint8))
    ok, ov = O.reshape_and_cache(kc0, vc0, host(b.k_new), host(b.v_new), hs, block_size=bs)
    assert np.array_equal(host(vc).view(np.uint8), ov.view(np.uint8))
    assert np.array_equal(k_now[written][..., rot:], ok.transpose(0, 2, 1, 3)[written][..., rot:])


@pytest.mark.parametrize("offset", [0, 1])   # vector kernel, per-element kernel
def test_rope_bad_position_is_reported(offset):
    b = W.build_batch([W.Request(20, 4)], num_q_heads=4, num_kv_heads=2, head_dim=64,
                      dtype="bf16", seed=2, device=DEV)
    buf = torch.empty(32 * 64 + offset, dtype=torch.float32, device=DEV)
    table = buf[offset:].view(32, 64)
    table.copy_(torch.from_numpy(O.rope_table(32, 64).astype(np.float32)))
    positions = torch.tensor([16, 17, 40, 19], dtype=torch.int32, device=DEV)   # 40 >= 32
    q = b.q.clone()
    pa.pa_rope_reshape_and_cache(q, b.k_new, b.v_new, b.k_cache, b.v_cache, b.slot_mapping,
                                 positions, table)
    with pytest.raises(pa.PaError) as e:
        pa.pa_get_device_error()
    assert e.value.status == pa.Status.DEVICE_BOUNDS
    assert torch.equal(q[2], b.q[2])       # that token is left as it was
