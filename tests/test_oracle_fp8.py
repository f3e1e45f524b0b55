"""Pins for the oracle's FP8 (e4m3) KV cache, CPU only.

* The codec against torch's float8_e4m3fn (a library routine): all 256 codes
  decode to the same values, and in-range fp32 values encode to the same codes.
* Closed forms from the format's definition: saturation at 448, ties to the
  even mantissa in the normal and the subnormal range, exact round trips.
* The quantising cache write on values that are exact multiples of the scale.
* Attention on an FP8 cache against torch's scaled_dot_product_attention in
  float64 on the dequantized contiguous sequence (decode and a causal chunk).
Planted mistakes (a wrong exponent bias, truncation instead of rounding, the
scale multiplied instead of divided, the V scale dropped, saturation to NaN)
each fail at least one pin.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8 as OF
from oracle import paged_attention as OA
from tests.test_oracle_pins import BS, add_sequence, sdpa_ref


def torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def torch_encode(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def pin_decode_table():
    codes = np.arange(256, dtype=np.uint8)
    mine, ref = OF.e4m3_decode(codes), torch_decode(codes)
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    assert OF.e4m3_decode([0x7E])[0] == 448.0 and OF.e4m3_decode([0x01])[0] == 2.0 ** -9


def pin_encode_matches_torch():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(6000) * np.exp(rng.uniform(-12, 6, 6000))).astype(np.float32)
    x = x[np.abs(x) < 440]
    assert np.array_equal(OF.e4m3_encode(x), torch_encode(x))


def pin_closed_forms():
    enc = OF.e4m3_encode
    # saturation, both signs
    assert list(enc([448.0, 449.0, 500.0, 1e30, -1e30])) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]
    # ties to the even mantissa: 1 + 1/16 lies between 1 (m=0) and 1.125 (m=1)
    assert enc([1.0625])[0] == 0x38
    assert enc([1.1875])[0] == 0x3A          # between m=1 and m=2: to m=2
    # subnormals: 2^-10 between 0 and 2^-9 -> 0; 3 * 2^-10 -> 2 * 2^-9
    assert enc([2.0 ** -10])[0] == 0x00 and enc([3 * 2.0 ** -10])[0] == 0x02
    # every finite code round-trips
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    assert np.array_equal(enc(OF.e4m3_decode(codes)), codes)


def pin_quantising_write():
    """Values that are scale * (an e4m3 value) are stored exactly; others are
    the nearest code of x / scale."""
    rng = np.random.default_rng(4)
    hkv, d, nb = 2, 8, 6
    ks = np.array([0.25, 0.0125], np.float32)
    vs = np.array([2.0, 0.5], np.float32)
    vals = OF.e4m3_decode(rng.integers(0, 0x7E, size=(3, hkv, d)).astype(np.uint8))
    k = (vals * ks[None, :, None]).astype(np.float32)
    v = (vals * vs[None, :, None]).astype(np.float32)
    kc = np.full((nb, hkv, BS, d), 0x7F, np.uint8)
    vc = kc.copy()
    slots = np.array([5 * BS + 2, -1, 0 * BS + 15])
    k2, v2 = OF.reshape_and_cache_fp8(kc, vc, k, v, slots, ks, vs, "f32")
    assert np.array_equal(OF.e4m3_decode(k2[5, :, 2]), vals[0])
    assert np.array_equal(OF.e4m3_decode(v2[0, :, 15]), vals[2])
    untouched = np.ones((nb, BS), bool)
    untouched[5, 2] = untouched[0, 15] = False
    assert np.all(k2.transpose(0, 2, 1, 3)[untouched] == 0x7F)
    # a value between codes: x / scale rounded to nearest
    x = np.array([[[0.3] * d] * hkv], np.float32)
    k3, _ = OF.reshape_and_cache_fp8(kc, vc, x, x, np.array([7]), ks, vs, "f32")
    assert np.array_equal(k3[0, :, 7], torch_encode(np.float32(0.3) / ks)[:, None].repeat(d, 1))


def pin_attention_on_fp8_cache():
    rng = np.random.default_rng(8)
    hkv, hq, d, nb = 2, 4, 16, 24
    ks = np.array([0.02, 0.05], np.float32)
    vs = np.array([0.01, 0.03], np.float32)
    L = 2 * BS + 7
    kcodes = rng.integers(0, 0x7E, size=(L, hkv, d)).astype(np.uint8) ^ \
        (rng.integers(0, 2, size=(L, hkv, d)).astype(np.uint8) << 7)
    vcodes = rng.integers(0, 0x7E, size=(L, hkv, d)).astype(np.uint8)
    table = np.array([[9, 3, 17]], np.int32)
    kc = np.full((nb, hkv, BS, d), 0x7F, np.uint8)
    vc = kc.copy()
    add_sequence(kc, kcodes, table[0])
    add_sequence(vc, vcodes, table[0])
    k64 = OF.e4m3_decode(kcodes) * ks[None, :, None]
    v64 = OF.e4m3_decode(vcodes) * vs[None, :, None]
    q = rng.standard_normal((1, hq, d)).astype(np.float32)
    out = OF.paged_decode_fp8(q, kc, vc, ks, vs, table, np.array([L]), 0.3, "f32")
    ref = sdpa_ref(q.astype(np.float64), k64, v64, 0.3)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    # a causal chunk of 9 queries at the end of the same sequence
    qc = rng.standard_normal((9, hq, d)).astype(np.float32)
    outc = OF.paged_varlen_fp8(qc, kc, vc, ks, vs, table, np.array([0, 9]), np.array([L]), 0.3,
                               "f32")
    mask = np.array([[j <= L - 9 + i for j in range(L)] for i in range(9)])
    refc = sdpa_ref(qc.astype(np.float64), k64, v64, 0.3, mask=mask[None])
    np.testing.assert_allclose(outc, refc, rtol=1e-12, atol=1e-13)


ALL_PINS = [pin_decode_table, pin_encode_matches_torch, pin_closed_forms, pin_quantising_write,
            pin_attention_on_fp8_cache]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin()


def _mut_bias8(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e, m = (c >> 3) & 0xF, c & 0x7
    out = np.where(e == 0, sign * np.ldexp(m / 8.0, -7),
                   sign * np.ldexp(1.0 + m / 8.0, (e - 8).astype(np.int64)))
    return np.where((e == 15) & (m == 7), np.nan, out)


def _truncating(x):
    out = OF_encode_orig(x)
    dec = OF.e4m3_decode(out)
    xx = np.asarray(x, np.float64)
    # step toward zero where rounding went away from zero
    away = np.abs(dec) > np.abs(xx)
    out = out.copy()
    out[away & ((out & 0x7F) > 0)] -= 1
    return out


def _mut_nan_saturation(x):
    out = OF_encode_orig(x)
    big = np.abs(np.asarray(x, np.float64)) >= 448
    out = out.copy()
    out[big] |= 0x7F
    return out


OF_encode_orig = OF.e4m3_encode


@pytest.mark.parametrize("name", ["bias8", "truncate", "scale_multiplied", "v_scale_dropped",
                                  "nan_saturation"])
def test_pins_catch_planted_mistake(name, monkeypatch):
    if name == "bias8":
        monkeypatch.setattr(OF, "e4m3_decode", _mut_bias8)
    elif name == "truncate":
        monkeypatch.setattr(OF, "e4m3_encode", _truncating)
    elif name == "nan_saturation":
        monkeypatch.setattr(OF, "e4m3_encode", _mut_nan_saturation)
    elif name == "scale_multiplied":
        orig = OF.reshape_and_cache_fp8

        def wrong(kc, vc, k, v, slots, ks, vs, dtype, block_size=BS):
            return orig(kc, vc, k, v, slots, 1.0 / np.asarray(ks, np.float32),
                        1.0 / np.asarray(vs, np.float32), dtype, block_size)
        monkeypatch.setattr(OF, "reshape_and_cache_fp8", wrong)
    elif name == "v_scale_dropped":
        orig_deq = OF.dequantize
        calls = {"n": 0}

        def deq(codes, scales):
            calls["n"] += 1
            return orig_deq(codes, scales if calls["n"] % 2 == 1 else np.ones_like(scales))
        monkeypatch.setattr(OF, "dequantize", deq)
    caught = 0
    for pin in ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"{name} passed every pin"
