"""FP8 (e4m3) KV cache: encoding, the quantising cache write, attention on it.

TEST INFRASTRUCTURE ONLY (see the package header).

"vLLM 深度拆解" §10.1 names native FP8 support with calibrated scales as the
next step for the engine.  The reading taken here: K and V are stored as FP8
e4m3 codes with one fp32 scale per KV head for K and one for V (the
calibration), and a cached value stands for ``decode(code) * scale``.

e4m3 (the OCP 8-bit floating-point format E4M3, "fn" variant): bit 7 sign,
bits 6..3 exponent field E with bias 7, bits 2..0 mantissa m.
  E in 1..15:  (-1)^s * 2^(E-7) * (1 + m/8), except E = 15, m = 7: NaN
  E = 0:       (-1)^s * 2^(-6) * (m/8)           (subnormals, 2^-9 apart)
There is no infinity; the largest finite magnitude is 2^8 * 1.75 = 448.

Encoding of an fp32 value x: round to the nearest representable value, ties
to the even mantissa; magnitudes at or above 448 saturate to 448 (a finite
code, never NaN).  The cache write encodes ``x / scale`` with the division
done in fp32 (one correctly rounded quotient), so the device and this oracle
take the same rounding decision on the same fp32 number.
"""

from __future__ import annotations

import numpy as np

from .paged_attention import (BLOCK_SIZE, paged_decode, paged_varlen, slot_to_block_offset,
                              to_f64)

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of e4m3 codes (uint8 array); NaN for the two NaN codes."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, -6)
    out = np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, out)


def e4m3_encode(x) -> np.ndarray:
    """e4m3 codes (uint8) of fp32 values ``x``: round to nearest, ties to even,
    saturating at +-448.  NaN inputs give the NaN code 0x7F (sign kept)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    out = np.zeros(x.shape, dtype=np.uint8)
    flat_x, flat_o = x.reshape(-1), out.reshape(-1)
    for i, v in enumerate(flat_x):
        s = 0x80 if np.signbit(v) else 0
        a = abs(v)
        if np.isnan(v):
            flat_o[i] = s | 0x7F
            continue
        if a >= E4M3_MAX:
            flat_o[i] = s | 0x7E                      # E = 15, m = 6: 448
            continue
        if a < 2.0 ** -6:                             # subnormal range: steps of 2^-9
            n = int(np.rint(a / 2.0 ** -9))           # rint rounds half to even
            if n == 8:                                # rounded up to 2^-6: the first normal
                flat_o[i] = s | (1 << 3)
            else:
                flat_o[i] = s | n
            continue
        _, k = np.frexp(a)                            # a = f * 2^k, f in [0.5, 1)
        e = k - 1                                     # a in [2^e, 2^(e+1))
        n = int(np.rint(a / 2.0 ** (e - 3)))          # 8 .. 16 steps of 2^(e-3)
        if n == 16:                                   # rounded up to the next power of two
            e, n = e + 1, 8
        code = ((e + 7) << 3) | (n - 8)
        if code > 0x7E:                               # past 448 after rounding: saturate
            code = 0x7E
        flat_o[i] = s | code
    return out


def dequantize(cache_codes, scales) -> np.ndarray:
    """float64 values of a cache ``[num_blocks, Hkv, block_size, D]`` of codes
    with per-KV-head ``scales`` ``[Hkv]``."""
    return e4m3_decode(cache_codes) * np.asarray(scales, dtype=np.float32).astype(
        np.float64)[None, :, None, None]


def reshape_and_cache_fp8(k_cache, v_cache, k, v, slot_mapping, k_scale, v_scale, dtype: str,
                          block_size: int = BLOCK_SIZE):
    """The quantising cache write: token t's rows go to slot ``slot_mapping[t]``
    (negative = padding, skipped) as ``encode(float32(x) / float32(scale[h]))``
    for KV head h ("vLLM 架构源码解析" §3.3.3 for the write itself).  Returns new
    code arrays; the inputs are not modified."""
    k_out = np.array(k_cache, dtype=np.uint8, copy=True)
    v_out = np.array(v_cache, dtype=np.uint8, copy=True)
    ks = np.asarray(k_scale, dtype=np.float32)
    vs = np.asarray(v_scale, dtype=np.float32)
    for t in range(len(slot_mapping)):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        blk, off = slot_to_block_offset(slot, block_size)
        for h in range(k.shape[1]):
            kq = to_f64(k[t, h], dtype).astype(np.float32) / ks[h]
            vq = to_f64(v[t, h], dtype).astype(np.float32) / vs[h]
            k_out[blk, h, off, :] = e4m3_encode(kq)
            v_out[blk, h, off, :] = e4m3_encode(vq)
    return k_out, v_out


def paged_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                     scale: float, dtype: str, block_size: int = BLOCK_SIZE, seqs=None):
    """Decode attention over an e4m3 cache: exactly ``paged_decode`` on the
    dequantized cache (``dtype`` is that of q and out)."""
    return paged_decode(to_f64(q, dtype), dequantize(k_cache, k_scale),
                        dequantize(v_cache, v_scale), block_tables, context_lens, scale, "f64",
                        block_size=block_size, seqs=seqs)


def paged_varlen_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables, query_start_loc,
                     seq_lens, scale: float, dtype: str, block_size: int = BLOCK_SIZE,
                     seqs=None):
    """Mixed batch over an e4m3 cache: ``paged_varlen`` on the dequantized cache."""
    return paged_varlen(to_f64(q, dtype), dequantize(k_cache, k_scale),
                        dequantize(v_cache, v_scale), block_tables, query_start_loc, seq_lens,
                        scale, "f64", block_size=block_size, seqs=seqs)
