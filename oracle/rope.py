"""Rotary position embedding fused with the cache write.

TEST INFRASTRUCTURE ONLY (see the package header).

The pages do not define a position encoding; this is the kernel-fusion theme
of "vLLM 深度拆解" §6.1 (fold elementwise work into the kernel next to it so the
activations make one trip through HBM) applied to the cache write: q and k are
rotated on their way through, and the rotated k lands in the cache.

The rotation is the rotary position embedding as published with RoFormer
(Su et al., 2021): the first ``rot_dim`` dims of a head form rot_dim/2 pairs,
and the pair (x1, x2) of a token at position p is turned by the angle of
frequency i at p:
    x1' = x1 cos - x2 sin,   x2' = x2 cos + x1 sin.
Pairs are (2i, 2i+1) ("GPT-J" layout, neox=False) or (i, i + rot_dim/2)
("NeoX" layout, neox=True); dims from rot_dim on pass through.  The angles
come from the caller's table ``cos_sin[position] = [cos_0 .. cos_{R/2-1},
sin_0 .. sin_{R/2-1}]`` (fp32), as a serving engine keeps it.

The oracle computes each rotated value exactly (float64, from the fp32 table
and the stored inputs); the device rounds each once to the storage type.
"""

from __future__ import annotations

import numpy as np

from .paged_attention import BLOCK_SIZE, slot_to_block_offset, to_f64


def rope_table(max_position: int, rot_dim: int, base: float = 10000.0) -> np.ndarray:
    """The usual frequency table in float64: angle(p, i) = p * base^(-2i/R)."""
    inv = base ** (-np.arange(0, rot_dim, 2, dtype=np.float64) / rot_dim)
    ang = np.arange(max_position, dtype=np.float64)[:, None] * inv[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1)


def rotate(x64: np.ndarray, cos_sin_row, rot_dim: int, neox: bool) -> np.ndarray:
    """Rotate the head vectors ``x64`` (float64, [..., D]) of one token."""
    cs = np.asarray(cos_sin_row, dtype=np.float64)
    half = rot_dim // 2
    c, s = cs[:half], cs[half:rot_dim]
    out = np.array(x64, dtype=np.float64, copy=True)
    if neox:
        i1, i2 = np.arange(half), np.arange(half) + half
    else:
        i1, i2 = np.arange(0, rot_dim, 2), np.arange(1, rot_dim, 2)
    x1, x2 = x64[..., i1], x64[..., i2]
    out[..., i1] = x1 * c - x2 * s
    out[..., i2] = x2 * c + x1 * s
    return out


def rope_reshape_and_cache(q, k, v, k_cache, v_cache, slot_mapping, positions, cos_sin,
                           rot_dim: int, neox: bool, dtype: str,
                           block_size: int = BLOCK_SIZE):
    """Returns (q_rot, k_cache_values, v_cache): q rotated (float64), and the
    caches after the write, as float64 values, with token t's rotated k and its
    v at slot ``slot_mapping[t]`` (negative: padding, skipped; q is rotated
    all the same).  Cache entries the call does not write keep their values."""
    q64 = to_f64(q, dtype)
    kc = to_f64(k_cache, dtype)
    vc = to_f64(v_cache, dtype)
    q_out = np.array(q64, copy=True)
    for t in range(len(positions)):
        row = cos_sin[int(positions[t])]
        q_out[t] = rotate(q64[t], row, rot_dim, neox)
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        blk, off = slot_to_block_offset(slot, block_size)
        kc[blk, :, off, :] = rotate(to_f64(k[t], dtype), row, rot_dim, neox)
        vc[blk, :, off, :] = to_f64(v[t], dtype)
    return q_out, kc, vc
