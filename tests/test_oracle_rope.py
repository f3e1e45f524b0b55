"""Pins for the oracle's rotary embedding + cache write, CPU only.

The pages do not define RoPE; these pins tie the oracle to the mathematics of
the rotation (RoFormer): the angle-0 row is the identity, every pair keeps its
norm, a unit pair turned by a known angle lands on (cos, sin), the dot product
of a rotated query at position m and a rotated key at position n depends only
on n - m, the two pair layouts agree up to the permutation that maps one to
the other, and dims past rot_dim pass through.  The cache write itself is
checked against the oracle's plain reshape_and_cache.  Planted mistakes (the
sine's sign flipped, the pairs crossed, the position off by one, rot_dim
ignored) each fail at least one pin.
"""

import numpy as np
import pytest

from oracle import paged_attention as OA
from oracle import rope as OR

BS = 16


def pin_identity_and_norm():
    rng = np.random.default_rng(0)
    table = OR.rope_table(64, 32).astype(np.float32)
    x = rng.standard_normal((4, 64))
    for neox in (False, True):
        assert np.array_equal(OR.rotate(x, table[0], 32, neox), x)   # cos 1, sin 0
        y = OR.rotate(x, table[37], 32, neox)
        if neox:
            n0 = x[:, :16] ** 2 + x[:, 16:32] ** 2
            n1 = y[:, :16] ** 2 + y[:, 16:32] ** 2
        else:
            n0 = x[:, 0:32:2] ** 2 + x[:, 1:32:2] ** 2
            n1 = y[:, 0:32:2] ** 2 + y[:, 1:32:2] ** 2
        np.testing.assert_allclose(n1, n0, rtol=1e-6)
        assert np.array_equal(y[:, 32:], x[:, 32:])                    # past rot_dim


def pin_known_angle():
    theta = 0.7
    row = np.array([np.cos(theta), np.sin(theta)])
    y = OR.rotate(np.array([1.0, 0.0, 5.0]), row, 2, False)
    np.testing.assert_allclose(y, [np.cos(theta), np.sin(theta), 5.0], rtol=0, atol=1e-15)
    y = OR.rotate(np.array([0.0, 1.0]), row, 2, True)
    np.testing.assert_allclose(y, [-np.sin(theta), np.cos(theta)], rtol=0, atol=1e-15)


def pin_relative_position():
    rng = np.random.default_rng(1)
    table = OR.rope_table(200, 64)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for neox in (False, True):
        dots = [OR.rotate(q, table[m], 64, neox) @ OR.rotate(k, table[m + 23], 64, neox)
                for m in (0, 5, 90, 150)]
        np.testing.assert_allclose(dots, dots[0], rtol=1e-9, atol=1e-9)


def pin_layouts_agree():
    rng = np.random.default_rng(2)
    table = OR.rope_table(50, 16)
    x = rng.standard_normal(24)
    perm = np.concatenate([np.arange(0, 16, 2), np.arange(1, 16, 2), np.arange(16, 24)])
    g = OR.rotate(x, table[11], 16, False)
    n = OR.rotate(x[perm], table[11], 16, True)
    np.testing.assert_allclose(n, g[perm], rtol=0, atol=1e-15)


def pin_cache_write():
    rng = np.random.default_rng(3)
    hq, hkv, d, nb, R = 4, 2, 32, 5, 16
    table = OR.rope_table(100, R).astype(np.float32)
    q = rng.standard_normal((3, hq, d)).astype(np.float32)
    k = rng.standard_normal((3, hkv, d)).astype(np.float32)
    v = rng.standard_normal((3, hkv, d)).astype(np.float32)
    kc = rng.standard_normal((nb, hkv, BS, d)).astype(np.float32)
    vc = rng.standard_normal((nb, hkv, BS, d)).astype(np.float32)
    slots = np.array([2 * BS + 4, -1, 0 * BS + 15])
    pos = np.array([0, 41, 99])
    qr, kr, vr = OR.rope_reshape_and_cache(q, k, v, kc, vc, slots, pos, table, R, True, "f32")
    # position 0: the k row is stored unrotated; v rows as given
    ok, ov = OA.reshape_and_cache(kc, vc, k, v, slots)
    assert np.array_equal(kr[2, :, 4], ok[2, :, 4].astype(np.float64))
    assert np.array_equal(vr, ov.astype(np.float64))
    np.testing.assert_allclose(kr[0, :, 15], OR.rotate(k[2].astype(np.float64), table[99], R,
                                                       True))
    untouched = np.ones((nb, BS), bool)
    untouched[2, 4] = untouched[0, 15] = False
    assert np.array_equal(kr.transpose(0, 2, 1, 3)[untouched],
                          kc.astype(np.float64).transpose(0, 2, 1, 3)[untouched])
    # q is rotated for padding tokens too
    np.testing.assert_allclose(qr[1], OR.rotate(q[1].astype(np.float64), table[41], R, True))


def pin_table_values():
    """The angle table of RoFormer: pair i of a rot_dim-dim rotation turns by
    p * base^(-2i/rot_dim) at position p.  Values fixed by the mathematics:
    row 0 is (cos 0, sin 0) = (1, 0); pair 0 has frequency 1, so row 1 holds
    (cos 1, sin 1) = (0.5403023058681398, 0.8414709848078965); with rot_dim 4
    and base 10000 pair 1 has frequency 10000^(-1/2) = 0.01, so at position
    100 it too is turned by exactly one radian; and cos^2 + sin^2 = 1."""
    t = OR.rope_table(128, 4)
    assert t.shape == (128, 4)
    assert np.array_equal(t[0], [1.0, 1.0, 0.0, 0.0])
    assert t[1, 0] == pytest.approx(0.5403023058681398, abs=1e-15)
    assert t[1, 2] == pytest.approx(0.8414709848078965, abs=1e-15)
    assert t[100, 1] == pytest.approx(0.5403023058681398, abs=1e-13)
    assert t[100, 3] == pytest.approx(0.8414709848078965, abs=1e-13)
    big = OR.rope_table(300, 64)
    np.testing.assert_allclose(big[:, :32] ** 2 + big[:, 32:] ** 2, 1.0, atol=1e-14)


ALL_PINS = [pin_identity_and_norm, pin_known_angle, pin_relative_position, pin_layouts_agree,
            pin_cache_write, pin_table_values]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin()


_orig_rotate = OR.rotate


def _mut_sign(x64, row, rot_dim, neox):
    cs = np.asarray(row, dtype=np.float64).copy()
    cs[rot_dim // 2:rot_dim] *= -1
    return _orig_rotate(x64, cs, rot_dim, neox)


def _mut_cross(x64, row, rot_dim, neox):
    return _orig_rotate(x64, row, rot_dim, not neox)


def _mut_no_rot_dim(x64, row, rot_dim, neox):
    d = x64.shape[-1]
    half = rot_dim // 2
    cs = np.asarray(row, dtype=np.float64)
    full = np.concatenate([cs[:half], np.ones(d // 2 - half), cs[half:rot_dim],
                           np.zeros(d // 2 - half)])
    return _orig_rotate(x64, full, d, neox)


def _mut_table(max_position, rot_dim, base=10000.0):
    inv = base ** (-np.arange(0, rot_dim // 2, dtype=np.float64) / rot_dim)  # exponent halved
    ang = np.arange(max_position, dtype=np.float64)[:, None] * inv[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1)


@pytest.mark.parametrize("name", ["sign", "cross", "position", "rot_dim", "table"])
def test_pins_catch_planted_mistake(name, monkeypatch):
    if name == "table":
        monkeypatch.setattr(OR, "rope_table", _mut_table)
    elif name == "sign":
        monkeypatch.setattr(OR, "rotate", _mut_sign)
    elif name == "cross":
        monkeypatch.setattr(OR, "rotate", _mut_cross)
    elif name == "rot_dim":
        monkeypatch.setattr(OR, "rotate", _mut_no_rot_dim)
    elif name == "position":
        orig = OR.rope_reshape_and_cache

        def shifted(q, k, v, kc, vc, slots, pos, table, R, neox, dtype, block_size=BS):
            return orig(q, k, v, kc, vc, slots, np.minimum(np.asarray(pos) + 1, len(table) - 1),
                        table, R, neox, dtype, block_size)
        monkeypatch.setattr(OR, "rope_reshape_and_cache", shifted)
    caught = 0
    for pin in ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"{name} passed every pin"
