"""Pins for the oracle's block operations (copy-on-write and swap), CPU only.

Each pin ties ``oracle.copy_blocks`` / ``oracle.swap_blocks`` to something
other than themselves: the copy-on-write scenario of "vLLM 架构源码解析"
§4.3.2 (three samples share a prompt's blocks, one writes into the shared,
partly filled last block after taking a private copy of it) checked with
torch's scaled_dot_product_attention in float64 on the contiguous sequences,
and a swap-out / swap-in round trip ("vLLM 架构源码解析" §1, v0 (Swap)) that
must leave every request's attention output bit-identical.  Planted mistakes
(K copied but not V, source and destination exchanged, one head dropped) are
each caught.
"""

import numpy as np
import pytest

import oracle
from oracle import block_ops as OB
from oracle import paged_attention as OA
from tests.test_oracle_pins import BS, add_sequence, golden, sdpa_ref


def test_copy_moves_exactly_the_pairs():
    rng = np.random.default_rng(3)
    kc = rng.standard_normal((9, 2, BS, 8)).astype(np.float32)
    vc = rng.standard_normal((9, 2, BS, 8)).astype(np.float32)
    kc0, vc0 = kc.copy(), vc.copy()
    k2, v2 = oracle.copy_blocks(kc, vc, np.array([[3, 5], [7, 7], [0, 8]], np.int32))
    for b in range(9):
        want_k = kc[3] if b == 5 else kc[0] if b == 8 else kc[b]
        want_v = vc[3] if b == 5 else vc[0] if b == 8 else vc[b]
        assert np.array_equal(k2[b], want_k) and np.array_equal(v2[b], want_v), b
    assert np.array_equal(kc, kc0) and np.array_equal(vc, vc0)  # inputs untouched
    k3, _ = oracle.copy_blocks(kc, vc, np.zeros((0, 2), np.int32))
    assert np.array_equal(k3, kc)


def pin_cow_fork():
    """[ARCH] §4.3.2: samples share prompt blocks [0, 1, 2] (golden tables).
    The prompt has 37 tokens, so block 2 is shared and only 5/16 full.  Sample
    0 appends a token: copy-on-write gives it a private copy of block 2 (here
    block 10, the first block of its own tail in the page's table) and the new
    token goes to slot 5 of that copy.  Afterwards sample 0 attends to the
    prompt plus its token, samples 1 and 2 to the prompt alone."""
    tables_g = golden("block_sharing_examples.json")["cow_example"]["tables"]
    rng = np.random.default_rng(21)
    hkv, hq, d, nb = 2, 4, 16, 40
    plen = 2 * BS + 5
    pk = rng.standard_normal((plen, hkv, d)).astype(np.float32)
    pv = rng.standard_normal((plen, hkv, d)).astype(np.float32)
    kc = np.full((nb, hkv, BS, d), np.nan, np.float32)
    vc = np.full((nb, hkv, BS, d), np.nan, np.float32)
    prompt_blocks = tables_g[0][:3]
    add_sequence(kc, pk, prompt_blocks)
    add_sequence(vc, pv, prompt_blocks)
    private = tables_g[0][3]
    kc, vc = oracle.copy_blocks(kc, vc, np.array([[prompt_blocks[2], private]], np.int32))
    nk = rng.standard_normal((1, hkv, d)).astype(np.float32)
    nv = rng.standard_normal((1, hkv, d)).astype(np.float32)
    kc, vc = OA.reshape_and_cache(kc, vc, nk, nv, np.array([private * BS + 5]))
    tables = np.array([prompt_blocks[:2] + [private], prompt_blocks, prompt_blocks], np.int32)
    lens = np.array([plen + 1, plen, plen])
    q = rng.standard_normal((3, hq, d)).astype(np.float32)
    out = OA.paged_decode(q, kc, vc, tables, lens, 0.25, "f32")
    f64 = lambda a: a.astype(np.float64)  # noqa: E731
    ref0 = sdpa_ref(f64(q[:1]), f64(np.concatenate([pk, nk])), f64(np.concatenate([pv, nv])),
                    0.25)
    np.testing.assert_allclose(out[0], ref0[0], rtol=1e-12, atol=1e-13)
    for i in (1, 2):
        ref = sdpa_ref(f64(q[i:i + 1]), f64(pk), f64(pv), 0.25)
        np.testing.assert_allclose(out[i], ref[0], rtol=1e-12, atol=1e-13)


def pin_swap_round_trip():
    """[ARCH] §1 v0 (Swap): swap a request's blocks out to a host pool, let
    other work overwrite the device blocks, swap them back in to different
    device blocks; the request's output is bit-identical through its new
    table."""
    rng = np.random.default_rng(5)
    hkv, hq, d, nb, host_nb = 2, 4, 8, 24, 10
    L = 3 * BS + 9
    table = np.array([[4, 17, 9, 2]], np.int32)
    kc = rng.standard_normal((nb, hkv, BS, d)).astype(np.float32)
    vc = rng.standard_normal((nb, hkv, BS, d)).astype(np.float32)
    q = rng.standard_normal((1, hq, d)).astype(np.float32)
    before = OA.paged_decode(q, kc, vc, table, np.array([L]), 0.4, "f32")
    host_k = np.zeros((host_nb, hkv, BS, d), np.float32)
    host_v = np.zeros((host_nb, hkv, BS, d), np.float32)
    out_map = np.array([[b, i + 3] for i, b in enumerate(table[0])], np.int32)
    host_k, host_v = oracle.swap_blocks(kc, vc, host_k, host_v, out_map)
    kc[:] = np.nan
    vc[:] = np.nan
    new_table = np.array([[11, 0, 23, 6]], np.int32)
    in_map = np.array([[i + 3, b] for i, b in enumerate(new_table[0])], np.int32)
    kc, vc = oracle.swap_blocks(host_k, host_v, kc, vc, in_map)
    after = OA.paged_decode(q, kc, vc, new_table, np.array([L]), 0.4, "f32")
    assert np.array_equal(before, after)
    k64 = OA.gather_sequence(kc, new_table[0], L).astype(np.float64)
    v64 = OA.gather_sequence(vc, new_table[0], L).astype(np.float64)
    ref = sdpa_ref(q.astype(np.float64), k64, v64, 0.4)
    np.testing.assert_allclose(after, ref, rtol=1e-12, atol=1e-13)


def test_cow_fork():
    pin_cow_fork()


def test_swap_round_trip():
    pin_swap_round_trip()


def _mut_k_only(src_k, src_v, dst_k, dst_v, block_mapping):
    k_out, v_out = np.array(dst_k, copy=True), np.array(dst_v, copy=True)
    for s, t in np.asarray(block_mapping).reshape(-1, 2):
        k_out[t] = src_k[s]
    return k_out, v_out


def _mut_reversed(src_k, src_v, dst_k, dst_v, block_mapping):
    k_out, v_out = np.array(dst_k, copy=True), np.array(dst_v, copy=True)
    for s, t in np.asarray(block_mapping).reshape(-1, 2):
        if t < len(src_k) and s < len(k_out):
            k_out[s] = src_k[t]
            v_out[s] = src_v[t]
    return k_out, v_out


def _mut_first_head(src_k, src_v, dst_k, dst_v, block_mapping):
    k_out, v_out = np.array(dst_k, copy=True), np.array(dst_v, copy=True)
    for s, t in np.asarray(block_mapping).reshape(-1, 2):
        k_out[t, 0] = src_k[s, 0]
        v_out[t, 0] = src_v[s, 0]
    return k_out, v_out


@pytest.mark.parametrize("mutant", [_mut_k_only, _mut_reversed, _mut_first_head])
def test_pins_catch_planted_mistake(mutant, monkeypatch):
    monkeypatch.setattr(OB, "swap_blocks", mutant)
    monkeypatch.setattr(oracle, "swap_blocks", mutant)
    monkeypatch.setattr(oracle, "copy_blocks",
                        lambda k, v, m: mutant(k, v, k, v, m))
    caught = 0
    for pin in (pin_cow_fork, pin_swap_round_trip):
        try:
            with np.errstate(invalid="ignore"):
                pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"{mutant.__name__} passed every pin"
