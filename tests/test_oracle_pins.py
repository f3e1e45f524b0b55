"""Pins of the fp64 oracle against what the pages and the mathematics fix.

CPU only.  Each pin checks the oracle against something other than itself:
the pages' worked examples (``tests/golden``), closed forms, invariants the
pages state for paged attention, and the contiguous special case computed by
``torch.nn.functional.scaled_dot_product_attention`` in float64 on a cache
that the test lays out itself (never through the oracle's own gather).  The
last test plants plausible mistakes in the oracle and checks that the pins
catch every one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import paged_attention as OA

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BS = 16


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# helpers that build inputs without touching the oracle
# --------------------------------------------------------------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (RNE) via torch, for test inputs."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def encode(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return x.astype(np.float32)
    if dtype == "f16":
        return x.astype(np.float16)
    return bf16_bits(x)


def decoded(x_enc: np.ndarray, dtype: str) -> np.ndarray:
    """Values of encoded inputs in float64, computed by torch (not the oracle)."""
    if dtype == "bf16":
        return torch.from_numpy(x_enc.view(np.int16)).view(torch.bfloat16).double().numpy()
    return x_enc.astype(np.float64)


def lay_out(contig, table, num_blocks, fill=np.nan):
    """Place a contiguous [L, Hkv, D] sequence into a fresh pool through ``table``."""
    L, hkv, d = contig.shape
    pool = np.full((num_blocks, hkv, BS, d), fill, dtype=contig.dtype) if contig.dtype != np.uint16 \
        else np.full((num_blocks, hkv, BS, d), 0x7FC0, dtype=np.uint16)
    for pos in range(L):
        pool[table[pos // BS], :, pos % BS, :] = contig[pos]
    return pool


def add_sequence(pool, contig, table):
    for pos in range(contig.shape[0]):
        pool[table[pos // BS], :, pos % BS, :] = contig[pos]


def sdpa_ref(q, k, v, scale, mask=None, causal=False):
    """torch SDPA in float64.  q [n, Hq, D]; k, v [L, Hkv, D] (GQA via repeat)."""
    hq, hkv = q.shape[1], k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2).unsqueeze(0)           # [1, Hq, n, D]
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(hq // hkv, 0).unsqueeze(0)
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(hq // hkv, 0).unsqueeze(0)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m,
                                                         is_causal=causal, scale=scale)
    return o.squeeze(0).permute(1, 0, 2).numpy()


def random_case(rng, lengths, hq, hkv, d, dtype, extra_blocks=5):
    """Random contiguous sequences placed into a shuffled pool by the test."""
    nblk = [-(-L // BS) for L in lengths]
    num_blocks = sum(nblk) + extra_blocks + 1
    perm = rng.permutation(num_blocks)
    poison = int(perm[0])
    tables = np.full((len(lengths), max(nblk) + 2), poison, dtype=np.int32)
    cur = 1
    for i, n in enumerate(nblk):
        tables[i, :n] = perm[cur:cur + n]
        cur += n
    ks = [encode(rng.standard_normal((L, hkv, d)), dtype) for L in lengths]
    vs = [encode(rng.standard_normal((L, hkv, d)), dtype) for L in lengths]
    fillv = 0x7FC0 if dtype == "bf16" else np.nan
    kdt = ks[0].dtype
    kc = np.full((num_blocks, hkv, BS, d), fillv, dtype=kdt)
    vc = np.full((num_blocks, hkv, BS, d), fillv, dtype=kdt)
    for i in range(len(lengths)):
        add_sequence(kc, ks[i], tables[i])
        add_sequence(vc, vs[i], tables[i])
    return ks, vs, kc, vc, tables


# --------------------------------------------------------------------------
# the pages' worked examples
# --------------------------------------------------------------------------

def pin_block_table_example():
    g = golden("block_table_example.json")
    table = np.array(g["block_table"] + [0], dtype=np.int32)
    assert table[g["seq_id"] * len(table) + g["lookup_logical"]] == g["lookup_physical"]
    num_blocks = 100
    # every row of physical block b holds the value b in every element
    pool = np.broadcast_to(np.arange(num_blocks, dtype=np.float32)[:, None, None, None],
                           (num_blocks, 1, BS, 4)).copy()
    seq = OA.gather_sequence(pool, table, 3 * BS)
    assert seq.shape == (48, 1, 4)
    for logical, physical in enumerate(g["block_table"]):
        assert np.all(seq[logical * BS:(logical + 1) * BS] == physical)
    # a 17-token request reads only the first row of its second block
    seq17 = OA.gather_sequence(pool, table, 17)
    assert seq17.shape[0] == 17 and np.all(seq17[16] == g["lookup_physical"])


def pin_slot_placement():
    g = golden("block_table_example.json")
    table = g["block_table"]
    # token at logical position 17 of request A: physical block 88, offset 1
    slot = table[17 // BS] * BS + 17 % BS
    assert OA.slot_to_block_offset(slot) == (88, 1)
    num_blocks, hkv, d = 100, 2, 8
    sentinel = np.float32(-7.0)
    kc = np.full((num_blocks, hkv, BS, d), sentinel, np.float32)
    vc = kc.copy()
    k = np.arange(3 * hkv * d, dtype=np.float32).reshape(3, hkv, d)
    v = -k
    slots = np.array([slot, -1, 3 * BS + 15], dtype=np.int32)
    k2, v2 = OA.reshape_and_cache(kc, vc, k, v, slots)
    assert np.array_equal(k2[88, :, 1, :], k[0]) and np.array_equal(v2[88, :, 1, :], v[0])
    assert np.array_equal(k2[3, :, 15, :], k[2]) and np.array_equal(v2[3, :, 15, :], v[2])
    touched = np.zeros((num_blocks, BS), bool)
    touched[88, 1] = touched[3, 15] = True
    kt, vt = k2.transpose(0, 2, 1, 3), v2.transpose(0, 2, 1, 3)   # [blocks, slot, heads, D]
    assert np.all(kt[~touched] == sentinel) and np.all(vt[~touched] == sentinel)
    assert np.all(kc == sentinel)   # inputs untouched


def pin_prepare_inputs_positions():
    g = golden("prepare_inputs_example.json")
    pre = g["prefill"]
    qsl = np.concatenate([[0], np.cumsum(pre["prompt_lens"])]).tolist()
    assert qsl == pre["query_start_loc"]
    for L, pos in zip(pre["prompt_lens"], pre["positions"]):
        assert OA.query_positions(L, L) == pos
    dec = g["decode"]
    for n, pos in zip(dec["num_computed_tokens"], dec["positions"]):
        assert OA.query_positions(n + 1, 1) == pos


def test_pages_worked_examples():
    pin_block_table_example()
    pin_slot_placement()
    pin_prepare_inputs_positions()


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

def pin_bf16_decoding():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0001, 0x7F80, 0x8000], dtype=np.uint16)
    want = [1.0, -2.0, 1.0 + 2.0 ** -7, 2.0 ** -133, math.inf, -0.0]
    got = OA.to_f64(bits, "bf16")
    assert got.tolist() == want
    assert math.copysign(1.0, got[5]) == -1.0


def pin_context_one_returns_v():
    rng = np.random.default_rng(1)
    for dtype in ("f32", "bf16", "f16"):
        hq, hkv, d = 8, 2, 16
        ks, vs, kc, vc, tables = random_case(rng, [1, 1], hq, hkv, d, dtype)
        q = encode(rng.standard_normal((2, hq, d)) * 3, dtype)
        out = OA.paged_decode(q, kc, vc, tables, np.array([1, 1]), 0.125, dtype)
        for r in range(2):
            v64 = decoded(vs[r], dtype)[0]          # [Hkv, D]
            for h in range(hq):
                assert np.array_equal(out[r, h], v64[h // (hq // hkv)])


def pin_equal_values():
    rng = np.random.default_rng(2)
    hq, hkv, d, L = 4, 4, 8, 37
    ks, vs, kc, vc, tables = random_case(rng, [L], hq, hkv, d, "f32")
    row = rng.standard_normal((hkv, d)).astype(np.float32)
    vs[0][:] = row
    add_sequence(vc, vs[0], tables[0])
    q = rng.standard_normal((1, hq, d)).astype(np.float32)
    out = OA.paged_decode(q, kc, vc, tables, np.array([L]), 0.3, "f32")
    np.testing.assert_allclose(out[0], row.astype(np.float64), rtol=1e-14, atol=1e-14)


def pin_zero_query_gives_mean():
    rng = np.random.default_rng(3)
    hq, hkv, d, L = 4, 2, 8, 50
    ks, vs, kc, vc, tables = random_case(rng, [L], hq, hkv, d, "f32")
    q = np.zeros((1, hq, d), np.float32)
    out = OA.paged_decode(q, kc, vc, tables, np.array([L]), 0.3, "f32")
    mean = vs[0].astype(np.float64).mean(axis=0)
    for h in range(hq):
        np.testing.assert_allclose(out[0, h], mean[h // 2], rtol=1e-13, atol=1e-14)


def pin_dominant_key():
    rng = np.random.default_rng(4)
    hq, hkv, d, L = 2, 1, 8, 40
    ks, vs, kc, vc, tables = random_case(rng, [L], hq, hkv, d, "f32")
    q = np.zeros((1, hq, d), np.float32)
    q[0, :, 0] = 1.0
    k = np.zeros((L, hkv, d), np.float32)
    k[23, 0, 0] = 60.0          # score gap 60 * scale(=1) over every other key
    add_sequence(kc, k, tables[0])
    out = OA.paged_decode(q, kc, vc, tables, np.array([L]), 1.0, "f32")
    np.testing.assert_allclose(out[0, 0], vs[0][23, 0].astype(np.float64), rtol=0, atol=1e-20)


def pin_two_keys_closed_form():
    """Two keys: w1 = 1 / (1 + exp(scale * (s2 - s1))) -- pins scale and sign."""
    d, scale = 4, 0.7
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0] = [1.0, 2.0, 0.0, 0.0]
    k = np.zeros((2, 1, d), np.float32)
    k[0, 0] = [1.0, 0.0, 0.0, 0.0]      # q.k1 = 1
    k[1, 0] = [0.0, 1.5, 0.0, 0.0]      # q.k2 = 3
    v = np.zeros((2, 1, d), np.float32)
    v[0, 0] = [1.0, 0.0, 0.0, 0.0]
    v[1, 0] = [0.0, 1.0, 0.0, 0.0]
    table = np.array([[5, 0]], np.int32)
    kc = lay_out(k, table[0], 8)
    vc = lay_out(v, table[0], 8)
    out = OA.paged_decode(q, kc, vc, table, np.array([2]), scale, "f32")
    w1 = 1.0 / (1.0 + math.exp(scale * (3.0 - 1.0)))
    np.testing.assert_allclose(out[0, 0], [w1, 1.0 - w1, 0.0, 0.0], rtol=1e-15, atol=1e-16)


def pin_gqa_head_mapping():
    hq, hkv, d, L = 8, 2, 4, 20
    rng = np.random.default_rng(5)
    k = rng.standard_normal((L, hkv, d)).astype(np.float32)
    v = np.zeros((L, hkv, d), np.float32)
    v[:, 0, :] = 1.0
    v[:, 1, :] = 2.0
    table = np.array([[3, 1, 0]], np.int32)
    kc, vc = lay_out(k, table[0], 4), lay_out(v, table[0], 4)
    q = rng.standard_normal((1, hq, d)).astype(np.float32)
    out = OA.paged_decode(q, kc, vc, table, np.array([L]), 0.5, "f32")
    for h in range(hq):
        np.testing.assert_allclose(out[0, h], 1.0 + (h // 4), rtol=1e-14)


def test_closed_forms():
    pin_bf16_decoding()
    pin_context_one_returns_v()
    pin_equal_values()
    pin_zero_query_gives_mean()
    pin_dominant_key()
    pin_two_keys_closed_form()
    pin_gqa_head_mapping()


def test_empty_context_is_zero_row():
    rng = np.random.default_rng(6)
    ks, vs, kc, vc, tables = random_case(rng, [5], 2, 1, 8, "f32")
    q = rng.standard_normal((1, 2, 8)).astype(np.float32)
    out = OA.paged_decode(q, kc, vc, tables, np.array([0]), 0.3, "f32")
    assert np.array_equal(out, np.zeros_like(out))


# --------------------------------------------------------------------------
# paged == contiguous brute force (torch SDPA, float64)
# --------------------------------------------------------------------------

def pin_decode_matches_contiguous(dtype="bf16", seed=7):
    rng = np.random.default_rng(seed)
    hq, hkv, d = 8, 2, 32
    lengths = [1, 15, 16, 17, 64, 100]
    ks, vs, kc, vc, tables = random_case(rng, lengths, hq, hkv, d, dtype)
    q = encode(rng.standard_normal((len(lengths), hq, d)), dtype)
    scale = 1.0 / math.sqrt(d)
    out = OA.paged_decode(q, kc, vc, tables, np.array(lengths), scale, dtype)
    for r, L in enumerate(lengths):
        ref = sdpa_ref(decoded(q[r:r + 1], dtype), decoded(ks[r], dtype),
                       decoded(vs[r], dtype), scale)
        np.testing.assert_allclose(out[r], ref[0], rtol=1e-12, atol=1e-13)


def pin_varlen_matches_contiguous(dtype="f32", seed=8):
    rng = np.random.default_rng(seed)
    hq, hkv, d = 4, 2, 16
    # (seq_len, q_len): a chunk with no cache, a chunk on cache, decode rows
    rows = [(40, 40), (70, 23), (33, 1), (1, 1), (48, 16)]
    lengths = [s for s, _ in rows]
    ks, vs, kc, vc, tables = random_case(rng, lengths, hq, hkv, d, dtype)
    qsl = np.concatenate([[0], np.cumsum([ql for _, ql in rows])]).astype(np.int32)
    q = encode(rng.standard_normal((int(qsl[-1]), hq, d)), dtype)
    scale = 0.2
    out = OA.paged_varlen(q, kc, vc, tables, qsl, np.array(lengths), scale, dtype)
    for r, (L, ql) in enumerate(rows):
        qr = decoded(q[qsl[r]:qsl[r + 1]], dtype)
        k64, v64 = decoded(ks[r], dtype), decoded(vs[r], dtype)
        if ql == L:
            ref = sdpa_ref(qr, k64, v64, scale, causal=True)
        else:
            pos = np.arange(L - ql, L)[:, None]
            mask = np.arange(L)[None, :] <= pos         # key j visible iff j <= position
            ref = sdpa_ref(qr, k64, v64, scale, mask=mask)
        np.testing.assert_allclose(out[qsl[r]:qsl[r + 1]], ref, rtol=1e-12, atol=1e-13)


def test_paged_equals_contiguous_sdpa():
    for dtype in ("f32", "bf16", "f16"):
        pin_decode_matches_contiguous(dtype)
        pin_varlen_matches_contiguous(dtype)


def test_varlen_decode_rows_equal_decode():
    rng = np.random.default_rng(9)
    lengths = [3, 31, 77]
    ks, vs, kc, vc, tables = random_case(rng, lengths, 4, 4, 8, "bf16")
    q = encode(rng.standard_normal((3, 4, 8)), "bf16")
    a = OA.paged_decode(q, kc, vc, tables, np.array(lengths), 0.4, "bf16")
    b = OA.paged_varlen(q, kc, vc, tables, np.arange(4, dtype=np.int32), np.array(lengths),
                        0.4, "bf16")
    assert np.array_equal(a, b)


# --------------------------------------------------------------------------
# invariants the pages fix for paged attention
# --------------------------------------------------------------------------

def pin_permutation_invariance():
    rng = np.random.default_rng(10)
    lengths = [19, 64, 5]
    ks, vs, kc, vc, tables = random_case(rng, lengths, 4, 2, 16, "bf16")
    q = encode(rng.standard_normal((3, 4, 16)), "bf16")
    base = OA.paged_decode(q, kc, vc, tables, np.array(lengths), 0.25, "bf16")
    sigma = rng.permutation(kc.shape[0])             # physical id b -> sigma[b]
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[sigma], vc2[sigma] = kc, vc
    out = OA.paged_decode(q, kc2, vc2, sigma[tables].astype(np.int32), np.array(lengths),
                          0.25, "bf16")
    assert np.array_equal(out, base)


def pin_sharing_equals_private_copies():
    g = golden("block_sharing_examples.json")
    rng = np.random.default_rng(11)
    hq, hkv, d = 4, 2, 16
    t1, t2 = g["pool_example"]["tables"]
    shared = g["pool_example"]["shared"]
    L1, L2 = 4 * BS - 3, 3 * BS - 7
    prefix = encode(rng.standard_normal((len(shared) * BS, hkv, d)), "bf16")
    s1 = np.concatenate([prefix, encode(rng.standard_normal((L1 - len(prefix), hkv, d)), "bf16")])
    s2 = np.concatenate([prefix, encode(rng.standard_normal((L2 - len(prefix), hkv, d)), "bf16")])
    v1 = encode(rng.standard_normal((L1, hkv, d)), "bf16")
    v2 = encode(rng.standard_normal((L2, hkv, d)), "bf16")
    v2[:len(prefix)] = v1[:len(prefix)]
    nb = 12
    kc = np.full((nb, hkv, BS, d), 0x7FC0, np.uint16)
    vc = kc.copy()
    tables = np.array([t1, t2 + [0]], np.int32)
    add_sequence(kc, s1, tables[0]); add_sequence(vc, v1, tables[0])
    add_sequence(kc, s2, tables[1]); add_sequence(vc, v2, tables[1])
    q = encode(rng.standard_normal((2, hq, d)), "bf16")
    lens = np.array([L1, L2])
    shared_out = OA.paged_decode(q, kc, vc, tables, lens, 0.25, "bf16")
    # private copies: request 2's prefix moved to fresh blocks 6 and 7
    private = tables.copy()
    private[1, :2] = [6, 7]
    kc[6:8], vc[6:8] = kc[0:2], vc[0:2]
    priv_out = OA.paged_decode(q, kc, vc, private, lens, 0.25, "bf16")
    assert np.array_equal(shared_out, priv_out)


def pin_padding_never_read():
    rng = np.random.default_rng(12)
    lengths = [17, 30, 1]
    ks, vs, kc, vc, tables = random_case(rng, lengths, 4, 4, 8, "f32")
    q = encode(rng.standard_normal((3, 4, 8)), "f32")
    poisoned = OA.paged_decode(q, kc, vc, tables, np.array(lengths), 0.3, "f32")
    assert np.all(np.isfinite(poisoned))
    kc0, vc0 = np.nan_to_num(kc, nan=0.0), np.nan_to_num(vc, nan=0.0)
    clean = OA.paged_decode(q, kc0, vc0, tables, np.array(lengths), 0.3, "f32")
    assert np.array_equal(poisoned, clean)


def test_invariants():
    pin_permutation_invariance()
    pin_sharing_equals_private_copies()
    pin_padding_never_read()


def test_prefix_sharing_example_three_sharers():
    g = golden("block_sharing_examples.json")["prefix_example"]
    rng = np.random.default_rng(13)
    sysb, tails = g["system_prompt_blocks"], g["tails"]
    nb = 40
    hkv, d = 1, 8
    prefix_k = rng.standard_normal((len(sysb) * BS, hkv, d)).astype(np.float32)
    prefix_v = rng.standard_normal((len(sysb) * BS, hkv, d)).astype(np.float32)
    kc = np.full((nb, hkv, BS, d), np.nan, np.float32)
    vc = kc.copy()
    width = len(sysb) + max(len(t) for t in tails)
    tables = np.zeros((3, width), np.int32)
    lens = []
    for i, tail in enumerate(tails):
        row = sysb + tail
        L = len(row) * BS - i
        tables[i, :len(row)] = row
        lens.append(L)
        tk = rng.standard_normal((L - len(prefix_k), hkv, d)).astype(np.float32)
        tv = rng.standard_normal((L - len(prefix_k), hkv, d)).astype(np.float32)
        add_sequence(kc, np.concatenate([prefix_k, tk]), tables[i])
        add_sequence(vc, np.concatenate([prefix_v, tv]), tables[i])
    refs = np.bincount(tables[:, :len(sysb)].ravel(), minlength=nb)
    assert all(refs[b] == g["ref_count"] for b in sysb)
    q = rng.standard_normal((3, 2, d)).astype(np.float32)
    out = OA.paged_decode(q, kc, vc, tables, np.array(lens), 0.3, "f32")
    for i in range(3):
        k64 = OA.gather_sequence(kc, tables[i], lens[i]).astype(np.float64)
        v64 = OA.gather_sequence(vc, tables[i], lens[i]).astype(np.float64)
        assert np.array_equal(k64[:len(prefix_k)], prefix_k.astype(np.float64))
        ref = sdpa_ref(q[i:i + 1].astype(np.float64), k64, v64, 0.3)
        np.testing.assert_allclose(out[i], ref[0], rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# planted mistakes: every one must be caught by at least one pin
# --------------------------------------------------------------------------

ALL_PINS = [
    pin_block_table_example, pin_slot_placement, pin_prepare_inputs_positions,
    pin_bf16_decoding, pin_context_one_returns_v, pin_equal_values,
    pin_zero_query_gives_mean, pin_dominant_key, pin_two_keys_closed_form,
    pin_gqa_head_mapping, pin_decode_matches_contiguous, pin_varlen_matches_contiguous,
    pin_permutation_invariance, pin_sharing_equals_private_copies, pin_padding_never_read,
]


def _mut_kv_head_modulo(h, hq, hkv):
    return h % hkv


def _mut_positions_off_by_one(seq_len, q_len):
    return [seq_len - q_len + i - 1 for i in range(q_len)]


def _mut_positions_forward(seq_len, q_len):
    return [i for i in range(q_len)]


def _mut_slot_swapped(slot, block_size=BS):
    return slot % block_size, slot // block_size


def _mut_to_f64_shift(a, dtype):
    if dtype == "bf16":
        wide = a.astype(np.uint32) << np.uint32(15)
        return wide.view(np.float32).astype(np.float64)
    return np.asarray(a).astype(np.float64)


def _mut_no_scale(q_row, keys, values, scale):
    n = keys.shape[0]
    if n == 0:
        return np.zeros(values.shape[1])
    s = keys @ q_row
    w = np.exp(s - s.max())
    return (w / w.sum()) @ values


def _mut_values_are_keys(q_row, keys, values, scale):
    s = scale * (keys @ q_row)
    w = np.exp(s - s.max())
    return (w / w.sum()) @ keys


def _mut_sign(q_row, keys, values, scale):
    s = -scale * (keys @ q_row)
    w = np.exp(s - s.max())
    return (w / w.sum()) @ values


def _mut_unnormalised(q_row, keys, values, scale):
    s = scale * (keys @ q_row)
    return np.exp(s - s.max()) @ values


def _mut_gather_reads_padding(cache, table_row, length, block_size=BS):
    nlog = -(-length // block_size)
    rows = [cache[int(table_row[j])].transpose(1, 0, 2) for j in range(nlog)]
    # keeps the whole last block: the padding rows past ``length`` are attended to
    return np.concatenate(rows) if length else cache[:0, 0].transpose(1, 0, 2)


def _mut_gather_skips_block(cache, table_row, length, block_size=BS):
    hkv, d = cache.shape[1], cache.shape[3]
    out = np.empty((length, hkv, d), cache.dtype)
    for j in range(-(-length // block_size)):
        phys = int(table_row[j + 1 if j > 0 else 0])
        n = min(block_size, length - j * block_size)
        out[j * block_size:j * block_size + n] = cache[phys, :, :n, :].transpose(1, 0, 2)
    return out


def _mut_gather_offset_transposed(cache, table_row, length, block_size=BS):
    hkv, d = cache.shape[1], cache.shape[3]
    out = np.empty((length, hkv, d), cache.dtype)
    for j in range(-(-length // block_size)):
        phys = int(table_row[j])
        n = min(block_size, length - j * block_size)
        blk = cache[phys, :, ::-1, :][:, :n, :]
        out[j * block_size:j * block_size + n] = blk.transpose(1, 0, 2)
    return out


MUTATIONS = {
    "kv_head_of": _mut_kv_head_modulo,
    "query_positions/off_by_one": _mut_positions_off_by_one,
    "query_positions/forward": _mut_positions_forward,
    "slot_to_block_offset": _mut_slot_swapped,
    "to_f64": _mut_to_f64_shift,
    "softmax_attention/no_scale": _mut_no_scale,
    "softmax_attention/values_are_keys": _mut_values_are_keys,
    "softmax_attention/sign": _mut_sign,
    "softmax_attention/unnormalised": _mut_unnormalised,
    "gather_sequence/reads_padding": _mut_gather_reads_padding,
    "gather_sequence/skips_block": _mut_gather_skips_block,
    "gather_sequence/offset_reversed": _mut_gather_offset_transposed,
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    # Sanity: every pin passes on the unmodified oracle.
    for pin in ALL_PINS:
        pin()
    attr = name.split("/")[0]
    monkeypatch.setattr(OA, attr, MUTATIONS[name])
    caught = []
    for pin in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except Exception:      # an assertion, or a shape/index error the mistake causes
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
