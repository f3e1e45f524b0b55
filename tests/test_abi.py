"""The C-ABI library: it loads, exports every symbol include/pa.h declares, and
rejects bad arguments on the host before any launch.  CPU only: no call here
reaches a kernel (every argument-error case fails host validation first, and
the cases that pass validation are empty batches, which launch nothing)."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

import pagedattention_paged_kv_reshape_b200 as pa
from pagedattention_paged_kv_reshape_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")

# Host-validation tests pass dummy (never dereferenced) addresses.  They only
# run where no GPU exists, so a validation bug can never turn into a launch.
cpu_only = pytest.mark.skipif(torch.cuda.is_available(), reason="host-validation tests run on CPU")

FAKE = 0x100000  # 1 MiB: 256-byte aligned, never dereferenced


@pytest.fixture(scope="module")
def lib():
    pa_build.build(quiet=True)
    return pa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("pa_reshape_and_cache", "pa_decode", "pa_decode_workspace_size", "pa_varlen",
                 "pa_varlen_workspace_size", "pa_get_device_error", "pa_status_string"):
        assert must in names


def _header_enum(prefix):
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return {m.group(1): int(m.group(2))
            for m in re.finditer(r"\b(" + prefix + r"[A-Z0-9_]*)\s*=\s*(\d+)", text)}


def test_binding_enums_mirror_the_header():
    """The Python enums carry the header's values, so a new path or status
    cannot drift between the C ABI and the binding."""
    paths = _header_enum("PA_PATH_")
    assert paths == {"PA_PATH_" + p.name: int(p) for p in pa.Path}
    statuses = _header_enum("PA_(?:OK|ERR_)")
    assert statuses == {("PA_OK" if s.name == "OK" else "PA_ERR_" + s.name): int(s)
                        for s in pa.Status}


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from libpa.so"
    nm = subprocess.run(["nm", "-D", "--defined-only", pa.LIBRARY_PATH], capture_output=True,
                        text=True)
    if nm.returncode == 0:
        exported = set(re.findall(r"\bT (pa_[a-z_]+)\b", nm.stdout))
        assert set(declared_functions()) <= exported


def test_build_targets_sm100a():
    """The build compiles for sm_100a only (no PTX or other architectures)."""
    flags = pa_build.NVCC_FLAGS
    i = flags.index("-gencode")
    assert flags[i + 1] == "arch=compute_100a,code=sm_100a"
    assert flags.count("-gencode") == 1


@pytest.mark.gpu
def test_loaded_kernels_are_sm100_code(lib):
    """The CUDA runtime reports the library's kernels as sm_100 code on this device."""
    assert pa.pa_binary_version() == 100


def test_version_and_status_strings(lib):
    assert pa.pa_version() == 100
    for st in pa.Status:
        assert pa.pa_status_string(st) == "PA_" + ("OK" if st.name == "OK" else "ERR_" + st.name)


def test_set_path_roundtrip(lib):
    prev = pa.pa_set_path(pa.Path.SIMT)
    assert pa.pa_set_path(prev) == pa.Path.SIMT


def _a256(x):
    return (x + 255) // 256 * 256


def _layout(S, T, hq, hkv, d, max_len, varlen):
    """Mirror of the workspace layout documented in csrc/pa_api.cu."""
    g = hq // hkv
    ns = -(-g // 16)
    p = -(-max_len // 512) if max_len > 0 else 1
    off = _a256(16 + 2 * (S + 1) * 4)                 # schedule block + two row prefixes
    gs = min(g, 16)
    if varlen and gs in (1, 2, 4, 8, 16):             # tcgen05 chunk-tile list, int2 entries
        qt = 128 // gs
        off = _a256(off + (2 * -(-T // qt) + 1) * 8)
    if p > 1:
        off = _a256(off + T * hq * p * 4)             # partial log-sum-exp
        off = _a256(off + T * hq * p * d * 4)         # partial outputs
    return off


def test_workspace_sizes(lib):
    assert pa.pa_decode_workspace_size(64, 32, 32, 128, 512) == _layout(64, 64, 32, 32, 128, 512,
                                                                        False)
    assert pa.pa_decode_workspace_size(8, 64, 8, 128, 32768) == _layout(8, 8, 64, 8, 128, 32768,
                                                                        False)
    assert pa.pa_decode_workspace_size(0, 32, 8, 128, 100) == 0
    assert pa.pa_varlen_workspace_size(3, 10, 4, 2, 64, 8, 1024) == _layout(3, 10, 4, 2, 64, 1024,
                                                                            True)
    # the split-K partials dominate: [T][Hq][P] lse + [T][Hq][P][D] outputs
    big = pa.pa_decode_workspace_size(8, 64, 8, 128, 32768)
    assert big >= 8 * 64 * 64 * 129 * 4


def _decode(lib, **kw):
    args = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, stride=4, cl=FAKE, S=2, hq=8, hkv=2,
                d=128, bs=16, nb=10, maxc=64, scale=0.1, ws=FAKE, wsb=1 << 20, dt=1)
    args.update(kw)
    return lib.pa_decode(args["out"], args["q"], args["k"], args["v"], args["bt"], args["stride"],
                         args["cl"], args["S"], args["hq"], args["hkv"], args["d"], args["bs"],
                         args["nb"], args["maxc"], args["scale"], args["ws"], args["wsb"],
                         args["dt"], None)


@cpu_only
@pytest.mark.parametrize("kw,status", [
    (dict(out=None), pa.Status.INVALID_ARG),
    (dict(q=FAKE + 8), pa.Status.INVALID_ARG),         # misaligned
    (dict(hq=6, hkv=4), pa.Status.INVALID_ARG),        # Hq % Hkv != 0
    (dict(hkv=0), pa.Status.INVALID_ARG),
    (dict(d=96), pa.Status.UNSUPPORTED),
    (dict(d=512), pa.Status.UNSUPPORTED),
    (dict(bs=24), pa.Status.UNSUPPORTED),
    (dict(bs=64), pa.Status.UNSUPPORTED),
    (dict(dt=7), pa.Status.INVALID_ARG),
    (dict(S=-1), pa.Status.INVALID_ARG),
    (dict(scale=float("nan")), pa.Status.INVALID_ARG),
    (dict(ws=None), pa.Status.WORKSPACE),
    (dict(ws=FAKE + 16), pa.Status.WORKSPACE),         # not 256-byte aligned
    (dict(maxc=4096, wsb=64), pa.Status.WORKSPACE),    # too small for split-K partials
    (dict(nb=0), pa.Status.INVALID_ARG),
    (dict(bt=None), pa.Status.INVALID_ARG),
])
def test_decode_rejects_bad_arguments(lib, kw, status):
    assert _decode(lib, **kw) == status
    assert lib.pa_last_error_message()


@cpu_only
def test_empty_batches_launch_nothing(lib):
    assert _decode(lib, S=0) == pa.Status.OK
    assert lib.pa_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 8, 128, 16, 10, 1, None) == 0
    assert lib.pa_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, 4, FAKE, FAKE, 3, 0, 0, 64, 8, 2, 128, 16,
                         10, 0.1, FAKE, 1 << 20, 1, None) == 0


@cpu_only
@pytest.mark.parametrize("args,status", [
    ((None, FAKE, FAKE, FAKE, FAKE, 4, 8, 128, 16, 10, 1), pa.Status.INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, None, 4, 8, 128, 16, 10, 1), pa.Status.INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 80, 16, 10, 1), pa.Status.UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 128, 12, 10, 1), pa.Status.UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 128, 64, 10, 1), pa.Status.UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, -1, 8, 128, 16, 10, 1), pa.Status.INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 128, 16, 10, 9), pa.Status.INVALID_ARG),
])
def test_reshape_rejects_bad_arguments(lib, args, status):
    assert lib.pa_reshape_and_cache(*args, None) == status


@cpu_only
def test_varlen_rejects_bad_arguments(lib):
    base = [FAKE, FAKE, FAKE, FAKE, FAKE, 4, FAKE, FAKE, 3, 10, 8, 64, 8, 2, 128, 16, 10, 0.1,
            FAKE, 1 << 20, 1, None]
    bad_qsl = list(base)
    bad_qsl[6] = None
    assert lib.pa_varlen(*bad_qsl) == pa.Status.INVALID_ARG
    small_ws = list(base)
    small_ws[11] = 4096   # max_seq_len: 8 partitions of split-K partials
    need = pa.pa_varlen_workspace_size(3, 10, 8, 2, 128, 8, 4096)
    small_ws[19] = need - 1
    assert lib.pa_varlen(*small_ws) == pa.Status.WORKSPACE
    tf32 = list(base)
    tf32[20] = 0
    prev = pa.pa_set_path(pa.Path.MMA)
    try:
        assert lib.pa_varlen(*tf32) == pa.Status.UNSUPPORTED   # tensor-core path needs 16-bit
    finally:
        pa.pa_set_path(prev)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from pagedattention_paged_kv_reshape_b200 import _binding
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "LIBRARY_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _binding.lib()


@cpu_only
def test_block_ops_reject_bad_arguments(lib):
    # pa_copy_blocks(k, v, map, num_pairs, Hkv, D, block_size, num_blocks, dtype, stream)
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, 0, 8, 128, 16, 10, 1, None) == pa.Status.OK
    assert lib.pa_copy_blocks(None, FAKE, FAKE, 3, 8, 128, 16, 10, 1, None) == \
        pa.Status.INVALID_ARG
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, 3, 8, 80, 16, 10, 1, None) == \
        pa.Status.UNSUPPORTED
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, -1, 8, 128, 16, 10, 1, None) == \
        pa.Status.INVALID_ARG
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, 3, 8, 128, 16, 10, 7, None) == \
        pa.Status.INVALID_ARG
    # pa_swap_blocks(src_k, src_v, dst_k, dst_v, map, n, Hkv, D, bs, src_nb, dst_nb, dtype, s)
    assert lib.pa_swap_blocks(FAKE, FAKE, FAKE, None, FAKE, 3, 8, 128, 16, 10, 10, 1, None) == \
        pa.Status.INVALID_ARG
    assert lib.pa_swap_blocks(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 8, 128, 16, 10, 10, 1, None) == \
        pa.Status.OK
