"""pa_decode_static: decode attention for callers that cannot allocate device memory.

Some callers only ever hold their input and output buffers -- a plugin inside a
host runtime that owns every device allocation, or a hot loop that must not
call cudaMalloc because it can synchronise the device.  pa_decode_static gives
them pa_decode with its split-K scratch taken from a fixed 32 MiB array built
into the library.  This file checks it through the C ABI against pa_decode
with a caller-provided workspace and against the fp64 oracle, on calls in a
row (the later calls find the earlier calls' leftovers in the shared array,
once with the same shape and once with another).  It is collected last so that
a run stopping at the first failure has already run every other test.
"""

import numpy as np
import pytest
import torch

import pagedattention_paged_kv_reshape_b200 as pa
from pagedattention_paged_kv_reshape_b200 import workload as W
from tests._helpers import TOL, assert_close, f64, gpu_attention, gpu_cache_write, oracle_step

pytestmark = pytest.mark.gpu
DEV = "cuda"
CODES = {"f32": 0, "bf16": 1, "f16": 2}


def call_static(b, kc, vc, out, max_context_len=None):
    """Call the C entry point directly (no binding logic in between)."""
    return pa.lib().pa_decode_static(
        out.data_ptr(), b.q.data_ptr(), kc.data_ptr(), vc.data_ptr(), b.block_tables.data_ptr(),
        b.block_tables.shape[1], b.seq_lens.data_ptr(), b.num_seqs, b.num_q_heads,
        b.num_kv_heads, b.head_dim, b.block_size, b.num_blocks,
        b.max_seq_len if max_context_len is None else max_context_len, b.scale,
        CODES[b.dtype], torch.cuda.current_stream().cuda_stream)


def check_static(b, kc, vc):
    """pa_decode_static against pa_decode with a workspace (within the bf16/f16
    tolerance) and against the fp64 oracle."""
    need = pa.pa_decode_workspace_size(b.num_seqs, b.num_q_heads, b.num_kv_heads, b.head_dim,
                                       b.max_seq_len)
    assert 0 < need <= pa.STATIC_WORKSPACE_BYTES
    ref = gpu_attention(b, kc, vc)                 # pa_decode with a workspace
    out = torch.full_like(b.q, float("nan"))
    assert call_static(b, kc, vc, out) == 0
    pa.pa_get_device_error()
    got, want = f64(out), f64(ref)
    assert np.all(np.isfinite(got))
    err = np.abs(got - want)
    max_tol, mean_tol = TOL[b.dtype]
    assert err.max() <= max_tol and err.mean() <= mean_tol, (err.max(), err.mean())
    oracle, _, _ = oracle_step(b)
    assert_close(out, oracle, b.dtype, "pa_decode_static vs the oracle")


def test_static_scratch_matches_workspace_decode_on_two_calls():
    """Two calls of one shape with different inputs (the second reads a layout
    the first left full of its own partials), then a call of another shape."""
    def gqa(seed):
        # GQA 4, contexts spanning up to six 512-token partitions (split-K reduce)
        return W.build_batch([W.Request(L) for L in (1, 700, 1500, 3000)], num_q_heads=32,
                             num_kv_heads=8, head_dim=128, dtype="bf16", seed=seed, device=DEV,
                             pool_factor=1.3)
    batches = [
        gqa(7),
        gqa(17),
        # a different shape: MHA, head_dim 64, f16
        W.build_batch([W.Request(L) for L in (2048, 513, 9)], num_q_heads=8, num_kv_heads=8,
                      head_dim=64, dtype="f16", seed=8, device=DEV, pool_factor=1.3),
    ]
    for b in batches:
        kc, vc = gpu_cache_write(b)
        check_static(b, kc, vc)


def test_static_scratch_rejects_sizes_beyond_its_maximum():
    # 256 requests x 32 heads x 16 partitions of partials need ~68 MB > 32 MiB.
    # The tensors are real and consistent, so even a launch would stay in bounds.
    b = W.build_batch([W.Request(1) for _ in range(256)], num_q_heads=32, num_kv_heads=8,
                      head_dim=128, dtype="bf16", seed=9, device=DEV)
    out = torch.zeros_like(b.q)
    st = call_static(b, b.k_cache, b.v_cache, out, max_context_len=8192)
    assert st == pa.Status.WORKSPACE
    assert b"32 MiB" in pa.lib().pa_last_error_message() or \
        str(pa.STATIC_WORKSPACE_BYTES).encode() in pa.lib().pa_last_error_message()
    assert torch.all(out == 0)
