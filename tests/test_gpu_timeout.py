"""Bounded waits: a load that never lands ends in PA_ERR_TIMEOUT, not a hang.

Every wait inside the kernels gives up after a limit, records PA_ERR_TIMEOUT
and lets its CTA leave (the copies it already issued land first; the chunk
kernel frees its tensor memory).  The test hook pa_debug_lost_load makes
every CTA of one kernel leave its first K/V tile unissued -- nothing is in flight
for it, and nothing ever arrives -- with the limit lowered to about a
millisecond.  The call must come back, pa_get_device_error must report the
timeout, and the next call, with the hook off, must match the oracle: the
context and the library are still usable.
"""

import pytest

import pagedattention_paged_kv_reshape_b200 as pa
from pagedattention_paged_kv_reshape_b200 import workload as W
from tests._helpers import assert_close, gpu_attention, gpu_cache_write, oracle_step

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("kernel", [1, 2], ids=["attn_mma_kernel", "chunk_tc2_kernel"])
def test_lost_load_times_out_and_next_call_is_clean(kernel):
    if kernel == 1:   # decode rows: the TMA + mma.sync attention kernel
        b = W.build_batch([W.Request(L) for L in (700, 40, 1500)], num_q_heads=32,
                          num_kv_heads=8, head_dim=128, dtype="bf16", seed=81, device=DEV,
                          pool_factor=1.3)
    else:             # a causal chunk row: the tcgen05 chunk kernel
        b = W.build_batch([W.Request(s, q) for s, q in [(900, 300), (64, 1)]], num_q_heads=32,
                          num_kv_heads=8, head_dim=128, dtype="bf16", seed=82, device=DEV,
                          pool_factor=1.3)
    kc, vc = gpu_cache_write(b)
    pa.pa_get_device_error()
    pa.pa_debug_lost_load(kernel)
    try:
        with pytest.raises(pa.PaError) as e:
            gpu_attention(b, kc, vc)        # synchronises and reads the error word
        assert e.value.status == pa.Status.TIMEOUT, str(e.value)
    finally:
        pa.pa_debug_lost_load(0)
    pa.pa_get_device_error()                # the word was cleared
    out = gpu_attention(b, kc, vc)
    ref, _, _ = oracle_step(b)
    assert_close(out, ref, "bf16", f"call after the timeout (kernel {kernel})")
