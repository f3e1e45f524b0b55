"""fp64 CPU oracle for paged KV-cache attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.  It
shares no code with the CUDA library: it is the plain definition of what the
hot path computes, written out step by step in float64 so a reader can check
it against the pages by eye.

Pages it follows (cited by title and section everywhere in this package):

* [CORE]  "2. 核心思想" -- the vLLM core-ideas page
  (ai-infra.cypggs.com, 04-llmops/vllm/02-core-ideas).
* [DEEP]  "vLLM 深度拆解：当 KV Cache 学会「分页」——用操作系统智慧重写 LLM
  推理的心智模型" (chenxutan.com/d/4801.html).
* [ARCH]  "vLLM 架构源码解析 | 第 1 篇：从 API 到 token 生成"
  (wazhb.com, 2026-07-06, vllm-architecture-api-to-token-generation).

Every function is pinned by ``tests/test_oracle_pins.py`` against something
other than itself (closed forms, invariants the pages fix, the pages' worked
examples, and ``torch.nn.functional.scaled_dot_product_attention`` in float64
for the contiguous special case).  No function here is "parity unpinned".
"""

from .paged_attention import (  # noqa: F401
    BLOCK_SIZE,
    to_f64,
    slot_to_block_offset,
    reshape_and_cache,
    gather_sequence,
    kv_head_of,
    query_positions,
    softmax_attention,
    paged_decode,
    paged_varlen,
)
from .block_ops import copy_blocks, swap_blocks  # noqa: F401,E402
from .fp8 import (  # noqa: F401,E402
    E4M3_MAX, e4m3_decode, e4m3_encode, dequantize, reshape_and_cache_fp8, paged_decode_fp8,
    paged_varlen_fp8,
)
from .rope import rope_table, rotate, rope_reshape_and_cache  # noqa: F401,E402
