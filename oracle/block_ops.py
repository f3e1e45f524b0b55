"""Whole-block operations on a paged KV pool: copy-on-write and swap.

TEST INFRASTRUCTURE ONLY (see the package header).  Plain Python loops over
the (src, dst) pairs; values are moved bit for bit in their stored encoding.

* Copy-on-write ([CORE] §核心抽象: a block's ref_cnt supports copy-on-write and
  sharing across requests; [ARCH] §4.3.2: parallel samples of one prompt share
  the prompt's blocks and then each appends blocks of its own): before a
  request writes into a block another request still references, it is given a
  private copy of that block.
* Swap ([ARCH] §1, the preemption table, v0 (Swap)): a preempted request's KV
  cache moves to CPU memory and back to the GPU pool when it resumes.

Both are: for each pair (src, dst), block ``dst`` of the destination pools
becomes block ``src`` of the source pools, in K and in V, for every KV head and
slot.  Pairs are independent (no dst is another pair's src or dst), so their
order does not matter.
"""

from __future__ import annotations

import numpy as np


def swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping):
    """Return copies of ``dst_k``/``dst_v`` ``[num_blocks, Hkv, block_size, D]``
    in which block ``dst`` holds block ``src`` of ``src_k``/``src_v`` for every
    row ``(src, dst)`` of ``block_mapping``.  The inputs are not modified."""
    k_out = np.array(dst_k, copy=True)
    v_out = np.array(dst_v, copy=True)
    for src, dst in np.asarray(block_mapping).reshape(-1, 2):
        k_out[int(dst)] = src_k[int(src)]
        v_out[int(dst)] = src_v[int(src)]
    return k_out, v_out


def copy_blocks(k_cache, v_cache, block_mapping):
    """Copy-on-write inside one pool: ``swap_blocks`` with the pool as both the
    source and the destination (sources are read from the pool as it was
    before the call, which independent pairs make equivalent to any order)."""
    return swap_blocks(k_cache, v_cache, k_cache, v_cache, block_mapping)
