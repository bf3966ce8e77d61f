"""Host-side block arithmetic of the paged KV cache.

The vLLM case-study page ("vLLM 与 PagedAttention", section 二) and the
``PagedKVCache`` sketch on the 298.name page ("PagedAttention怎么解决") fix the
data model: a sequence of n tokens occupies ceil(n / block_size) fixed-size
blocks, and its block table maps logical block i to a physical block id.  A
token at position ``pos`` therefore lives in physical slot
``block_table[pos // block_size] * block_size + pos % block_size`` of the pool
laid out as ``[num_blocks, block_size, num_kv_heads, head_dim]``.

This is the host's share of the path: it turns block tables and positions
into the ``slot_mapping`` that ``reshape_and_cache`` consumes.  All device
work happens in the CUDA library.
"""
from __future__ import annotations

import numpy as np


def blocks_needed(num_tokens, block_size: int):
    """ceil(num_tokens / block_size), element-wise for arrays."""
    n = np.asarray(num_tokens, dtype=np.int64)
    out = (n + block_size - 1) // block_size
    return int(out) if out.ndim == 0 else out


def slot_mapping(block_tables: np.ndarray, seq_ids, positions, block_size: int) -> np.ndarray:
    """Physical slot of token ``positions[t]`` of sequence ``seq_ids[t]``.

    ``block_tables`` is ``[num_seqs, max_blocks_per_seq]`` int32.  Returns
    int64 slots; raises if a position falls outside its table row.
    """
    bt = np.asarray(block_tables)
    s = np.asarray(seq_ids, dtype=np.int64)
    pos = np.asarray(positions, dtype=np.int64)
    logical = pos // block_size
    if np.any(pos < 0) or np.any(logical >= bt.shape[1]):
        raise ValueError("position outside the block table")
    physical = bt[s, logical].astype(np.int64)
    if np.any(physical < 0):
        raise ValueError("position maps to an unassigned logical block")
    return physical * block_size + pos % block_size
