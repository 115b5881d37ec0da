"""Cache maintenance ops as literal copies (oracle; test infrastructure only).

Sources (page title, section):
  [BLOG] "How PagedAttention Powers vLLM's KV Cache", "Quick recap: the KV cache is
         per token, and it grows": every generated token adds a key and a value.
  [BLOG] "The bonus contiguous storage can't give you: sharing" and [LAB]
         "PagedAttention" explainer, "Share matching prefixes": before a sequence
         writes into a shared block it gets a private copy of that block.

Layout reading: caches are [num_blocks, num_kv_heads, block_size, head_dim]; a slot
number s names block s // block_size, offset s % block_size; slot -1 means "no
write" (padding).  Values are copied as stored bits (no dtype conversion).
"""
from __future__ import annotations

import numpy as np


def reshape_and_cache(key: np.ndarray, value: np.ndarray, k_cache: np.ndarray,
                      v_cache: np.ndarray, slot_mapping, block_size: int) -> None:
    """In place: token t's [num_kv_heads, head_dim] rows go to slot slot_mapping[t]."""
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        blk, off = divmod(int(slot), block_size)
        for h in range(key.shape[1]):
            k_cache[blk, h, off, :] = key[t, h, :]
            v_cache[blk, h, off, :] = value[t, h, :]


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, block_mapping) -> None:
    """In place, in pair order: block dst becomes a copy of block src (all heads)."""
    for src, dst in np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2):
        k_cache[dst] = k_cache[src]
        v_cache[dst] = v_cache[src]
