"""One decode step of the whole path, on the CPU (oracle; test infrastructure only).

The order of a step (sources as in the sibling modules):
  1. every sequence gets room for one more token (block manager append; a new
     block when the last one is full, a private copy when it is shared);
  2. the private copies are made (copy-on-write) - before the write, because the
     new token goes into the copy;
  3. the new token's K/V is written into its slot;
  4. decode attention over all cached tokens, new one included.

Context for the shared-prefix workload: each group's first sample is admitted
with the prefix, the other samples fork from it (sharing every prefix block), then
sample by sample, in index order, the private tokens are appended.  Their K/V is
whatever the seeded pool fill holds in their slots; the copy-on-write copies made
on the way are applied to the cache.
"""
from __future__ import annotations

import numpy as np

from .allocator import BlockManager
from .attention import paged_decode_attention
from .cache_ops import copy_blocks, reshape_and_cache


def build_context(inp, copy_pool: bool = True):
    """Block manager + caches holding every sequence's context (before the step)."""
    cfg = inp.cfg
    bm = BlockManager(cfg.num_blocks, cfg.block_size, inp.free_order)
    k = inp.k_pool.copy() if copy_pool else inp.k_pool
    v = inp.v_pool.copy() if copy_pool else inp.v_pool
    build_pairs = []
    if inp.prefix is None:
        for s in range(cfg.num_seqs):
            bm.add(s, int(inp.context_lens[s]))
    else:
        p = inp.prefix
        for g in range(p.groups):
            parent = g * p.samples
            bm.add(parent, p.prefix_len)
            for i in range(1, p.samples):
                bm.fork(parent, parent + i)
        for s in range(cfg.num_seqs):
            for _ in range(int(p.private_lens[s])):
                _, src, dst = bm.append_slot(s)
                if src >= 0:
                    build_pairs.append((src, dst))
        if build_pairs and k.size:
            copy_blocks(k, v, build_pairs)
    return bm, k, v, build_pairs


def decode_step(bm: BlockManager, k, v, inp, max_blocks: int, q=None, new_k=None,
                new_v=None, seqs=None, heads=None, attend: bool = True):
    """Run steps 1-4 in place on (bm, k, v); returns a dict of everything produced."""
    cfg = inp.cfg
    q = inp.q if q is None else q
    new_k = inp.new_k if new_k is None else new_k
    new_v = inp.new_v if new_v is None else new_v
    ids = list(range(cfg.num_seqs))
    res = bm.append_slots(ids)
    slots = np.array([r[0] for r in res], dtype=np.int64)
    pairs = np.array([(r[1], r[2]) for r in res if r[1] >= 0], dtype=np.int32).reshape(-1, 2)
    if k.size:
        copy_blocks(k, v, pairs)
        reshape_and_cache(new_k, new_v, k, v, slots, cfg.block_size)
    rows, lens = bm.block_tables(ids, max_blocks)
    tables = np.array(rows, dtype=np.int32).reshape(cfg.num_seqs, max_blocks)
    seq_lens = np.array(lens, dtype=np.int32)
    out = None
    if attend:
        out = paged_decode_attention(q, k, v, tables, seq_lens, cfg.scale, cfg.block_size,
                                     cfg.num_kv_heads, cfg.dtype, seqs=seqs, heads=heads)
    return dict(slots=slots, pairs=pairs, tables=tables, seq_lens=seq_lens, out=out)
