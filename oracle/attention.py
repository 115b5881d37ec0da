"""Paged single-query attention, float64 (oracle; test infrastructure only).

Sources (page title, section):
  [BLOG] "How PagedAttention Powers vLLM's KV Cache", section "The attention kernel
         has to read scattered blocks": the kernel walks the block table and gathers
         keys and values block by block.
  [BLOG] section "PagedAttention: paging, borrowed from the operating system": a
         block holds the keys and values of a fixed number of tokens; the block
         table maps each logical block of a sequence to a physical block.
  [LAB]  "PagedAttention" explainer, section "Keep pages in order": logical token
         order is preserved and the kernel locates each block through the table;
         sections "Measure memory use across requests" and "How it works": the
         attention equation itself does not change.
  [BLOG] section "Where it bites": grouped-query attention lets several query heads
         share one set of keys and values.

Readings taken where the pages are silent:
  * cache layout [num_blocks, num_kv_heads, block_size, head_dim] for K and V;
  * query head h uses kv head h // (num_heads // num_kv_heads) (consecutive groups);
  * the single decode query attends to all seq_len cached tokens (no mask), and a
    sequence of length 0 gives an all-zero output;
  * the partitioned form (split the tokens into fixed-size partitions, keep each
    partition's max, exp-sum and normalised output, merge with log-sum-exp weights)
    is the long-sequence split the GPU path uses; it reaches the same value.
"""
from __future__ import annotations

import numpy as np

from .numerics import to_f64


def gather_sequence(cache: np.ndarray, table_row, seq_len: int, block_size: int,
                    kv_head: int) -> np.ndarray:
    """Rows of one kv head of one sequence, in logical token order.

    Logical block j of the sequence holds tokens [j*bs, (j+1)*bs); it lives in
    physical block table_row[j].  Only the first seq_len tokens are taken, so only
    the last block may contribute fewer than bs rows.
    """
    pieces = []
    nblocks = (seq_len + block_size - 1) // block_size
    for j in range(nblocks):
        phys = int(table_row[j])
        take = min(block_size, seq_len - j * block_size)
        pieces.append(cache[phys, kv_head, :take, :])
    if not pieces:
        return cache[:0, 0, 0, :].copy()
    return np.concatenate(pieces, axis=0)


def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * K q) V for one query vector, float64, max-subtracted exp."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    logits = scale * (K @ q)
    p = np.exp(logits - logits.max())
    return (p @ V) / p.sum()


def paged_decode_attention(q, k_cache, v_cache, block_tables, seq_lens, scale,
                           block_size, num_kv_heads, dtype, seqs=None, heads=None):
    """Decode attention for every (sequence, query head), float64 [S, Hq, D].

    ``seqs`` / ``heads`` restrict the work to a sample (other rows stay NaN).
    """
    S, Hq, D = q.shape
    G = Hq // num_kv_heads
    out = np.full((S, Hq, D), np.nan, dtype=np.float64)
    seqs = range(S) if seqs is None else seqs
    heads = range(Hq) if heads is None else heads
    for s in seqs:
        L = int(seq_lens[s])
        by_kv = {}
        for h in heads:
            by_kv.setdefault(h // G, []).append(h)
        for g, hs in by_kv.items():
            K = to_f64(gather_sequence(k_cache, block_tables[s], L, block_size, g), dtype)
            V = to_f64(gather_sequence(v_cache, block_tables[s], L, block_size, g), dtype)
            for h in hs:
                out[s, h] = softmax_attention(to_f64(q[s, h], dtype), K, V, scale)
    return out


def partition_state(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """(max logit m, exp-sum l, normalised output o) of one partition."""
    logits = scale * (K @ q)
    m = logits.max()
    p = np.exp(logits - m)
    l = p.sum()
    return m, l, (p @ V) / l


def merge_partitions(states):
    """Log-sum-exp merge: M = max m_p, w_p = l_p e^(m_p - M), out = sum w_p o_p / sum w_p."""
    M = max(m for m, _, _ in states)
    w = [l * np.exp(m - M) for m, l, _ in states]
    num = sum(wp * o for wp, (_, _, o) in zip(w, states))
    return num / sum(w)


def partitioned_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float,
                          partition_size: int) -> np.ndarray:
    """Same value as ``softmax_attention`` via fixed-size partitions + merge."""
    L = K.shape[0]
    if L == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    states = [partition_state(q, K[a:a + partition_size], V[a:a + partition_size], scale)
              for a in range(0, L, partition_size)]
    return merge_partitions(states)
