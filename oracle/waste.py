"""Slot-count arithmetic of the pages' worked examples (oracle; test infrastructure only).

Sources (page title, section):
  [LAB] "PagedAttention" explainer (divagr.pages.dev/attention-lab/paged):
    "Reserved space can go unused" - a fixed contiguous reservation of which only
      part is used; the rest is wasted.
    "Add pages as the request grows" - pages of a fixed number of slots, a new page
      only when the current one is full.
    "Measure memory use across requests" - a batch compared under a fixed
      per-request contiguous reservation and under paging.
  [BLOG] "How PagedAttention Powers vLLM's KV Cache", "PagedAttention: paging,
    borrowed from the operating system" - the only waste left is the last, partly
    filled block of each sequence.

The paged counts come from running the block manager model, not from a formula.
"""
from __future__ import annotations

from .allocator import BlockManager


def contiguous_reservation(used: int, reserved: int) -> dict:
    empty = reserved - used
    return dict(used=used, reserved=reserved, empty=empty, wasted_fraction=empty / reserved)


def paged_growth(n_tokens: int, block_size: int) -> dict:
    """Grow one request token by token; report pages, slots and empty slots."""
    pool = max(1, n_tokens)  # one block per token is always enough
    bm = BlockManager(pool, block_size)
    bm.add(0, 0)
    for _ in range(n_tokens):
        bm.append_slot(0)
    pages = len(bm.tables[0])
    return dict(tokens=n_tokens, pages=pages, slots=pages * block_size,
                empty_slots=pages * block_size - n_tokens,
                logical_pages=list(range(pages)))


def batch_memory(lengths, block_size: int, reservation: int) -> dict:
    """Contiguous reservations vs paged allocation for a batch of requests."""
    pool = sum(lengths)  # one block per token is always enough
    bm = BlockManager(pool, block_size)
    for i, n in enumerate(lengths):
        bm.add(i, n)
    st = bm.stats()
    contiguous = len(lengths) * reservation
    return dict(contiguous_slots=contiguous, paged_slots=st["allocated_slots"],
                stored_tokens=st["logical_tokens"],
                blocks=[len(bm.tables[i]) for i in range(len(lengths))],
                saving_fraction=1.0 - st["allocated_slots"] / contiguous,
                paged_waste_fraction=st["tail_waste_slots"] / st["allocated_slots"])
