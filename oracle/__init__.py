"""CPU oracle for the paged KV-cache decode path.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import anything from this package.  The product (the C-ABI
library under ``paged_kv_cache_342_b200``) never calls it and shares no code with
it; the two meet only in the seeded inputs from ``workloads``.

What it computes, written plainly and slowly from three pages about PagedAttention:

  [GLOSS] "PagedAttention", inferensys.com LLM-operations glossary.
  [BLOG]  "How PagedAttention Powers vLLM's KV Cache", hassanahmed.net.
  [LAB]   "PagedAttention", divagr.pages.dev attention-lab explainer.

* ``attention``  - single-query attention over a block-paged cache: gather each
  sequence's keys/values in logical order through its block table, then
  softmax(scale * K q) V in float64 ([BLOG] "The attention kernel has to read
  scattered blocks"; [LAB] "Keep pages in order", "Measure memory use across
  requests": paging leaves the attention equation unchanged).  Also the
  partitioned form (per-partition max / sum / output merged by log-sum-exp
  weights) that the GPU path uses for long sequences.
* ``cache_ops``  - writing a new token's K/V into its slot and copying whole
  blocks (the private copy of copy-on-write), as literal element copies.
* ``allocator``  - the block manager: shared free pool, per-sequence block
  tables, reference counts, fork (prefix sharing) and copy-on-write
  ([BLOG] "PagedAttention: paging, borrowed from the operating system",
  "The bonus contiguous storage can't give you: sharing"; [LAB] "Add pages as
  the request grows", "Share matching prefixes").
* ``waste``      - the slot-count arithmetic of the pages' worked examples.

Pins (checks against things other than the oracle itself) live in
``tests/test_oracle_pins.py`` and ``tests/golden/``.  Parity unpinned: the
prefix-sharing example's counts on [LAB] "Share matching prefixes" (its printed
values did not survive text extraction), so no pin uses them.
"""
