"""One decode step of the paged KV-cache path, driven through the C ABI.

Order of a step (the sources are the pages cited in ``include/pa.h``):
  1. the block manager gives every sequence room for one more token
     (``pa_seq_append_slots``): a slot, and a (src, dst) copy where the token's
     block is shared;
  2. slots, copy pairs, lengths and block tables are packed into one pinned staging
     buffer and sent to the device in one copy (the only host-to-device traffic of
     a step);
  3. ``pa_copy_blocks`` makes the copy-on-write copies - before the write, since
     the new token lands in the copy;
  4. ``pa_reshape_and_cache`` writes the new token's K/V into its slot;
  5. ``pa_decode_attention`` attends over every cached token, the new one included.

With ``rolling=True`` each step first rolls the sequences back to the lengths they
had when bound (``pa_seq_truncate``): every step then decodes the same lengths,
which is how a long benchmark run stays on one workload.

Sequences that share leading blocks (forks of one prompt) are found each step by
``pa_build_prefix_groups``; their shared partitions are then read once per group
(``pa_decode_attention_grouped``).  ``group_members`` caps a chunk (default: as many
members as fill one 8-column tensor-core tile, 8 // (num_heads/num_kv_heads); 0
turns grouping off).

One-byte caches (uint8 / float8_e4m3fn tensors) are fp8 e4m3 caches with the
per-tensor ``kv_scales`` (k_scale, v_scale): the step writes with
``pa_reshape_and_cache_fp8`` and attends with ``pa_decode_attention_fp8``.

This module only moves arguments: the work of every step is done by the library.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (DEFAULT_PARTITION, BlockAllocator, _dtype_code, pa_copy_blocks,
               pa_decode_attention, pa_decode_attention_fp8, pa_decode_attention_grouped,
               pa_decode_partition_size, pa_decode_workspace_bytes, pa_reshape_and_cache,
               pa_reshape_and_cache_fp8)


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


class PagedDecoder:
    """Device caches + block manager + staging for a fixed batch of sequences.

    ``k_cache``/``v_cache`` are caller-owned CUDA tensors [NB, Hkv, bs, D].
    ``max_blocks_per_seq`` is the block-table width (capacity per sequence).
    ``partition_size`` 0 takes ``pa_decode_partition_size`` for the bound batch at
    that capacity (resolved by ``bind``; it ignores prefix groups, so batches of
    forks do better with an explicit size shorter than their shared prefix).
    """

    def __init__(self, k_cache, v_cache, num_heads: int, scale: float, max_blocks_per_seq: int,
                 free_order=None, partition_size: int = DEFAULT_PARTITION, stream=None,
                 group_members: int | None = None, kv_scales=None):
        self.k_cache, self.v_cache = k_cache, v_cache
        self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim = k_cache.shape
        self.num_heads, self.scale = num_heads, scale
        self.max_blocks = max_blocks_per_seq
        self._partition_arg = partition_size
        self.partition_size = partition_size or DEFAULT_PARTITION
        self.device = k_cache.device
        self.stream = stream
        self.alloc = BlockAllocator(self.num_blocks, self.block_size, free_order)
        self._seq_ids = None
        self._ws = torch.empty(0, dtype=torch.uint8, device=self.device)
        group = num_heads // self.num_kv_heads
        self.fp8 = k_cache.element_size() == 1
        if self.fp8 and kv_scales is None:
            raise ValueError("an fp8 cache needs kv_scales=(k_scale, v_scale)")
        self.kv_scales = kv_scales
        self.group_members = (8 // group if group <= 8 else 0) if group_members is None \
            else group_members
        if self.fp8:
            self.group_members = 0

    # -- context building ------------------------------------------------------
    def admit(self, seq_id: int, num_tokens: int) -> None:
        self.alloc.add(seq_id, num_tokens)

    def admit_shared_prefix(self, groups: int, samples: int, prefix_len: int, private_lens,
                            first_id: int = 0) -> np.ndarray:
        """Groups of ``samples`` sequences sharing a prefix: the group's first sample is
        admitted with the prefix, the others fork from it; then, sample by sample, the
        private tokens are appended.  Returns the copy-on-write pairs those appends
        produced (apply them with ``apply_copies`` before reading the cache)."""
        pairs = []
        for g in range(groups):
            parent = first_id + g * samples
            self.alloc.add(parent, prefix_len)
            for i in range(1, samples):
                self.alloc.fork(parent, parent + i)
        for i, n in enumerate(np.asarray(private_lens, dtype=np.int64)):
            sid = first_id + i
            for _ in range(int(n)):
                _, src, dst = self.alloc.append_slot(sid)
                if src >= 0:
                    pairs.append((src, dst))
        return np.array(pairs, dtype=np.int32).reshape(-1, 2)

    def apply_copies(self, pairs: np.ndarray) -> None:
        if len(pairs):
            dev = torch.from_numpy(np.ascontiguousarray(pairs)).to(self.device)
            pa_copy_blocks(self.k_cache, self.v_cache, dev, pairs, stream=self._torch_stream())

    # -- the step ---------------------------------------------------------------
    def bind(self, seq_ids, rolling: bool = False) -> None:
        """Fix the batch the steps run over and allocate the staging buffers."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        self._seq_ids = ids
        self.rolling = rolling
        self._stepped = False
        self.base_lens = np.array([self.alloc.seq_len(int(s)) for s in ids], np.int64)
        S, MB, MM = ids.size, self.max_blocks, max(1, self.group_members)
        S1 = max(S, 1)
        sizes = [("slots", 8 * S), ("pairs", 8 * S1), ("lens", 4 * S), ("tables", 4 * S * MB),
                 ("pparts", 4 * S1), ("cmembers", 4 * S1 * MM), ("cparts", 4 * S1)]
        offs, total = {}, 0
        for name, n in sizes:
            offs[name] = total
            total += _align(n)
        # two staging sets: step k fills set k % 2 while step k - 1's kernels still
        # read the other one; the copy runs on its own stream
        self._h_bufs = [torch.empty(total, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
        self._d_bufs = [torch.empty(total, dtype=torch.uint8, device=self.device)
                        for _ in range(2)]
        self._copy_stream = torch.cuda.Stream(device=self.device)
        self._h2d_done = [None, None]       # the set's host buffer may be rewritten
        self._kernels_done = [None, None]   # the set's device buffer may be overwritten
        self._set = 1

        def views(buf):
            def sec(name, n, dt):
                return buf[offs[name]:offs[name] + n].view(dt)
            return dict(
                slots=sec("slots", 8 * S, torch.int64),
                pairs=sec("pairs", 8 * S1, torch.int32).view(-1, 2),
                lens=sec("lens", 4 * S, torch.int32),
                tables=sec("tables", 4 * S * MB, torch.int32).view(S, MB),
                pparts=sec("pparts", 4 * S1, torch.int32),
                cmembers=sec("cmembers", 4 * S1 * MM, torch.int32).view(S1, MM),
                cparts=sec("cparts", 4 * S1, torch.int32))

        self._views = [(views(self._h_bufs[i]), views(self._d_bufs[i])) for i in range(2)]
        self._use_set(0)
        cap = MB * self.block_size
        if self._partition_arg == 0:
            ps = pa_decode_partition_size(_dtype_code(self.k_cache), S, self.num_heads, self.num_kv_heads,
                                          self.head_dim, self.block_size, cap)
            if ps <= 0:
                raise RuntimeError("pa_decode_partition_size rejected the bound batch")
            self.partition_size = ps
        ws = pa_decode_workspace_bytes(S, self.num_heads, self.head_dim, cap, self.partition_size)
        if ws > self._ws.numel():
            self._ws = torch.empty(ws, dtype=torch.uint8, device=self.device)

    def _use_set(self, i: int) -> None:
        """Point the h_* / d_* views at staging set i."""
        self._set = i
        h, d = self._views[i]
        self.h_stage, self.d_stage = self._h_bufs[i], self._d_bufs[i]
        self.h_slots, self.h_pairs, self.h_lens, self.h_tables = (h["slots"], h["pairs"],
                                                                  h["lens"], h["tables"])
        self.d_slots, self.d_pairs, self.d_lens, self.d_tables = (d["slots"], d["pairs"],
                                                                  d["lens"], d["tables"])
        self.h_groups = (h["pparts"], h["cmembers"], h["cparts"])
        self.d_groups = (d["pparts"], d["cmembers"], d["cparts"])

    @property
    def staging_bytes(self) -> int:
        return self.h_stage.numel()

    def prepare(self) -> dict:
        """Host side of a step: slots and copies from the block manager, tables and
        lengths, all staged and sent to the device in one copy (on the copy stream;
        the compute stream waits for it)."""
        i = self._set ^ 1 if self._stepped else 0
        if self._h2d_done[i] is not None:
            self._h2d_done[i].synchronize()  # that set's host buffer is free again
        self._use_set(i)
        if self.rolling and self._stepped:
            self.alloc.truncate(self._seq_ids, self.base_lens)
        slots, pairs = self.alloc.append_slots(self._seq_ids, self.h_slots.numpy(),
                                               self.h_pairs.numpy())
        self._stepped = True
        n_cow = len(pairs)
        _, lens = self.alloc.build_block_tables(self._seq_ids, self.max_blocks,
                                                self.h_tables.numpy(), self.h_lens.numpy())
        max_len = int(lens.max()) if lens.size else 0
        num_chunks = max_chunk_parts = first_part = 0
        if self.group_members > 0:
            hp, hm, hc = self.h_groups
            pp, members, _, max_chunk_parts = self.alloc.prefix_groups(
                self._seq_ids, self.partition_size, self.group_members, hp.numpy(), hm.numpy(),
                hc.numpy())
            num_chunks = len(members)
            if num_chunks and lens.size:
                # the lowest partition any sequence computes itself
                own = np.minimum(pp, np.maximum(lens.astype(np.int64) - 1, 0) // self.partition_size)
                first_part = int(own.min())
        comp, cs = self._torch_stream(), self._copy_stream
        if self._kernels_done[i] is not None:
            cs.wait_event(self._kernels_done[i])   # kernels two steps back read it
        with torch.cuda.stream(cs):
            self.d_stage.copy_(self.h_stage, non_blocking=True)
            done = torch.cuda.Event()
            done.record(cs)
        self._h2d_done[i] = done
        comp.wait_event(done)
        return dict(num_cow=n_cow, max_len=max_len, pairs=self.h_pairs.numpy()[:n_cow],
                    num_chunks=num_chunks, max_chunk_parts=max_chunk_parts,
                    first_part=first_part)

    def launch(self, meta: dict, q, new_k, new_v, out, events=None) -> None:
        """Device side of a step: copies, the new token's K/V, attention.  ``events``
        (a pair of CUDA events) are recorded around the attention call."""
        st = self._torch_stream()
        n = meta["num_cow"]
        if n:
            pa_copy_blocks(self.k_cache, self.v_cache, self.d_pairs[:n], meta["pairs"], stream=st)
        if self.fp8:
            pa_reshape_and_cache_fp8(new_k, new_v, self.k_cache, self.v_cache, self.d_slots,
                                     *self.kv_scales, stream=st)
        else:
            pa_reshape_and_cache(new_k, new_v, self.k_cache, self.v_cache, self.d_slots, stream=st)
        ws = self._ws if self._ws.numel() else None
        if events is not None:
            events[0].record(st)
        if self.fp8:
            pa_decode_attention_fp8(out, q, self.k_cache, self.v_cache, self.d_tables, self.d_lens,
                                    self.scale, self.block_size, self.num_kv_heads,
                                    meta["max_len"], *self.kv_scales, self.partition_size, ws,
                                    stream=st)
        elif meta.get("num_chunks", 0):
            pp, cm, cp = self.d_groups
            pa_decode_attention_grouped(
                out, q, self.k_cache, self.v_cache, self.d_tables, self.d_lens, self.scale,
                self.block_size, self.num_kv_heads, meta["max_len"], pp, cm, cp,
                meta["num_chunks"], meta["max_chunk_parts"], self.partition_size, ws, stream=st,
                first_part=meta["first_part"])
        else:
            pa_decode_attention(out, q, self.k_cache, self.v_cache, self.d_tables, self.d_lens,
                                self.scale, self.block_size, self.num_kv_heads, meta["max_len"],
                                self.partition_size, ws, stream=st)
        if events is not None:
            events[1].record(st)
        done = torch.cuda.Event()
        done.record(st)
        self._kernels_done[self._set] = done

    def step(self, q, new_k, new_v, out) -> dict:
        meta = self.prepare()
        self.launch(meta, q, new_k, new_v, out)
        return meta

    # -- steps fed from host memory ----------------------------------------------
    def step_host(self, q_h, new_k_h, new_v_h, out_h):
        """One step whose inputs come from, and whose result goes back to, page-locked
        host tensors.  Copies run on their own streams and overlap the neighbouring
        steps' kernels: two device buffer sets alternate, and events order the
        input copy -> kernels -> output copy of each step.  Returns the event after
        which ``out_h`` holds this step's result (do not reuse ``out_h`` before)."""
        if not hasattr(self, "_io"):
            self._io_init(q_h, new_k_h, out_h)
        io = self._io[self._io_next]
        self._io_next ^= 1
        comp = self._torch_stream()
        h2d, d2h = self._h2d_stream, self._d2h_stream
        h2d.wait_event(io["compute_done"])          # the kernels two steps ago used them
        with torch.cuda.stream(h2d):
            for dst, src in zip(io["inputs"], (q_h, new_k_h, new_v_h)):
                dst.copy_(src, non_blocking=True)
            io["h2d_done"].record(h2d)
        comp.wait_event(io["h2d_done"])
        comp.wait_event(io["d2h_done"])             # the output buffer was read back
        meta = self.prepare()
        self.launch(meta, *io["inputs"], io["out"])
        io["compute_done"].record(comp)
        d2h.wait_event(io["compute_done"])
        with torch.cuda.stream(d2h):
            out_h.copy_(io["out"], non_blocking=True)
            io["d2h_done"].record(d2h)
        return io["d2h_done"]

    def drain_host_io(self) -> None:
        """Make the compute stream wait for every outstanding host-I/O copy."""
        if hasattr(self, "_io"):
            comp = self._torch_stream()
            for io in self._io:
                comp.wait_event(io["d2h_done"])

    def _io_init(self, q_h, kv_h, out_h) -> None:
        dev = self.device
        self._h2d_stream = torch.cuda.Stream(device=dev)
        self._d2h_stream = torch.cuda.Stream(device=dev)
        self._io, self._io_next = [], 0
        for _ in range(2):
            io = {"inputs": [torch.empty(q_h.shape, dtype=q_h.dtype, device=dev),
                             torch.empty(kv_h.shape, dtype=kv_h.dtype, device=dev),
                             torch.empty(kv_h.shape, dtype=kv_h.dtype, device=dev)],
                  "out": torch.empty(out_h.shape, dtype=out_h.dtype, device=dev)}
            for name in ("h2d_done", "compute_done", "d2h_done"):
                io[name] = torch.cuda.Event()
                io[name].record(self._torch_stream())   # start out completed
            self._io.append(io)

    def kernel_launches(self, meta: dict) -> int:
        """Library kernels one step launches (copy, write, group, partitions, merge)."""
        parts = max(1, -(-meta["max_len"] // self.partition_size))
        grouped = (meta.get("num_chunks", 0) > 0 and parts > 1 and not self.fp8
                   and self.k_cache.dtype != torch.float32
                   and self.block_size in (16, 32)
                   and self.group_members * (self.num_heads // self.num_kv_heads) <= 16)
        return (1 if meta["num_cow"] else 0) + 2 + (1 if grouped else 0) + (1 if parts > 1 else 0)

    def _torch_stream(self):
        return torch.cuda.current_stream(self.device) if self.stream is None else self.stream
