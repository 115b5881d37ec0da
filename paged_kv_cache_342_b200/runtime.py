"""One decode step of the paged KV-cache path, driven through the native step runtime
(``pa_decoder_*`` in ``include/pa.h``).

Order of a step (the sources are the pages cited in ``include/pa.h``), all of it in
the library's C++ and CUDA code:
  1. the block manager gives every sequence room for one more token
     (``pa_seq_append_slots``): a slot, and a (src, dst) copy where the token's
     block is shared;
  2. slots, copy pairs, lengths, block tables and prefix groups are written into one
     of two page-locked staging sets and sent to the device in one copy (the only
     host-to-device traffic of a step), on the decoder's own copy stream;
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
per-tensor ``kv_scales`` (k_scale, v_scale) and a 16-bit ``query_dtype`` for q, the
new K/V rows and out: the step writes with ``pa_reshape_and_cache_fp8`` and attends
with ``pa_decode_attention_fp8``.

This module only moves arguments: the work of every step is done by the library.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import (DEFAULT_PARTITION, BlockAllocator, _check, _dtype_code, lib, pa_copy_blocks,
               pa_decoder_config_t, pa_step_info_t)


class StepInfo:
    """Facts of one step, from the library's ``pa_step_info_t``.  ``slots``,
    ``tables``, ``lens`` and ``pairs`` are numpy views of the step's page-locked
    staging set, valid until the step after the next (copy them to keep them)."""

    __slots__ = ("num_cow", "max_len", "partition_size", "num_chunks", "max_chunk_parts",
                 "first_part", "kernels", "_info", "_S", "_MB")

    def __init__(self, info: pa_step_info_t, S: int, MB: int):
        self.num_cow, self.max_len = info.num_cow, info.max_seq_len
        self.partition_size, self.num_chunks = info.partition_size, info.num_chunks
        self.max_chunk_parts, self.first_part = info.max_chunk_parts, info.first_part
        self.kernels = info.kernels
        self._info, self._S, self._MB = info, S, MB

    @property
    def slots(self) -> np.ndarray:
        return np.ctypeslib.as_array(self._info.slots, (self._S,))

    @property
    def lens(self) -> np.ndarray:
        return np.ctypeslib.as_array(self._info.seq_lens, (self._S,))

    @property
    def tables(self) -> np.ndarray:
        return np.ctypeslib.as_array(self._info.block_tables, (self._S, self._MB))

    @property
    def pairs(self) -> np.ndarray:
        if self.num_cow == 0:
            return np.zeros((0, 2), np.int32)
        return np.ctypeslib.as_array(self._info.cow_pairs, (self.num_cow, 2))

    # dict-style access to the scalar facts and the pairs
    _KEYS = {"num_cow": "num_cow", "max_len": "max_len", "num_chunks": "num_chunks",
             "max_chunk_parts": "max_chunk_parts", "first_part": "first_part",
             "kernels": "kernels", "pairs": "pairs", "partition_size": "partition_size"}

    def __getitem__(self, key):
        return getattr(self, self._KEYS[key])

    def get(self, key, default=None):
        return getattr(self, self._KEYS[key]) if key in self._KEYS else default


class HostStep:
    """Completion handle of a host-fed step: ``synchronize()`` blocks until the step's
    output is in its host buffer (and its inputs have been read)."""

    __slots__ = ("_dec", "ticket")

    def __init__(self, dec, ticket: int):
        self._dec, self.ticket = dec, ticket

    def synchronize(self) -> None:
        _check(lib.pa_decoder_wait(self._dec, self.ticket), "pa_decoder_wait")


class PagedDecoder:
    """Device caches + block manager + the library's step runtime for a fixed batch.

    ``k_cache``/``v_cache`` are caller-owned CUDA tensors [NB, Hkv, bs, D].
    ``max_blocks_per_seq`` is the block-table width (capacity per sequence).
    ``partition_size`` 0 takes ``pa_decode_partition_size`` for the bound batch at
    that capacity (it ignores prefix groups, so batches of forks do better with an
    explicit size shorter than their shared prefix).
    """

    def __init__(self, k_cache, v_cache, num_heads: int, scale: float, max_blocks_per_seq: int,
                 free_order=None, partition_size: int = DEFAULT_PARTITION, stream=None,
                 group_members: int | None = None, kv_scales=None, query_dtype=None):
        self.k_cache, self.v_cache = k_cache, v_cache
        self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim = k_cache.shape
        self.num_heads, self.scale = num_heads, scale
        self.max_blocks = max_blocks_per_seq
        self.partition_size = partition_size
        self.device = k_cache.device
        self.stream = stream
        self.alloc = BlockAllocator(self.num_blocks, self.block_size, free_order)
        group = num_heads // self.num_kv_heads
        self.fp8 = k_cache.element_size() == 1
        if self.fp8 and (kv_scales is None or query_dtype is None):
            raise ValueError("an fp8 cache needs kv_scales=(k_scale, v_scale) and query_dtype")
        self.kv_scales = kv_scales
        self.group_members = (8 // group if group <= 8 else 0) if group_members is None \
            else group_members
        if self.fp8:
            self.group_members = 0
        self.workspace_bytes = self.staging_bytes = 0
        self._S = 0
        self._device_buffer = None
        cfg = pa_decoder_config_t()
        cfg.struct_size = ctypes.sizeof(pa_decoder_config_t)
        cfg.k_cache, cfg.v_cache = k_cache.data_ptr(), v_cache.data_ptr()
        cfg.num_blocks, cfg.num_kv_heads = self.num_blocks, self.num_kv_heads
        cfg.block_size, cfg.head_dim, cfg.num_heads = self.block_size, self.head_dim, num_heads
        cfg.cache_dtype = _dtype_code(k_cache)
        cfg.dtype = (_dtype_code(torch.empty(0, dtype=query_dtype)) if self.fp8
                     else cfg.cache_dtype)
        cfg.scale = float(scale)
        cfg.k_scale, cfg.v_scale = (float(x) for x in (kv_scales or (1.0, 1.0)))
        cfg.max_blocks_per_seq, cfg.partition_size = max_blocks_per_seq, partition_size
        cfg.group_members = self.group_members
        self._cfg = cfg
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(lib.pa_decoder_create(ctypes.byref(cfg), self.alloc._h, ctypes.byref(h)),
                   "pa_decoder_create")
        self._h = h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            try:
                lib.pa_decoder_destroy(h)   # waits for the work that uses the buffer
            except Exception:  # interpreter shutdown: the library may be gone already
                pass
            self._h = None
        self._device_buffer = None

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
        """Fix the batch the steps run over.  Its device buffers (staging, workspace,
        host-I/O sets) are one torch allocation of the size the library asks for,
        held until the next bind or the decoder's end."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        need = ctypes.c_size_t(0)
        with torch.cuda.device(self.device):
            _check(lib.pa_decoder_device_bytes(self._h, ids.size, ctypes.byref(need)),
                   "pa_decoder_device_bytes")
            buf = torch.empty(need.value, dtype=torch.uint8, device=self.device)
        # the library waits for the previous batch's work before it lets go of the old
        # buffer, so that one is released only after the call
        _check(lib.pa_decoder_bind(self._h, ids.ctypes.data, ids.size, int(rolling),
                                   buf.data_ptr(), need.value), "pa_decoder_bind")
        self._device_buffer = buf
        self._S = ids.size
        ps, ws, st = ctypes.c_int(0), ctypes.c_size_t(0), ctypes.c_size_t(0)
        _check(lib.pa_decoder_query(self._h, ctypes.byref(ps), ctypes.byref(ws), ctypes.byref(st)),
               "pa_decoder_query")
        self.partition_size = ps.value
        self.workspace_bytes, self.staging_bytes = ws.value, st.value

    def step(self, q, new_k, new_v, out, events=None) -> StepInfo:
        """One step on device tensors (q/out [S, Hq, D], new_k/new_v [S, Hkv, D]);
        ``events`` (a pair of CUDA events) are recorded around the attention call."""
        self._check_io(q, new_k, new_v, out, cuda=True)
        info = pa_step_info_t()
        info.struct_size = ctypes.sizeof(pa_step_info_t)
        e0 = e1 = None
        if events is not None:
            e0, e1 = (_event_handle(e) for e in events)
        _check(lib.pa_decoder_step(self._h, q.data_ptr(), new_k.data_ptr(), new_v.data_ptr(),
                                   out.data_ptr(), self._stream_handle(), e0, e1,
                                   ctypes.byref(info)), "pa_decoder_step")
        return StepInfo(info, self._S, self.max_blocks)

    # -- steps fed from host memory ----------------------------------------------
    def step_host(self, q_h, new_k_h, new_v_h, out_h) -> HostStep:
        """One step whose inputs come from, and whose result goes back to, page-locked
        host tensors; the copies overlap the neighbouring steps' kernels.  Returns the
        handle whose ``synchronize()`` waits for ``out_h`` (do not reuse the buffers
        before)."""
        self._check_io(q_h, new_k_h, new_v_h, out_h, cuda=False)
        ticket = ctypes.c_int64(0)
        _check(lib.pa_decoder_step_host(self._h, q_h.data_ptr(), new_k_h.data_ptr(),
                                        new_v_h.data_ptr(), out_h.data_ptr(),
                                        self._stream_handle(), ctypes.byref(ticket), None),
               "pa_decoder_step_host")
        return HostStep(self._h, ticket.value)

    def drain_host_io(self) -> None:
        """Make the compute stream wait for every outstanding host-I/O copy."""
        _check(lib.pa_decoder_drain(self._h, self._stream_handle()), "pa_decoder_drain")

    def kernel_launches(self, meta: StepInfo) -> int:
        """Library kernels one step launches (copies, new tokens' write, partition grid, merge
        or, for a grouped batch, the clear of its arrival counters)."""
        return meta.kernels

    def _check_io(self, q, new_k, new_v, out, cuda: bool) -> None:
        S, Hq, Hkv, D = self._S, self.num_heads, self.num_kv_heads, self.head_dim
        want = self._cfg.dtype
        for t, shape in ((q, (S, Hq, D)), (new_k, (S, Hkv, D)), (new_v, (S, Hkv, D)),
                         (out, (S, Hq, D))):
            if (tuple(t.shape) != shape or t.is_cuda != cuda or not t.is_contiguous()
                    or _dtype_code(t) != want):
                raise ValueError(f"step tensor {tuple(t.shape)} {t.dtype} "
                                 f"({'cuda' if t.is_cuda else 'host'}) does not fit the "
                                 f"bound batch {shape}")

    def _torch_stream(self):
        return torch.cuda.current_stream(self.device) if self.stream is None else self.stream

    def _stream_handle(self) -> int:
        return self._torch_stream().cuda_stream


def _event_handle(ev) -> int:
    """The cudaEvent_t of a torch CUDA event (recorded once if it was never used, so
    that it exists)."""
    h = ev.cuda_event
    if not h:
        ev.record()
        h = ev.cuda_event
    return h
