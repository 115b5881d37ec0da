"""B200 (sm_100a) paged KV-cache decode path: Python binding of ``libpa.so``.

The binding only marshals arguments: every GPU step runs in the library's CUDA
kernels and every allocator step in its C++ block manager.  Function names match
the C ABI in ``include/pa.h``.  Tensor arguments are torch CUDA tensors (torch is
used for device memory and streams only); importing this package fails loudly if
the library has not been built (``python paged_kv_cache_342_b200/csrc/build.py``).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_NO_FREE_BLOCKS, PA_ERR_UNKNOWN_SEQ = 0, 1, 2, 3
PA_ERR_SEQ_EXISTS, PA_ERR_BAD_INDEX, PA_ERR_CUDA, PA_ERR_UNSUPPORTED = 4, 5, 6, 7
PA_ERR_TOO_LARGE = 8
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "NO_FREE_BLOCKS", 3: "UNKNOWN_SEQ",
                4: "SEQ_EXISTS", 5: "BAD_INDEX", 6: "CUDA", 7: "UNSUPPORTED", 8: "TOO_LARGE"}
PA_STATIC_WORKSPACE_BYTES = 16 << 20
PA_F32, PA_BF16, PA_F16, PA_FP8_E4M3 = 0, 1, 2, 3
DEVERR_SLOT, DEVERR_COPY_BLOCK, DEVERR_TABLE, DEVERR_SEQ_LEN, DEVERR_TIMEOUT = 1, 2, 4, 8, 16
DEVERR_GROUP, DEVERR_ORDER, DEVERR_SMEM = 32, 64, 128
DEFAULT_PARTITION = 512


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where} failed: PA_ERR_{STATUS_NAMES.get(status, status)}")
        self.status = status
        self.code = STATUS_NAMES.get(status, str(status))


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python paged_kv_cache_342_b200/csrc/build.py`")

lib = ctypes.CDLL(LIB_PATH)

_i32, _i64, _p, _f = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float
_I32P, _I64P = ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)


class pa_stats_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "num_blocks", "block_size", "free_blocks", "used_blocks", "shared_blocks",
        "total_refs", "num_seqs", "logical_tokens", "allocated_slots", "tail_waste_slots",
        "cow_copies", "blocks_allocated", "cached_blocks", "evictable_blocks", "cache_hits",
        "cache_evictions")]


class pa_decoder_config_t(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_size_t), ("k_cache", _p), ("v_cache", _p),
                ("num_blocks", _i64), ("num_kv_heads", _i32), ("block_size", _i32),
                ("head_dim", _i32), ("num_heads", _i32), ("dtype", _i32), ("cache_dtype", _i32),
                ("scale", _f), ("k_scale", _f), ("v_scale", _f), ("max_blocks_per_seq", _i32),
                ("partition_size", _i32), ("group_members", _i32)]


class pa_decode_args_t(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_size_t), ("out", _p), ("q", _p), ("k_cache", _p),
                ("v_cache", _p), ("block_tables", _p), ("seq_lens", _p), ("scale", _f),
                ("block_size", _i32), ("num_kv_heads", _i32), ("num_seqs", _i32),
                ("num_heads", _i32), ("head_dim", _i32), ("max_blocks_per_seq", _i32),
                ("num_blocks", _i64), ("max_seq_len", _i32), ("partition_size", _i32),
                ("dtype", _i32), ("cache_dtype", _i32), ("k_scale", _f), ("v_scale", _f),
                ("seq_order", _p), ("prefix_parts", _p), ("chunk_members", _p),
                ("chunk_parts", _p), ("num_chunks", _i32), ("max_members", _i32),
                ("max_chunk_parts", _i32), ("first_part", _i32), ("workspace", _p),
                ("workspace_bytes", ctypes.c_size_t), ("stream", _p)]


class pa_step_info_t(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_size_t), ("num_cow", _i32), ("max_seq_len", _i32),
                ("partition_size", _i32), ("num_chunks", _i32), ("max_chunk_parts", _i32),
                ("first_part", _i32), ("kernels", _i32), ("slots", _I64P),
                ("cow_pairs", _I32P), ("block_tables", _I32P), ("seq_lens", _I32P)]


def _sig(name, res, *args):
    fn = getattr(lib, name)
    fn.restype = res
    fn.argtypes = list(args)


_sig("pa_reshape_and_cache", _i32, _p, _p, _p, _p, _p, _i64, _i32, _i32, _i32, _i64, _i32, _p)
_sig("pa_copy_blocks", _i32, _p, _p, _p, _p, _i32, _i32, _i32, _i32, _i64, _i32, _p)
_sig("pa_reshape_and_cache_fp8", _i32, _p, _p, _p, _p, _p, _i64, _i32, _i32, _i32, _i64, _i32,
     _f, _f, _p)
_sig("pa_decode_attention_fp8", _i32, _p, _p, _p, _p, _p, _p, _f, _i32, _i32, _i32, _i32, _i32,
     _i32, _i64, _i32, _i32, _i32, _f, _f, _p, ctypes.c_size_t, _p)
_sig("pa_swap_blocks", _i32, _p, _p, _i64, _p, _p, _i64, _p, _p, _i32, _i32, _i32, _i32, _i32, _p)
_sig("pa_decode_workspace_bytes", ctypes.c_size_t, _i32, _i32, _i32, _i32, _i32)
_sig("pa_decode_partition_size", _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32)
_sig("pa_decode_attention", _i32, _p, _p, _p, _p, _p, _p, _f, _i32, _i32, _i32, _i32, _i32,
     _i32, _i64, _i32, _i32, _i32, _p, ctypes.c_size_t, _p)
_sig("pa_decode_attention_static_ws", _i32, _p, _p, _p, _p, _p, _p, _f, _i32, _i32, _i32, _i32,
     _i32, _i32, _i64, _i32, _i32, _i32, _p)
_sig("pa_decode_attention_grouped", _i32, _p, _p, _p, _p, _p, _p, _f, _i32, _i32, _i32, _i32,
     _i32, _i32, _i64, _i32, _i32, _i32, _p, _p, _p, _i32, _i32, _i32, _i32, _p,
     ctypes.c_size_t, _p)
_sig("pa_decode_uses_tensor_cores", _i32, _i32, _i32, _i32, _i32, _i32)
_sig("pa_device_error_read", _i32, ctypes.POINTER(ctypes.c_uint32))
_sig("pa_last_cuda_error", ctypes.c_char_p)
_sig("pa_selftest_bounded_wait", _i32, _p)
_sig("pa_alloc_create", _i32, _i64, _i32, _p, ctypes.POINTER(_p))
_sig("pa_alloc_destroy", _i32, _p)
_sig("pa_seq_add", _i32, _p, _i64, _i64)
_sig("pa_seq_fork", _i32, _p, _i64, _i64)
_sig("pa_seq_add_prompt", _i32, _p, _i64, _p, _i64, _I64P)
_sig("pa_seq_append_slot", _i32, _p, _i64, _I64P, _I32P, _I32P)
_sig("pa_seq_append_slots", _i32, _p, _p, _i32, _p, _p, ctypes.POINTER(ctypes.c_int))
_sig("pa_seq_free", _i32, _p, _i64)
_sig("pa_seq_truncate", _i32, _p, _p, _p, _i32)
_sig("pa_seqs_move", _i32, _p, _p, _p, _i32, _p, _i64, _I64P)
_sig("pa_seq_len", _i32, _p, _i64, _I64P)
_sig("pa_seq_blocks", _i32, _p, _i64, _p, _i64, _I64P)
_sig("pa_build_block_tables", _i32, _p, _p, _i32, _p, _i32, _p)
_sig("pa_block_refcount", _i32, _p, _i32, _I32P)
_sig("pa_build_prefix_groups", _i32, _p, _p, _i32, _i32, _i32, _p, _p, _p,
     ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int))
_sig("pa_alloc_free_list", _i32, _p, _p, _i64, _I64P)
_sig("pa_alloc_stats", _i32, _p, ctypes.POINTER(pa_stats_t))
_sig("pa_decode", _i32, ctypes.POINTER(pa_decode_args_t))
_sig("pa_decoder_create", _i32, ctypes.POINTER(pa_decoder_config_t), _p, ctypes.POINTER(_p))
_sig("pa_decoder_destroy", _i32, _p)
_sig("pa_decoder_bind", _i32, _p, _p, _i32, _i32, _p, ctypes.c_size_t)
_sig("pa_decoder_device_bytes", _i32, _p, _i32, ctypes.POINTER(ctypes.c_size_t))
_sig("pa_decoder_step", _i32, _p, _p, _p, _p, _p, _p, _p, _p, ctypes.POINTER(pa_step_info_t))
_sig("pa_decoder_step_host", _i32, _p, _p, _p, _p, _p, _p, _I64P,
     ctypes.POINTER(pa_step_info_t))
_sig("pa_decoder_wait", _i32, _p, _i64)
_sig("pa_decoder_drain", _i32, _p, _p)
_sig("pa_decoder_query", _i32, _p, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_size_t),
     ctypes.POINTER(ctypes.c_size_t))


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        if status == PA_ERR_CUDA:
            where += " (" + pa_last_cuda_error() + ")"
        raise PagedAttentionError(status, where)


def pa_last_cuda_error() -> str:
    return (lib.pa_last_cuda_error() or b"").decode(errors="replace")


# ---------------------------------------------------------------------------
# GPU entry points (torch CUDA tensors in, nothing computed here)
# ---------------------------------------------------------------------------

def _dtype_code(t) -> int:
    import torch
    codes = {torch.float32: PA_F32, torch.bfloat16: PA_BF16, torch.float16: PA_F16,
             torch.uint8: PA_FP8_E4M3, torch.float8_e4m3fn: PA_FP8_E4M3}
    if t.dtype not in codes:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _dev(t, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """key/value [T, Hkv, D]; caches [NB, Hkv, bs, D]; slot_mapping int64 [T]."""
    import torch
    T, Hkv, D = key.shape
    NB, _, bs, _ = k_cache.shape
    _check(lib.pa_reshape_and_cache(
        _dev(key, "key"), _dev(value, "value"), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"), _dev(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D,
        bs, NB, _dtype_code(k_cache), _stream(stream)), "pa_reshape_and_cache")


def pa_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                             stream=None) -> None:
    """key/value [T, Hkv, D] (f32/bf16/f16); caches [NB, Hkv, bs, D] of e4m3 codes
    (a uint8 or float8_e4m3fn CUDA tensor)."""
    import torch
    T, Hkv, D = key.shape
    NB, _, bs, _ = k_cache.shape
    if k_cache.element_size() != 1:
        raise ValueError("fp8 caches hold one byte per element")
    _check(lib.pa_reshape_and_cache_fp8(
        _dev(key, "key"), _dev(value, "value"), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"), _dev(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D,
        bs, NB, _dtype_code(key), float(k_scale), float(v_scale), _stream(stream)),
        "pa_reshape_and_cache_fp8")


def pa_decode_attention_fp8(out, q, k_cache, v_cache, block_tables, seq_lens, scale,
                            block_size, num_kv_heads, max_seq_len, k_scale, v_scale,
                            partition_size=DEFAULT_PARTITION, workspace=None,
                            stream=None) -> None:
    """pa_decode_attention over e4m3 caches; q/out bf16 or f16."""
    import torch
    S, Hq, D = q.shape
    NB = k_cache.shape[0]
    if k_cache.element_size() != 1:
        raise ValueError("fp8 caches hold one byte per element")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_attention_fp8(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), block_size, num_kv_heads, S, Hq, D, block_tables.shape[1], NB,
        int(max_seq_len), partition_size, _dtype_code(q), float(k_scale), float(v_scale), ws_ptr,
        ws_bytes, _stream(stream)), "pa_decode_attention_fp8")


def pa_copy_blocks(k_cache, v_cache, block_mapping, block_mapping_host=None, stream=None) -> None:
    """block_mapping int32 [n, 2] on the device; block_mapping_host the same pairs as a
    host int32 array (validated by the library) or None."""
    import torch
    n = int(block_mapping.shape[0])
    NB, Hkv, bs, D = k_cache.shape
    host_ptr = None
    if block_mapping_host is not None:
        block_mapping_host = np.ascontiguousarray(block_mapping_host, dtype=np.int32)
        host_ptr = block_mapping_host.ctypes.data
    _check(lib.pa_copy_blocks(
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_mapping, "block_mapping", torch.int32) if n else None, host_ptr, n, Hkv, D, bs,
        NB, _dtype_code(k_cache), _stream(stream)), "pa_copy_blocks")


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, block_mapping, block_mapping_host=None,
                   stream=None) -> None:
    """Copy blocks src -> dst between two caches [NB, Hkv, bs, D]; each may be a CUDA
    tensor or a pinned CPU tensor.  block_mapping int32 [n, 2] (CUDA or pinned)."""
    import torch
    n = int(block_mapping.shape[0])
    if n == 0:
        return
    for t, name in ((dst_k, "dst_k"), (dst_v, "dst_v"), (src_k, "src_k"), (src_v, "src_v"),
                    (block_mapping, "block_mapping")):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    if block_mapping.dtype != torch.int32:
        raise ValueError("block_mapping must be int32")
    host_ptr = None
    if block_mapping_host is not None:
        block_mapping_host = np.ascontiguousarray(block_mapping_host, dtype=np.int32)
        host_ptr = block_mapping_host.ctypes.data
    NBd, Hkv, bs, D = dst_k.shape
    NBs = src_k.shape[0]
    _check(lib.pa_swap_blocks(dst_k.data_ptr(), dst_v.data_ptr(), NBd, src_k.data_ptr(),
                              src_v.data_ptr(), NBs, block_mapping.data_ptr(), host_ptr, n, Hkv,
                              D, bs, _dtype_code(dst_k), _stream(stream)), "pa_swap_blocks")


def pa_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_seq_len,
                              partition_size=DEFAULT_PARTITION) -> int:
    return int(lib.pa_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_seq_len,
                                             partition_size))


def pa_decode_partition_size(cache_dtype_code, num_seqs, num_heads, num_kv_heads, head_dim,
                             block_size, max_seq_len, num_sms=0) -> int:
    """The library's partition size for this decode grid (0 = invalid arguments)."""
    return int(lib.pa_decode_partition_size(cache_dtype_code, num_seqs, num_heads, num_kv_heads,
                                            head_dim, block_size, int(max_seq_len), num_sms))


def pa_decode_attention(out, q, k_cache, v_cache, block_tables, seq_lens, scale, block_size,
                        num_kv_heads, max_seq_len, partition_size=DEFAULT_PARTITION,
                        workspace=None, stream=None) -> None:
    """out/q [S, Hq, D]; caches [NB, Hkv, bs, D]; block_tables int32 [S, max_blocks];
    seq_lens int32 [S]; workspace a uint8 CUDA tensor of at least
    pa_decode_workspace_bytes(...) bytes (or None when that is 0)."""
    import torch
    S, Hq, D = q.shape
    NB = k_cache.shape[0]
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_attention(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), block_size, num_kv_heads, S, Hq, D, block_tables.shape[1], NB,
        int(max_seq_len), partition_size, _dtype_code(q), ws_ptr, ws_bytes, _stream(stream)),
        "pa_decode_attention")


def pa_decode_attention_grouped(out, q, k_cache, v_cache, block_tables, seq_lens, scale,
                                block_size, num_kv_heads, max_seq_len, prefix_parts,
                                chunk_members, chunk_parts, num_chunks, max_chunk_parts,
                                partition_size=DEFAULT_PARTITION, workspace=None,
                                stream=None, first_part=0) -> None:
    """pa_decode_attention with prefix groups (device int32 tensors prefix_parts [S],
    chunk_members [>= num_chunks, max_members], chunk_parts [>= num_chunks]);
    first_part as documented in pa.h (0 is always safe)."""
    import torch
    S, Hq, D = q.shape
    NB = k_cache.shape[0]
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_attention_grouped(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), block_size, num_kv_heads, S, Hq, D, block_tables.shape[1], NB,
        int(max_seq_len), partition_size, _dtype_code(q),
        _dev(prefix_parts, "prefix_parts", torch.int32),
        _dev(chunk_members, "chunk_members", torch.int32),
        _dev(chunk_parts, "chunk_parts", torch.int32), int(num_chunks),
        int(chunk_members.shape[1]), int(max_chunk_parts), int(first_part), ws_ptr, ws_bytes,
        _stream(stream)), "pa_decode_attention_grouped")


def pa_decode_attention_static_ws(out, q, k_cache, v_cache, block_tables, seq_lens, scale,
                                  block_size, num_kv_heads, max_seq_len,
                                  partition_size=DEFAULT_PARTITION, stream=None) -> None:
    """pa_decode_attention with the library's own fixed scratch array instead of a
    caller workspace: for callers that may not allocate device memory.  Raises
    PagedAttentionError (TOO_LARGE) when the call needs more than
    PA_STATIC_WORKSPACE_BYTES of scratch; overlapping calls on one device race."""
    import torch
    S, Hq, D = q.shape
    NB = k_cache.shape[0]
    _check(lib.pa_decode_attention_static_ws(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), block_size, num_kv_heads, S, Hq, D, block_tables.shape[1], NB,
        int(max_seq_len), partition_size, _dtype_code(q), _stream(stream)),
        "pa_decode_attention_static_ws")


def pa_decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale, block_size,
              num_kv_heads, max_seq_len, partition_size=DEFAULT_PARTITION, workspace=None,
              seq_order=None, kv_scales=None, stream=None) -> None:
    """pa_decode_attention (or, for a one-byte cache, pa_decode_attention_fp8 with
    kv_scales = (k_scale, v_scale)) through the argument block, with an optional
    int32 CUDA tensor seq_order [S] (the order the grid takes the sequences in)."""
    import torch
    S, Hq, D = q.shape
    a = pa_decode_args_t()
    a.struct_size = ctypes.sizeof(pa_decode_args_t)
    a.out, a.q = _dev(out, "out"), _dev(q, "q")
    a.k_cache, a.v_cache = _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache")
    a.block_tables = _dev(block_tables, "block_tables", torch.int32)
    a.seq_lens = _dev(seq_lens, "seq_lens", torch.int32)
    a.scale, a.block_size, a.num_kv_heads = float(scale), block_size, num_kv_heads
    a.num_seqs, a.num_heads, a.head_dim = S, Hq, D
    a.max_blocks_per_seq, a.num_blocks = block_tables.shape[1], k_cache.shape[0]
    a.max_seq_len, a.partition_size = int(max_seq_len), partition_size
    a.dtype, a.cache_dtype = _dtype_code(q), _dtype_code(k_cache)
    a.k_scale, a.v_scale = (float(x) for x in (kv_scales or (1.0, 1.0)))
    if seq_order is not None:
        a.seq_order = _dev(seq_order, "seq_order", torch.int32)
    if workspace is not None:
        a.workspace = _dev(workspace, "workspace")
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    a.stream = _stream(stream)
    _check(lib.pa_decode(ctypes.byref(a)), "pa_decode")


def pa_decode_uses_tensor_cores(dtype_code, num_heads, num_kv_heads, head_dim, block_size) -> bool:
    return bool(lib.pa_decode_uses_tensor_cores(dtype_code, num_heads, num_kv_heads, head_dim,
                                                block_size))


def pa_selftest_bounded_wait(stream=None) -> None:
    _check(lib.pa_selftest_bounded_wait(_stream(stream)), "pa_selftest_bounded_wait")


def pa_device_error_read() -> int:
    bits = ctypes.c_uint32(0)
    _check(lib.pa_device_error_read(ctypes.byref(bits)), "pa_device_error_read")
    return int(bits.value)


# ---------------------------------------------------------------------------
# host block allocator
# ---------------------------------------------------------------------------

class BlockAllocator:
    """Owns one ``pa_alloc_t``; each method is one C-ABI call."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self._h = _p()
        order = None
        if free_order is not None:
            self._order = np.ascontiguousarray(free_order, dtype=np.int32)
            order = self._order.ctypes.data
        _check(lib.pa_alloc_create(num_blocks, block_size, order, ctypes.byref(self._h)),
               "pa_alloc_create")
        self.num_blocks, self.block_size = num_blocks, block_size

    def close(self) -> None:
        if self._h:
            lib.pa_alloc_destroy(self._h)
            self._h = _p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def add(self, seq_id: int, num_tokens: int) -> None:
        _check(lib.pa_seq_add(self._h, seq_id, num_tokens), "pa_seq_add")

    def add_prompt(self, seq_id: int, token_ids) -> int:
        """Admit a sequence by its prompt tokens with prefix caching; returns the number
        of leading tokens served by cached blocks."""
        toks = np.ascontiguousarray(token_ids, dtype=np.int32)
        cached = ctypes.c_int64(0)
        _check(lib.pa_seq_add_prompt(self._h, seq_id, toks.ctypes.data, toks.size,
                                     ctypes.byref(cached)), "pa_seq_add_prompt")
        return cached.value

    def fork(self, parent: int, child: int) -> None:
        _check(lib.pa_seq_fork(self._h, parent, child), "pa_seq_fork")

    def append_slot(self, seq_id: int):
        slot, src, dst = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib.pa_seq_append_slot(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src),
                                      ctypes.byref(dst)), "pa_seq_append_slot")
        return slot.value, src.value, dst.value

    def append_slots(self, seq_ids, slots_out=None, pairs_out=None):
        """One append per id, in order, all or nothing.  Returns (slots int64 [n],
        cow pairs int32 [k, 2]); pass preallocated (pinned) arrays to avoid copies."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        slots = np.empty(n, np.int64) if slots_out is None else slots_out
        pairs = np.empty((max(n, 1), 2), np.int32) if pairs_out is None else pairs_out
        nc = ctypes.c_int(0)
        _check(lib.pa_seq_append_slots(self._h, ids.ctypes.data, n, slots.ctypes.data,
                                       pairs.ctypes.data, ctypes.byref(nc)), "pa_seq_append_slots")
        return slots[:n], pairs[:nc.value]

    def truncate(self, seq_ids, new_lens) -> None:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        lens = np.ascontiguousarray(new_lens, dtype=np.int64)
        if ids.size != lens.size:
            raise ValueError("seq_ids and new_lens differ in length")
        _check(lib.pa_seq_truncate(self._h, ids.ctypes.data, lens.ctypes.data, ids.size),
               "pa_seq_truncate")

    def move_to(self, other: "BlockAllocator", seq_ids) -> np.ndarray:
        """Move sequences into another pool; returns the (this_block, other_block) copy
        pairs (int32 [k, 2]) to make with pa_swap_blocks."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        cap = sum(len(self.seq_blocks(int(s))) for s in ids) if ids.size else 0
        pairs = np.empty((max(cap, 1), 2), np.int32)
        n = ctypes.c_int64(0)
        _check(lib.pa_seqs_move(self._h, other._h, ids.ctypes.data, ids.size, pairs.ctypes.data,
                                cap, ctypes.byref(n)), "pa_seqs_move")
        return pairs[:n.value]

    def free(self, seq_id: int) -> None:
        _check(lib.pa_seq_free(self._h, seq_id), "pa_seq_free")

    def seq_len(self, seq_id: int) -> int:
        n = ctypes.c_int64()
        _check(lib.pa_seq_len(self._h, seq_id, ctypes.byref(n)), "pa_seq_len")
        return n.value

    def seq_blocks(self, seq_id: int) -> list:
        n = ctypes.c_int64()
        _check(lib.pa_seq_blocks(self._h, seq_id, None, 0, ctypes.byref(n)), "pa_seq_blocks")
        out = np.empty(n.value, np.int32)
        _check(lib.pa_seq_blocks(self._h, seq_id, out.ctypes.data, n.value, ctypes.byref(n)),
               "pa_seq_blocks")
        return out.tolist()

    def build_block_tables(self, seq_ids, max_blocks: int, tables_out=None, lens_out=None):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tables = np.empty((ids.size, max_blocks), np.int32) if tables_out is None else tables_out
        lens = np.empty(ids.size, np.int32) if lens_out is None else lens_out
        _check(lib.pa_build_block_tables(self._h, ids.ctypes.data, ids.size, tables.ctypes.data,
                                         max_blocks, lens.ctypes.data), "pa_build_block_tables")
        return tables, lens

    def prefix_groups(self, seq_ids, partition_size: int, max_members: int, prefix_parts=None,
                      chunk_members=None, chunk_parts=None):
        """(prefix_parts [n], chunk_members [k, max_members], chunk_parts [k],
        max_chunk_parts) for pa_decode_attention_grouped; pass preallocated (pinned)
        arrays of full capacity to fill them in place."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        pp = np.empty(n, np.int32) if prefix_parts is None else prefix_parts
        cm = np.empty((max(n, 1), max_members), np.int32) if chunk_members is None else chunk_members
        cp = np.empty(max(n, 1), np.int32) if chunk_parts is None else chunk_parts
        nc, mp = ctypes.c_int(0), ctypes.c_int(0)
        _check(lib.pa_build_prefix_groups(self._h, ids.ctypes.data, n, partition_size, max_members,
                                          pp.ctypes.data, cm.ctypes.data, cp.ctypes.data,
                                          ctypes.byref(nc), ctypes.byref(mp)),
               "pa_build_prefix_groups")
        return pp[:n], cm[:nc.value], cp[:nc.value], mp.value

    def refcount(self, block: int) -> int:
        r = ctypes.c_int32()
        _check(lib.pa_block_refcount(self._h, block, ctypes.byref(r)), "pa_block_refcount")
        return r.value

    def free_list(self) -> list:
        n = ctypes.c_int64()
        out = np.empty(self.num_blocks, np.int32)
        _check(lib.pa_alloc_free_list(self._h, out.ctypes.data, self.num_blocks, ctypes.byref(n)),
               "pa_alloc_free_list")
        return out[:n.value].tolist()

    def stats(self) -> dict:
        st = pa_stats_t()
        _check(lib.pa_alloc_stats(self._h, ctypes.byref(st)), "pa_alloc_stats")
        return {name: getattr(st, name) for name, _ in pa_stats_t._fields_}
