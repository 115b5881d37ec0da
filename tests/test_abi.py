"""The C-ABI library loads, exports every function include/pa.h declares, and
rejects bad arguments before touching a GPU (host-only checks; no kernel runs)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    return m


def declared_functions():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(pa_\w+)\s*\(", text,
                                 flags=re.M)))


def test_header_declares_the_path():
    names = declared_functions()
    for must in ("pa_reshape_and_cache", "pa_copy_blocks", "pa_decode_attention",
                 "pa_decode_workspace_bytes", "pa_alloc_create", "pa_seq_fork",
                 "pa_seq_append_slot", "pa_alloc_stats"):
        assert must in names


def test_library_exports_every_declared_symbol(pa):
    lib = ctypes.CDLL(pa.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert missing == []


def test_library_is_built_for_sm100a(pa):
    # the fatbin of an sm_100a build names the architecture; a cheap check without
    # disassembling anything
    data = open(pa.LIB_PATH, "rb").read()
    assert b"sm_100a" in data


def test_workspace_bytes(pa):
    assert pa.pa_decode_workspace_bytes(64, 32, 128, 512, 512) == 0       # one partition
    assert pa.pa_decode_workspace_bytes(64, 32, 128, 0, 512) == 0
    b = pa.pa_decode_workspace_bytes(8, 64, 128, 131072, 512)
    rows = 8 * 64 * 256
    align = lambda x: (x + 255) // 256 * 256
    # partial outputs, maxima, exp-sums, then one int32 arrival counter per query row
    assert b == align(rows * 128 * 4) + 2 * align(rows * 4) + align(8 * 64 * 4)
    assert pa.pa_decode_workspace_bytes(2, 4, 64, 1000, 0) == \
        pa.pa_decode_workspace_bytes(2, 4, 64, 1000, 512)
    assert pa.pa_decode_workspace_bytes(-1, 4, 64, 1000, 512) == 0


def test_tensor_core_path_selection(pa):
    assert pa.pa_decode_uses_tensor_cores(pa.PA_BF16, 64, 8, 128, 16)
    assert pa.pa_decode_uses_tensor_cores(pa.PA_F16, 32, 2, 64, 32)
    assert not pa.pa_decode_uses_tensor_cores(pa.PA_BF16, 32, 32, 128, 16)   # MHA
    assert not pa.pa_decode_uses_tensor_cores(pa.PA_F32, 64, 8, 128, 16)     # fp32 cache
    assert not pa.pa_decode_uses_tensor_cores(pa.PA_BF16, 64, 8, 128, 8)     # block 8


def test_partition_size_choice(pa):
    ps = pa.pa_decode_partition_size
    # 7B-shaped: 64 seqs x 32 CUDA-core CTAs = 2048 >= 12 x 148, so one partition covers
    # the longest sequence (512 -> 5, 1024 -> 3, 2048 -> 2, 4096 -> 1 partitions)
    assert ps(pa.PA_BF16, 64, 32, 32, 128, 16, 2050, 148) == 4096
    # 13B-shaped: 256 x 40 CTAs, longest 4097 tokens
    assert ps(pa.PA_F16, 256, 40, 40, 128, 16, 4097, 148) == 8192
    # GQA 8:1 on tensor cores: 8 seqs x 8 kv-head CTAs; at 2048 tokens 65 partitions
    # give 64 * 33 = 2112 working CTAs (>= 1776), at 4096 only 64 * 17 = 1088
    assert ps(pa.PA_BF16, 8, 64, 8, 128, 16, 131073, 148) == 2048
    assert ps(pa.PA_FP8_E4M3, 8, 64, 8, 128, 16, 131073, 148) == 2048
    # the same shape on CUDA cores (block 8): 8 seqs x 64/4 CTAs = 128 rows
    assert ps(pa.PA_BF16, 8, 64, 8, 128, 8, 131073, 148) == 4096     # 128 * 17 = 2176
    # too few CTAs even at the default size: stay at 512
    assert ps(pa.PA_F32, 1, 8, 8, 64, 4, 100, 148) == 512
    assert ps(pa.PA_F32, 5, 4, 4, 64, 4, 0, 148) == 512
    # a single SM wants no split at all
    assert ps(pa.PA_BF16, 8, 64, 8, 128, 16, 131073, 1) == 262144
    # more SMs never give a longer partition
    sizes = [ps(pa.PA_BF16, 16, 32, 8, 128, 16, 65536, n) for n in (1, 16, 74, 148, 296)]
    assert sizes == sorted(sizes, reverse=True)
    assert all(s >= 512 and s % 512 == 0 and (s & (s - 1)) == 0 for s in sizes)
    # invalid arguments
    assert ps(9, 8, 64, 8, 128, 16, 1000, 148) == 0
    assert ps(pa.PA_BF16, 8, 64, 6, 128, 16, 1000, 148) == 0
    assert ps(pa.PA_BF16, 8, 64, 8, 128, 12, 1000, 148) == 0
    assert ps(pa.PA_BF16, -1, 64, 8, 128, 16, 1000, 148) == 0
    assert ps(pa.PA_BF16, 8, 64, 8, 128, 16, 1000, -2) == 0


def _decoder_config(pa, **kw):
    c = pa.pa_decoder_config_t()
    c.struct_size = ctypes.sizeof(pa.pa_decoder_config_t)
    c.k_cache = c.v_cache = 1 << 20
    c.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, c.num_heads = 64, 4, 16, 128, 8
    c.dtype = c.cache_dtype = pa.PA_BF16
    c.scale, c.k_scale, c.v_scale = 0.1, 1.0, 1.0
    c.max_blocks_per_seq, c.partition_size, c.group_members = 8, 0, 1
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_decoder_config_checks(pa):
    alloc = pa.BlockAllocator(64, 16)
    h = ctypes.c_void_p()
    create = lambda c, a=alloc._h: pa.lib.pa_decoder_create(ctypes.byref(c), a, ctypes.byref(h))
    bad = [dict(struct_size=8), dict(k_cache=0), dict(v_cache=(1 << 20) + 4), dict(num_heads=6),
           dict(dtype=9), dict(cache_dtype=pa.PA_F16), dict(dtype=pa.PA_F32,
           cache_dtype=pa.PA_FP8_E4M3), dict(partition_size=520), dict(group_members=17),
           dict(block_size=8),                                   # not the allocator's
           dict(num_blocks=32)]                                  # smaller than its pool
    for kw in bad:
        assert create(_decoder_config(pa, **kw)) == pa.PA_ERR_INVALID_ARG, kw
        assert not h.value
    assert create(_decoder_config(pa), None) == pa.PA_ERR_INVALID_ARG
    if not _has_gpu():
        # a valid configuration gets past every host check to the first CUDA call
        assert create(_decoder_config(pa)) == pa.PA_ERR_CUDA
        assert create(_decoder_config(pa, cache_dtype=pa.PA_FP8_E4M3)) == pa.PA_ERR_CUDA
        assert not h.value
    info = pa.pa_step_info_t()
    assert pa.lib.pa_decoder_bind(None, None, 0, 0, None, 0) == pa.PA_ERR_INVALID_ARG
    nbytes = ctypes.c_size_t(0)
    assert pa.lib.pa_decoder_device_bytes(None, 4, ctypes.byref(nbytes)) == pa.PA_ERR_INVALID_ARG
    assert pa.lib.pa_decoder_step(None, 0, 0, 0, 0, None, None, None,
                                  ctypes.byref(info)) == pa.PA_ERR_INVALID_ARG
    assert pa.lib.pa_decoder_wait(None, 1) == pa.PA_ERR_INVALID_ARG
    assert pa.lib.pa_decoder_query(None, None, None, None) == pa.PA_ERR_INVALID_ARG
    assert pa.lib.pa_decoder_destroy(None) == pa.PA_ERR_INVALID_ARG


def test_decode_argument_block(pa):
    a = pa.pa_decode_args_t()
    a.struct_size = ctypes.sizeof(pa.pa_decode_args_t)
    a.out = a.q = a.k_cache = a.v_cache = a.block_tables = a.seq_lens = FAKE
    a.scale, a.block_size, a.num_kv_heads, a.num_seqs, a.num_heads = 0.1, 16, 4, 0, 8
    a.head_dim, a.max_blocks_per_seq, a.num_blocks, a.max_seq_len = 128, 8, 64, 100
    a.partition_size, a.dtype, a.cache_dtype = 512, pa.PA_BF16, pa.PA_BF16
    # every field read where the library expects it: an empty batch is accepted
    assert pa.lib.pa_decode(ctypes.byref(a)) == pa.PA_OK
    for field, bad in (("struct_size", 16), ("cache_dtype", pa.PA_F16), ("head_dim", 96),
                       ("num_chunks", -1), ("partition_size", 520)):
        b = pa.pa_decode_args_t.from_buffer_copy(a)
        setattr(b, field, bad)
        assert pa.lib.pa_decode(ctypes.byref(b)) in (pa.PA_ERR_INVALID_ARG,
                                                    pa.PA_ERR_UNSUPPORTED), field
    c = pa.pa_decode_args_t.from_buffer_copy(a)
    c.num_chunks = 3                                    # groups without their arrays
    assert pa.lib.pa_decode(ctypes.byref(c)) == pa.PA_ERR_INVALID_ARG
    assert pa.lib.pa_decode(None) == pa.PA_ERR_INVALID_ARG


def _has_gpu():
    import torch
    return torch.cuda.is_available()


FAKE = 1 << 20  # an aligned, never-dereferenced pointer value: every call below fails
                # its host-side checks before any launch


def _decode(pa, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, lens=FAKE, scale=0.1, bs=16, hkv=4,
             S=2, hq=4, D=128, mb=8, nb=64, max_len=100, ps=512, dtype=pa.PA_BF16, ws=None,
             wsb=0)
    a.update(kw)
    return pa.lib.pa_decode_attention(a["out"], a["q"], a["k"], a["v"], a["tables"], a["lens"],
                                      a["scale"], a["bs"], a["hkv"], a["S"], a["hq"], a["D"],
                                      a["mb"], a["nb"], a["max_len"], a["ps"], a["dtype"],
                                      a["ws"], a["wsb"], None)


def test_decode_argument_checks(pa):
    assert _decode(pa, dtype=9) == pa.PA_ERR_INVALID_ARG
    assert _decode(pa, D=96) == pa.PA_ERR_UNSUPPORTED
    assert _decode(pa, bs=12) == pa.PA_ERR_UNSUPPORTED
    assert _decode(pa, hq=6, hkv=4) == pa.PA_ERR_INVALID_ARG
    assert _decode(pa, ps=520) == pa.PA_ERR_INVALID_ARG          # not a multiple of 16
    assert _decode(pa, q=FAKE + 4) == pa.PA_ERR_INVALID_ARG     # misaligned
    assert _decode(pa, tables=None) == pa.PA_ERR_INVALID_ARG
    assert _decode(pa, max_len=5000) == pa.PA_ERR_INVALID_ARG   # needs a workspace
    assert _decode(pa, max_len=5000, ws=FAKE, wsb=16) == pa.PA_ERR_INVALID_ARG  # too small
    assert _decode(pa, S=0) == pa.PA_OK                          # nothing to do


def _copy(pa, pairs, nb=16):
    host = np.ascontiguousarray(pairs, dtype=np.int32)
    return pa.lib.pa_copy_blocks(FAKE, FAKE, FAKE, host.ctypes.data, len(host), 2, 64, 16, nb,
                                 pa.PA_BF16, None)


def test_copy_blocks_mapping_checks(pa):
    assert _copy(pa, [(1, 2), (1, 2)]) == pa.PA_ERR_INVALID_ARG    # dst repeats
    assert _copy(pa, [(1, 2), (2, 3)]) == pa.PA_ERR_INVALID_ARG    # dst is also a src
    assert _copy(pa, [(1, 16)]) == pa.PA_ERR_INVALID_ARG           # outside the pool
    assert _copy(pa, [(-1, 3)]) == pa.PA_ERR_INVALID_ARG
    assert pa.lib.pa_copy_blocks(FAKE, FAKE, FAKE, None, 0, 2, 64, 16, 16, pa.PA_BF16,
                                 None) == pa.PA_OK                 # no pairs: no-op


def test_reshape_argument_checks(pa):
    f = pa.lib.pa_reshape_and_cache
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 6, 16, 8, pa.PA_BF16, None) == \
        pa.PA_ERR_INVALID_ARG                                       # 12-byte rows
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 5, None) == pa.PA_ERR_INVALID_ARG
    assert f(None, None, None, None, None, 0, 2, 64, 16, 8, pa.PA_F16, None) == pa.PA_OK


def test_importing_without_library_fails_loudly(tmp_path):
    """The binding refuses to load rather than fall back to anything else."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "paged_kv_cache_342_b200")
    dst = tmp_path / "paged_kv_cache_342_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "_build", "__pycache__"))
    r = subprocess.run([sys.executable, "-c", "import paged_kv_cache_342_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libpa.so is missing" in r.stderr


def test_plain_c_program_builds_and_runs(tmp_path):
    # the header is C99 (no C++ in it) and the host-only calls work from C
    import shutil
    import subprocess
    import paged_kv_cache_342_b200 as m
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_consumer"
    libdir = os.path.dirname(m.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_consumer.c"), "-L", libdir, "-lpa",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.strip()
    # pool order 0, 1, ...: seq 7 holds blocks 0, 1; the fork's append copies block 1
    # into the next free block, 2, at offset 1 (slot 9)
    assert out == ("rc=0 slot=9 copy=1->2 used=3 shared=1 ps=4096 bad=1"), out
