"""The allocation-free decode entry point (pa_decode_attention_static_ws) against the
regular one.

Some callers may not allocate device memory at all - a host program that owns and
budgets every byte of the GPU, a plug-in inside another process, a loop that cannot
pay for cudaMalloc.  For them the library keeps its own fixed scratch array.  These
tests call that entry point through the C ABI and check that it gives the same
result as pa_decode_attention with a caller workspace, bit for bit, on two calls in
a row (the array keeps the previous call's contents), for the CUDA-core and the
tensor-core kernels; that a smaller call after a larger one reads none of the stale
scratch; and that an oversized request is refused without touching anything.

This file is collected last on purpose: a failure here leaves every other test run.
"""
import math

import numpy as np
import pytest
import torch

from gpu_util import TORCH_DT, out_f64, tables_from_order, to_dev
from workloads import normal_fill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    assert torch.cuda.is_available()
    return m


@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs,ps", [
    ("bf16", 8, 8, 128, 16, 128),      # CUDA-core kernel, several partitions
    ("f16", 16, 2, 128, 16, 64),       # tensor-core kernel
    ("f32", 4, 4, 64, 4, 32),
])
def test_static_workspace_matches_caller_workspace(pa, dtype, Hq, Hkv, D, bs, ps):
    lens = np.array([1, 100, 1500, 700, 2048, 33], np.int64)
    S = lens.size
    NB = int(sum(-(-int(L) // bs) for L in lens)) + 3
    k = to_dev(normal_fill((NB, Hkv, bs, D), dtype, 1.0, 21, 1), dtype)
    v = to_dev(normal_fill((NB, Hkv, bs, D), dtype, 1.0, 21, 2), dtype)
    order = np.random.default_rng(21).permutation(NB).astype(np.int32)
    width = -(-int(lens.max()) // bs) + 1
    tables = torch.from_numpy(tables_from_order(lens, bs, order, width)).cuda()
    seq_lens = torch.from_numpy(lens.astype(np.int32)).cuda()
    max_len = int(lens.max())
    wsb = pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps)
    assert 0 < wsb <= pa.PA_STATIC_WORKSPACE_BYTES
    scale = 1.0 / math.sqrt(D)
    for call in range(2):      # two calls in a row, different queries
        q = to_dev(normal_fill((S, Hq, D), dtype, 1.0, 21, 10 + call), dtype)
        ref = torch.empty((S, Hq, D), dtype=TORCH_DT[dtype], device="cuda")
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        pa.pa_decode_attention(ref, q, k, v, tables, seq_lens, scale, bs, Hkv, max_len, ps, ws)
        got = torch.full((S, Hq, D), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
        pa.pa_decode_attention_static_ws(got, q, k, v, tables, seq_lens, scale, bs, Hkv,
                                         max_len, ps)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        # the same kernels on the same inputs with the same scratch layout: bit for bit
        assert torch.equal(got, ref), f"call {call}"
    assert pa.pa_device_error_read() == 0


def _case(dtype, Hq, Hkv, D, bs, lens, seed):
    lens = np.asarray(lens, np.int64)
    NB = int(sum(-(-int(L) // bs) for L in lens)) + 3
    k_h = normal_fill((NB, Hkv, bs, D), dtype, 1.0, seed, 1)
    v_h = normal_fill((NB, Hkv, bs, D), dtype, 1.0, seed, 2)
    q_h = normal_fill((lens.size, Hq, D), dtype, 1.0, seed, 3)
    order = np.random.default_rng(seed).permutation(NB).astype(np.int32)
    width = -(-int(lens.max()) // bs) + 1
    tables = tables_from_order(lens, bs, order, width)
    return lens, k_h, v_h, q_h, tables


def test_stale_scratch_of_a_larger_call_does_not_leak(pa):
    """A first call with many partitions fills much of the shared array; a second,
    smaller call of another shape must not read any of it: its output equals the
    caller-workspace call bit for bit and the float64 oracle within tolerance."""
    import oracle.attention as oatt
    from gpu_util import assert_close
    dtype, D, bs = "bf16", 128, 16
    calls = [
        # 12 x 16 heads x 63 partitions of 32 tokens: about 6.5 MB of partials
        dict(Hq=16, Hkv=16, lens=[2000, 1999, 1500, 1024, 777, 2016, 1800, 640, 1300,
                                  2001, 999, 1234], ps=32, seed=31),
        # 5 sequences x 8 heads (tensor cores, group 8), 512-token partitions
        dict(Hq=8, Hkv=1, lens=[3000, 1, 513, 1024, 2047], ps=512, seed=32),
    ]
    for i, c in enumerate(calls):
        lens, k_h, v_h, q_h, tables = _case(dtype, c["Hq"], c["Hkv"], D, bs, c["lens"],
                                            c["seed"])
        S, Hq, Hkv = lens.size, c["Hq"], c["Hkv"]
        k, v, q = to_dev(k_h, dtype), to_dev(v_h, dtype), to_dev(q_h, dtype)
        t = torch.from_numpy(tables).cuda()
        sl = torch.from_numpy(lens.astype(np.int32)).cuda()
        max_len, scale = int(lens.max()), 1.0 / math.sqrt(D)
        wsb = pa.pa_decode_workspace_bytes(S, Hq, D, max_len, c["ps"])
        assert 0 < wsb <= pa.PA_STATIC_WORKSPACE_BYTES
        ref = torch.empty((S, Hq, D), dtype=TORCH_DT[dtype], device="cuda")
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        pa.pa_decode_attention(ref, q, k, v, t, sl, scale, bs, Hkv, max_len, c["ps"], ws)
        got = torch.full_like(ref, float("nan"))
        pa.pa_decode_attention_static_ws(got, q, k, v, t, sl, scale, bs, Hkv, max_len, c["ps"])
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {i}"
        want = oatt.paged_decode_attention(q_h, k_h, v_h, tables, lens, scale, bs, Hkv, dtype)
        assert_close(out_f64(got), want, dtype, f"call {i}")
    assert pa.pa_device_error_read() == 0


def test_static_workspace_refuses_oversized_requests(pa):
    # 256 sequences x 40 heads x 8 partitions of 512 at head_dim 128 need ~42 MB of
    # scratch: refused before any pointer is used (these pointers are never touched)
    fake = 1 << 20
    need = pa.pa_decode_workspace_bytes(256, 40, 128, 4096, 512)
    assert need > pa.PA_STATIC_WORKSPACE_BYTES
    rc = pa.lib.pa_decode_attention_static_ws(fake, fake, fake, fake, fake, fake, 0.1, 16, 40,
                                              256, 40, 128, 256, 16384, 4096, 512, pa.PA_F16,
                                              None)
    assert rc == pa.PA_ERR_TOO_LARGE
