"""Swapping sequences to a page-locked host pool and back (preemption by swapping):
the block manager moves the sequences, pa_swap_blocks copies their blocks, and after
the round trip attention is bit-identical to before - with the freed device blocks
overwritten by another sequence in between."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as oatt
from gpu_util import TORCH_DT, assert_close, out_f64, to_dev, to_host
from workloads import normal_fill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    assert torch.cuda.is_available()
    m.pa_device_error_read()
    return m


def _decode(pa, kd, vd, alloc, ids, q, bs, Hkv, dtype):
    tables, lens = alloc.build_block_tables(ids, 16)
    out = torch.full(q.shape, float("nan"), dtype=q.dtype, device="cuda")
    max_len = int(lens.max())
    wsb = pa.pa_decode_workspace_bytes(len(ids), q.shape[1], q.shape[2], max_len, 64)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    pa.pa_decode_attention(out, q, kd, vd, torch.from_numpy(tables).cuda(),
                           torch.from_numpy(lens).cuda(), 1 / math.sqrt(q.shape[2]), bs, Hkv,
                           max_len, 64, ws if wsb else None)
    torch.cuda.synchronize()
    return out, tables, lens


@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", [("bf16", 4, 4, 128, 16), ("f16", 16, 2, 64, 16),
                                              ("f32", 2, 2, 64, 8)])
def test_swap_round_trip_through_a_host_pool(pa, dtype, Hq, Hkv, D, bs):
    NBd, NBh = 48, 24
    lens = [100, 40, 17, 64]
    g = np.random.default_rng(5)
    dev = pa.BlockAllocator(NBd, bs, g.permutation(NBd))
    host = pa.BlockAllocator(NBh, bs, g.permutation(NBh))
    for s, L in enumerate(lens):
        dev.add(s, L)
    dev.fork(1, 7)                                   # seq 7 shares seq 1's blocks
    k = normal_fill((NBd, Hkv, bs, D), dtype, 1.0, 6, 1)
    v = normal_fill((NBd, Hkv, bs, D), dtype, 1.0, 6, 2)
    kd, vd = to_dev(k, dtype), to_dev(v, dtype)
    kh = torch.zeros((NBh, Hkv, bs, D), dtype=TORCH_DT[dtype]).pin_memory()
    vh = torch.zeros_like(kh).pin_memory()
    ids = [0, 1, 2, 3, 7]
    q = to_dev(normal_fill((len(ids), Hq, D), dtype, 1.0, 6, 3), dtype)
    before, tables0, lens0 = _decode(pa, kd, vd, dev, ids, q, bs, Hkv, dtype)

    # swap out sequences 1 and 3 (seq 7 stays: the shared blocks are copied, not moved)
    pairs = dev.move_to(host, [1, 3])
    mapping = torch.from_numpy(pairs.copy()).cuda()
    pa.pa_swap_blocks(kh, vh, kd, vd, mapping, pairs)
    torch.cuda.synchronize()
    for src, dst in pairs:
        assert np.array_equal(to_host(kh[dst], dtype), k[src])
        assert np.array_equal(to_host(vh[dst], dtype), v[src])

    # the freed device blocks are reused and overwritten by someone else
    freed = dev.free_list()
    dev.add(50, len(freed) * bs)
    junk = torch.tensor(dev.seq_blocks(50), device="cuda")
    kd.index_fill_(0, junk, 3.0)
    vd.index_fill_(0, junk, -3.0)
    dev.free(50)

    # swap back in (mapping given in pinned host memory this time)
    back = host.move_to(dev, [1, 3])
    mapping_h = torch.from_numpy(back.copy()).pin_memory()
    pa.pa_swap_blocks(kd, vd, kh, vh, mapping_h, back)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    after, tables1, lens1 = _decode(pa, kd, vd, dev, ids, q, bs, Hkv, dtype)
    assert np.array_equal(lens0, lens1)
    assert not np.array_equal(tables0[[1, 3]], tables1[[1, 3]])   # new physical blocks
    assert torch.equal(before, after)                                # same bits
    want = oatt.paged_decode_attention(to_host(q, dtype), to_host(kd, dtype), to_host(vd, dtype),
                                       tables1, lens1, 1 / math.sqrt(D), bs, Hkv, dtype)
    assert_close(out_f64(after), want, dtype, "after swap")


def test_swap_rejects_pageable_host_memory(pa):
    kd = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16, device="cuda")
    kh = torch.zeros((4, 2, 16, 64), dtype=torch.bfloat16)          # not pinned
    pairs = np.array([[0, 1]], np.int32)
    m = torch.from_numpy(pairs).cuda()
    with pytest.raises(ValueError):
        pa.pa_swap_blocks(kh, kh, kd, kd, m, pairs)                  # caught by the binding
    rc = pa.lib.pa_swap_blocks(kh.data_ptr(), kh.data_ptr(), 4, kd.data_ptr(), kd.data_ptr(), 4,
                               m.data_ptr(), pairs.ctypes.data, 1, 2, 64, 16, pa.PA_BF16, None)
    assert rc == pa.PA_ERR_INVALID_ARG                               # and by the library
    assert kh.abs().sum() == 0
