"""Automatic prefix caching end to end: a second request with the same prompt
reuses the cached blocks, writes K/V only for its own tokens, and attends to exactly
what it would have seen without the cache (bit-identical output), which also matches
the float64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as oatt
from gpu_util import assert_close, out_f64, to_dev, to_host
from workloads import normal_fill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    assert torch.cuda.is_available()
    m.pa_device_error_read()
    return m


def _slots(alloc, sid, first, last, bs):
    blocks = alloc.seq_blocks(sid)
    return np.array([blocks[t // bs] * bs + t % bs for t in range(first, last)], np.int64)


def _admit_and_write(pa, alloc, kd, vd, sid, tokens, kv_of_token, bs, use_cache):
    if use_cache:
        cached = alloc.add_prompt(sid, tokens)
    else:
        alloc.add(sid, len(tokens))
        cached = 0
    n = len(tokens)
    if n > cached:
        slots = _slots(alloc, sid, cached, n, bs)
        k, v = kv_of_token(tokens[cached:])
        pa.pa_reshape_and_cache(k, v, kd, vd, torch.from_numpy(slots).cuda())
    return cached


def test_second_request_reuses_the_prompt_blocks(pa):
    Hq = Hkv = 4
    D, bs, NB = 128, 16, 64
    vocab = 97
    table_k = to_dev(normal_fill((vocab, Hkv, D), "bf16", 1.0, 31, 1), "bf16")
    table_v = to_dev(normal_fill((vocab, Hkv, D), "bf16", 1.0, 31, 2), "bf16")

    def kv_of_token(toks):   # K/V of a token = a fixed row per token id (position-free)
        idx = torch.tensor(toks, device="cuda")
        return table_k[idx].contiguous(), table_v[idx].contiguous()

    g = np.random.default_rng(31)
    prompt = g.integers(0, vocab, 70).tolist()
    second = prompt + g.integers(0, vocab, 5).tolist()
    q = to_dev(normal_fill((2, Hq, D), "bf16", 1.0, 31, 3), "bf16")
    outs = []
    for use_cache in (True, False):
        alloc = pa.BlockAllocator(NB, bs, g.permutation(NB))
        kd = torch.zeros((NB, Hkv, bs, D), dtype=torch.bfloat16, device="cuda")
        vd = torch.zeros_like(kd)
        c0 = _admit_and_write(pa, alloc, kd, vd, 0, prompt, kv_of_token, bs, use_cache)
        c1 = _admit_and_write(pa, alloc, kd, vd, 1, second, kv_of_token, bs, use_cache)
        if use_cache:
            assert (c0, c1) == (0, 64)                  # 4 full blocks of the prompt
            assert alloc.seq_blocks(0)[:4] == alloc.seq_blocks(1)[:4]
            assert alloc.stats()["cache_hits"] == 4
        tables, lens = alloc.build_block_tables([0, 1], 8)
        out = torch.empty((2, Hq, D), dtype=torch.bfloat16, device="cuda")
        pa.pa_decode_attention(out, q, kd, vd, torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens).cuda(), 1 / math.sqrt(D), bs, Hkv,
                               int(lens.max()), 512, None)
        torch.cuda.synchronize()
        outs.append(out)
        if use_cache:
            want = oatt.paged_decode_attention(to_host(q, "bf16"), to_host(kd, "bf16"),
                                               to_host(vd, "bf16"), tables, lens, 1 / math.sqrt(D),
                                               bs, Hkv, "bf16")
            assert_close(out_f64(out), want, "bf16", "cached prompt")
    assert torch.equal(outs[0], outs[1])
    assert pa.pa_device_error_read() == 0
