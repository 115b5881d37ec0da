"""The runtime's host-buffer step (copies on their own streams, overlapped with the
neighbouring steps) gives exactly the results of the device-buffer step."""
import math

import numpy as np
import pytest
import torch

from gpu_util import to_dev
from workloads import normal_fill

pytestmark = pytest.mark.gpu


def _decoder(pa_rt, seed=0):
    S, Hq, Hkv, D, bs, NB = 6, 8, 8, 128, 16, 128
    g = np.random.default_rng(seed)
    kd = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, seed, 1), "bf16")
    vd = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, seed, 2), "bf16")
    dec = pa_rt.PagedDecoder(kd, vd, Hq, 1 / math.sqrt(D), 24, g.permutation(NB), 64)
    for s in range(S):
        dec.admit(s, int(g.integers(30, 300)))
    dec.bind(range(S), rolling=True)
    return dec, (S, Hq, Hkv, D)


def test_host_buffer_steps_match_device_steps():
    import paged_kv_cache_342_b200.runtime as rt
    steps = 5
    ref_dec, (S, Hq, Hkv, D) = _decoder(rt)
    host_dec, _ = _decoder(rt)
    toks = [[normal_fill(shape, "bf16", 1.0, 50 + i, j)
             for j, shape in enumerate(((S, Hq, D), (S, Hkv, D), (S, Hkv, D)))]
            for i in range(steps)]
    refs = []
    for i in range(steps):
        out = torch.empty((S, Hq, D), dtype=torch.bfloat16, device="cuda")
        ref_dec.step(*[to_dev(a, "bf16") for a in toks[i]], out)
        refs.append(out)
    outs_h = [torch.empty((S, Hq, D), dtype=torch.bfloat16, pin_memory=True)
              for _ in range(steps)]
    pinned = [[to_dev(a, "bf16").cpu().pin_memory() for a in t] for t in toks]
    events = [host_dec.step_host(*pinned[i], outs_h[i]) for i in range(steps)]
    for i in range(steps):
        events[i].synchronize()
        assert torch.equal(outs_h[i], refs[i].cpu()), f"step {i}"


def test_rolling_and_growing_steps_rebind_and_partition_choice():
    import paged_kv_cache_342_b200 as pa
    import paged_kv_cache_342_b200.runtime as rt
    import oracle.attention as oatt
    from gpu_util import assert_close, out_f64, to_host
    S, Hq, Hkv, D, bs, NB, MB = 6, 16, 2, 128, 16, 256, 40
    g = np.random.default_rng(3)
    kd = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 3, 1), "bf16")
    vd = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 3, 2), "bf16")
    dec = rt.PagedDecoder(kd, vd, Hq, 1 / math.sqrt(D), MB, g.permutation(NB), 0)
    lens0 = g.integers(40, 500, S)
    for s in range(S):
        dec.admit(s, int(lens0[s]))
    dec.bind(range(S), rolling=True)
    assert dec.partition_size == pa.pa_decode_partition_size(pa.PA_BF16, S, Hq, Hkv, D, bs,
                                                             MB * bs)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    def step(n, events=None):
        q, k, v = (to_dev(normal_fill(sh, "bf16", 1.0, 60 + n, j), "bf16")
                   for j, sh in enumerate(((n, Hq, D), (n, Hkv, D), (n, Hkv, D))))
        out = torch.empty((n, Hq, D), dtype=torch.bfloat16, device="cuda")
        meta = dec.step(q, k, v, out, events=events)
        return meta, q, out

    for _ in range(3):                                   # rolling: the same lengths
        meta, _, _ = step(S, ev)
        assert np.array_equal(meta.lens, lens0 + 1)
    torch.cuda.synchronize()
    assert ev[0].elapsed_time(ev[1]) > 0

    dec.bind([4, 1, 2], rolling=False)                   # a smaller batch, growing
    for i in range(3):
        meta, q, out = step(3)
        assert np.array_equal(meta.lens, lens0[[4, 1, 2]] + 2 + i)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    want = oatt.paged_decode_attention(to_host(q, "bf16"), to_host(kd, "bf16"),
                                       to_host(vd, "bf16"), meta.tables.copy(),
                                       meta.lens.copy(), 1 / math.sqrt(D), bs, Hkv, "bf16")
    assert_close(out_f64(out), want, "bf16", "after rebind")

    dec.bind(range(S), rolling=False)                    # back to the larger batch
    meta, q, out = step(S)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    assert meta.kernels == 2 + (1 if -(-meta.max_len // dec.partition_size) > 1 else 0)
    with pytest.raises(ValueError):                      # tensors must fit the batch
        dec.step(q[:2], q[:2, :Hkv], q[:2, :Hkv], out[:2])


def test_caller_buffer_and_capacity_refusal_leave_state_unchanged():
    """The decoder takes its device memory from the caller: a bind with a buffer that
    is too small (or misaligned) is refused and changes nothing.  A growing batch whose
    sequence reaches the table's capacity is refused before the block manager commits
    the step: lengths, tables and the pool stay as they were, and a rebind with more
    room lets the batch go on."""
    import ctypes

    import paged_kv_cache_342_b200 as pa
    import paged_kv_cache_342_b200.runtime as rt
    S, Hq, Hkv, D, bs, NB, MB = 2, 8, 8, 128, 16, 64, 4        # capacity 64 tokens
    kd = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 4, 1), "bf16")
    vd = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 4, 2), "bf16")
    dec = rt.PagedDecoder(kd, vd, Hq, 1 / math.sqrt(D), MB, None, 32)
    dec.admit(0, 61)
    dec.admit(1, 10)
    need = ctypes.c_size_t(0)
    assert pa.lib.pa_decoder_device_bytes(dec._h, S, ctypes.byref(need)) == pa.PA_OK
    small = torch.empty(need.value - 256, dtype=torch.uint8, device="cuda")
    ids = np.arange(S, dtype=np.int64)
    assert pa.lib.pa_decoder_bind(dec._h, ids.ctypes.data, S, 0, small.data_ptr(),
                                  small.numel()) == pa.PA_ERR_INVALID_ARG
    big = torch.empty(need.value + 512, dtype=torch.uint8, device="cuda")
    assert pa.lib.pa_decoder_bind(dec._h, ids.ctypes.data, S, 0, big.data_ptr() + 16,
                                  need.value) == pa.PA_ERR_INVALID_ARG
    dec.bind(range(S), rolling=False)
    q = torch.randn(S, Hq, D, device="cuda").bfloat16()
    kv = torch.randn(S, Hkv, D, device="cuda").bfloat16()
    out = torch.empty_like(q)
    for _ in range(3):                                   # 61 -> 64 tokens: at capacity
        dec.step(q, kv, kv, out)
    torch.cuda.synchronize()
    before = (dec.alloc.stats(), dec.alloc.free_list(), dec.alloc.seq_blocks(0),
              dec.alloc.seq_len(0), dec.alloc.seq_len(1))
    assert before[3] == 64
    with pytest.raises(pa.PagedAttentionError) as e:
        dec.step(q, kv, kv, out)
    assert e.value.code == "INVALID_ARG"
    after = (dec.alloc.stats(), dec.alloc.free_list(), dec.alloc.seq_blocks(0),
             dec.alloc.seq_len(0), dec.alloc.seq_len(1))
    assert after == before
    dec.bind([1], rolling=False)                         # the other sequence goes on
    meta = dec.step(q[:1], kv[:1], kv[:1], out[:1])
    torch.cuda.synchronize()
    assert int(meta.lens[0]) == 14 and pa.pa_device_error_read() == 0
