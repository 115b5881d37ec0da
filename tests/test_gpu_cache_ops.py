"""GPU parity of the cache kernels against the oracle: bit-exact over the entire
cache tensors (untouched slots included), plus the device error word."""
import numpy as np
import pytest
import torch

import oracle.cache_ops as ocache
from gpu_util import to_dev, to_host
from workloads import CONFIGS, make_inputs, normal_fill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    assert torch.cuda.is_available()
    m.pa_device_error_read()
    return m


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("D,bs,Hkv,T", [(64, 4, 4, 37), (128, 16, 32, 256), (256, 32, 2, 5)])
def test_reshape_and_cache_bit_exact(pa, dtype, D, bs, Hkv, T):
    NB = 48
    k = normal_fill((NB, Hkv, bs, D), dtype, 1.0, 1, 1)
    v = normal_fill((NB, Hkv, bs, D), dtype, 1.0, 1, 2)
    key = normal_fill((T, Hkv, D), dtype, 1.0, 1, 3)
    val = normal_fill((T, Hkv, D), dtype, 1.0, 1, 4)
    slots = np.random.default_rng(T).choice(NB * bs, T, replace=False).astype(np.int64)
    slots[T // 2] = -1
    kd, vd = to_dev(k, dtype), to_dev(v, dtype)
    pa.pa_reshape_and_cache(to_dev(key, dtype), to_dev(val, dtype), kd, vd,
                            torch.from_numpy(slots).cuda())
    ocache.reshape_and_cache(key, val, k, v, slots, bs)
    assert np.array_equal(to_host(kd, dtype), k)
    assert np.array_equal(to_host(vd, dtype), v)
    assert pa.pa_device_error_read() == 0


def test_reshape_and_cache_no_tokens(pa):
    k = torch.zeros((4, 2, 4, 64), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    e = torch.empty((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    pa.pa_reshape_and_cache(e, e, k, v, torch.empty(0, dtype=torch.int64, device="cuda"))
    assert not k.any() and not v.any()


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_copy_blocks_bit_exact(pa, dtype):
    NB, Hkv, bs, D = 64, 3, 8, 64
    k = normal_fill((NB, Hkv, bs, D), dtype, 1.0, 2, 1)
    v = normal_fill((NB, Hkv, bs, D), dtype, 1.0, 2, 2)
    # sources repeat (one shared block copied for several writers), destinations do not
    pairs = np.array([(5, 40), (5, 41), (5, 42), (7, 50), (0, 63), (12, 1)], np.int32)
    kd, vd = to_dev(k, dtype), to_dev(v, dtype)
    pa.pa_copy_blocks(kd, vd, torch.from_numpy(pairs).cuda(), pairs)
    ocache.copy_blocks(k, v, pairs)
    assert np.array_equal(to_host(kd, dtype), k)
    assert np.array_equal(to_host(vd, dtype), v)


def test_copy_blocks_fork_step_full_pool(pa):
    """The shared-prefix fork step's 224 copies on the full 8192-block bf16 pool."""
    from oracle.step import build_context
    cfg = CONFIGS["prefix_cow_bf16"]
    inp = make_inputs(cfg, 0, fork_step=True)
    kd, vd = to_dev(inp.k_pool, "bf16"), to_dev(inp.v_pool, "bf16")
    bm, k, v, _ = build_context(inp, copy_pool=False)
    res = bm.append_slots(range(cfg.num_seqs))
    pairs = np.array([(r[1], r[2]) for r in res if r[1] >= 0], np.int32)
    assert len(pairs) == 224
    pa.pa_copy_blocks(kd, vd, torch.from_numpy(pairs).cuda(), pairs)
    ocache.copy_blocks(k, v, pairs)
    assert np.array_equal(to_host(kd, "bf16"), k)
    assert np.array_equal(to_host(vd, "bf16"), v)


def test_out_of_range_slot_is_skipped_and_reported(pa):
    NB, Hkv, bs, D = 8, 2, 4, 64
    k = normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 3, 1)
    key = normal_fill((3, Hkv, D), "bf16", 1.0, 3, 2)
    slots = np.array([1, NB * bs + 5, 9], np.int64)
    kd, vd = to_dev(k, "bf16"), to_dev(k, "bf16")
    pa.pa_reshape_and_cache(to_dev(key, "bf16"), to_dev(key, "bf16"), kd, vd,
                            torch.from_numpy(slots).cuda())
    assert pa.pa_device_error_read() == pa.DEVERR_SLOT
    want = k.copy()
    ocache.reshape_and_cache(key[[0, 2]], key[[0, 2]], want, want.copy(), slots[[0, 2]], bs)
    assert np.array_equal(to_host(kd, "bf16"), want)
    assert pa.pa_device_error_read() == 0       # read clears


def test_out_of_range_copy_pair_is_skipped_and_reported(pa):
    NB, Hkv, bs, D = 8, 2, 4, 64
    k = normal_fill((NB, Hkv, bs, D), "f16", 1.0, 4, 1)
    kd, vd = to_dev(k, "f16"), to_dev(k, "f16")
    pairs = np.array([(1, 2), (3, NB)], np.int32)   # second dst outside the pool
    pa.pa_copy_blocks(kd, vd, torch.from_numpy(pairs).cuda(), None)   # no host check
    assert pa.pa_device_error_read() == pa.DEVERR_COPY_BLOCK
    want = k.copy()
    want[2] = k[1]
    assert np.array_equal(to_host(kd, "f16"), want)
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_copy_blocks(kd, vd, torch.from_numpy(pairs).cuda(), pairs)   # host check
