"""GPU parity of pa_decode_attention against the float64 oracle on small cases that
cover both kernels (CUDA-core and tensor-core), every dtype, head_dim 64/128/256,
block sizes 4-32, several partitions with ragged tails, empty and one-token
sequences, NaN in unused slots, and the device error word."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as oatt
from gpu_util import (NAN_BITS, PA_CODE, TORCH_DT, assert_close, blocks_for, out_f64,
                      tables_from_order, to_dev)
from workloads import normal_fill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    assert torch.cuda.is_available()
    m.pa_device_error_read()
    return m


def run_case(pa, dtype, Hq, Hkv, D, bs, ps, lens, seed=0, nan_unused=False, extra_blocks=5):
    lens = np.asarray(lens, np.int64)
    S = len(lens)
    NB = int(sum(blocks_for(L, bs) for L in lens)) + extra_blocks
    std = 1.0
    k = normal_fill((NB, Hkv, bs, D), dtype, std, seed, 11)
    v = normal_fill((NB, Hkv, bs, D), dtype, std, seed, 12)
    q = normal_fill((S, Hq, D), dtype, std, seed, 13)
    order = np.random.default_rng([seed, 5]).permutation(NB).astype(np.int32)
    width = max(1, int(max(blocks_for(L, bs) for L in lens))) + 1
    tables = tables_from_order(lens, bs, order, width)
    if nan_unused:
        used = np.zeros((NB, bs), bool)
        for s, L in enumerate(lens):
            for t in range(int(L)):
                used[tables[s, t // bs], t % bs] = True
        for arr in (k, v):
            arr.transpose(0, 2, 1, 3)[~used] = NAN_BITS[dtype]
    scale = 1.0 / math.sqrt(D)
    max_len = int(lens.max()) if S else 0
    out = torch.full((S, Hq, D), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
    wsb = pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda") if wsb else None
    pa.pa_decode_attention(out, to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype),
                           torch.from_numpy(tables).cuda(),
                           torch.from_numpy(lens.astype(np.int32)).cuda(), scale, bs, Hkv,
                           max_len, ps, ws)
    torch.cuda.synchronize()
    want = oatt.paged_decode_attention(q, k, v, tables, lens, scale, bs, Hkv, dtype)
    got = out_f64(out)
    assert pa.pa_device_error_read() == 0
    return got, want


LENS_A = (0, 1, 3, 15, 16, 17, 64, 65, 200, 333)
CASES = [
    # dtype, Hq, Hkv, D, bs, partition, lens
    ("f32", 4, 4, 64, 4, 512, (5, 13, 7, 18, 10)),          # tiny workload shape
    ("f32", 4, 4, 64, 4, 8, (5, 13, 7, 18, 10)),            # same, many partitions
    ("bf16", 4, 4, 128, 16, 64, LENS_A),
    ("f16", 3, 3, 128, 16, 32, LENS_A),
    ("bf16", 2, 2, 64, 8, 16, LENS_A),
    ("f16", 8, 2, 64, 8, 32, LENS_A),                       # group 4, CUDA cores
    ("bf16", 6, 3, 128, 32, 64, LENS_A),                    # group 2
    ("f32", 16, 2, 128, 16, 48, LENS_A),                    # group 8, fp32: CUDA cores
    ("bf16", 2, 2, 256, 8, 64, LENS_A),
    ("f32", 2, 1, 256, 32, 64, LENS_A),
    ("bf16", 16, 2, 128, 16, 64, LENS_A),                   # tensor cores, group 8
    ("f16", 16, 2, 128, 16, 512, LENS_A),
    ("bf16", 32, 2, 64, 32, 128, LENS_A),                   # tensor cores, group 16
    ("f16", 8, 1, 256, 16, 64, LENS_A),                     # tensor cores, head_dim 256
    ("bf16", 16, 1, 256, 32, 512, (1, 31, 32, 33, 700)),
    ("bf16", 16, 2, 64, 16, 32, (2000, 1, 513)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-h{c[1]}/{c[2]}-d{c[3]}-b{c[4]}-p{c[5]}")
def test_small_cases(pa, case):
    dtype, Hq, Hkv, D, bs, ps, lens = case
    got, want = run_case(pa, dtype, Hq, Hkv, D, bs, ps, lens)
    assert_close(got, want, dtype, str(case))


@pytest.mark.parametrize("case", [CASES[2], CASES[5], CASES[10], CASES[12]],
                         ids=["mha", "gqa4", "tc8", "tc16"])
def test_nan_in_unused_slots_is_never_used(pa, case):
    dtype, Hq, Hkv, D, bs, ps, lens = case
    got, want = run_case(pa, dtype, Hq, Hkv, D, bs, ps, lens, nan_unused=True)
    assert_close(got, want, dtype, "nan-filled pool")


@pytest.mark.parametrize("tc", [False, True])
def test_partition_size_does_not_change_the_result(pa, tc):
    Hq, Hkv = (16, 2) if tc else (4, 4)
    lens = (1000, 17, 512, 513)
    outs = []
    for ps in (16, 64, 512, 1024):
        got, want = run_case(pa, "bf16", Hq, Hkv, 128, 16, ps, lens, seed=7)
        assert_close(got, want, "bf16", f"partition {ps}")
        outs.append(got)
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2e-2


def test_all_empty_sequences_give_zeros(pa):
    got, _ = run_case(pa, "bf16", 4, 4, 128, 16, 512, (0, 0, 0))
    assert np.array_equal(got, np.zeros_like(got))


def test_out_of_range_table_entry_is_skipped_and_reported(pa):
    for Hq, Hkv in ((4, 4), (16, 2)):
        S, D, bs, NB = 2, 128, 16, 16
        k = normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 9, 1)
        q = normal_fill((S, Hq, D), "bf16", 1.0, 9, 2)
        tables = np.array([[3, 5, NB + 7], [1, -4, 2]], np.int32)
        lens = np.array([40, 40], np.int32)
        out = torch.empty((S, Hq, D), dtype=torch.bfloat16, device="cuda")
        kd = to_dev(k, "bf16")
        pa.pa_decode_attention(out, to_dev(q, "bf16"), kd, kd, torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens).cuda(), 0.1, bs, Hkv, 40, 512, None)
        assert pa.pa_device_error_read() == pa.DEVERR_TABLE
        assert torch.isfinite(out).all()


def test_length_beyond_bound_is_skipped_and_reported(pa):
    S, Hq, Hkv, D, bs, NB = 2, 4, 4, 64, 16, 8
    k = normal_fill((NB, Hkv, bs, D), "f16", 1.0, 10, 1)
    q = normal_fill((S, Hq, D), "f16", 1.0, 10, 2)
    tables = np.array([[0, 1], [2, 3]], np.int32)
    lens = np.array([20, 30], np.int32)
    out = torch.empty((S, Hq, D), dtype=torch.float16, device="cuda")
    kd = to_dev(k, "f16")
    # max_seq_len 25 < 30: sequence 1 is treated as empty and reported
    pa.pa_decode_attention(out, to_dev(q, "f16"), kd, kd, torch.from_numpy(tables).cuda(),
                           torch.from_numpy(lens).cuda(), 0.125, bs, Hkv, 25, 512, None)
    assert pa.pa_device_error_read() == pa.DEVERR_SEQ_LEN
    assert not out[1].any()
    want = oatt.paged_decode_attention(q[:1], k, k, tables[:1], lens[:1], 0.125, bs, Hkv, "f16")
    assert_close(out_f64(out[:1]), want, "f16")
