"""Failure detection on the GPU without a fault: a bounded wait that nothing completes
gives up, reports PA_DEVERR_TIMEOUT through the device error word, and the context
stays usable for the next decode."""
import math
import time

import numpy as np
import pytest
import torch

import oracle.attention as oatt
from gpu_util import assert_close, blocks_for, out_f64, tables_from_order, to_dev
from workloads import normal_fill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    assert torch.cuda.is_available()
    m.pa_device_error_read()
    return m


def test_bounded_wait_gives_up_and_reports(pa):
    t0 = time.perf_counter()
    pa.pa_selftest_bounded_wait()
    bits = pa.pa_device_error_read()           # synchronises
    elapsed = time.perf_counter() - t0
    assert bits == pa.DEVERR_TIMEOUT
    assert 0.5 < elapsed < 30.0                  # the bound is about one second
    assert pa.pa_device_error_read() == 0        # read clears the word

    # the context is still usable: a small decode afterwards matches the oracle
    S, Hq, Hkv, D, bs = 2, 4, 4, 128, 16
    lens = np.array([40, 77], np.int64)
    NB = int(sum(blocks_for(int(L), bs) for L in lens)) + 1
    order = np.random.default_rng(1).permutation(NB).astype(np.int32)
    tables = tables_from_order(lens, bs, order, 6)
    k = normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 31, 1)
    v = normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 31, 2)
    q = normal_fill((S, Hq, D), "bf16", 1.0, 31, 3)
    out = torch.empty((S, Hq, D), dtype=torch.bfloat16, device="cuda")
    pa.pa_decode_attention(out, to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"),
                           torch.from_numpy(tables).cuda(),
                           torch.from_numpy(lens.astype(np.int32)).cuda(), 1 / math.sqrt(D),
                           bs, Hkv, int(lens.max()), 512, None)
    assert pa.pa_device_error_read() == 0
    want = oatt.paged_decode_attention(q, k, v, tables, lens, 1 / math.sqrt(D), bs, Hkv, "bf16")
    assert_close(out_f64(out), want, "bf16", "after the timeout")
