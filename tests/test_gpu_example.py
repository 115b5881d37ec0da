"""The usage example (examples/decode_step.py) runs as written, and its step's output
matches the float64 oracle on the cache it leaves behind."""
import math
import os
import runpy

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

EXAMPLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "examples", "decode_step.py")


def test_example_runs_and_matches_the_oracle():
    import torch

    import oracle.attention as oatt
    import paged_kv_cache_342_b200 as pa
    from gpu_util import assert_close, out_f64, to_host
    ns = runpy.run_path(EXAMPLE, run_name="example")
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    info, dec = ns["info"], ns["dec"]
    lens = info.lens.astype(np.int64).copy()
    tables = info.tables.copy()
    assert list(lens) == [701, 1201, 36]
    want = oatt.paged_decode_attention(
        to_host(ns["q"], "bf16"), to_host(ns["k_cache"], "bf16"), to_host(ns["v_cache"], "bf16"),
        tables, lens, 1 / math.sqrt(128), dec.block_size, dec.num_kv_heads, "bf16")
    assert_close(out_f64(ns["out"]), want, "bf16", "usage example")
