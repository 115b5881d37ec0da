"""The README's Python example runs as written, and its step's output matches the
float64 oracle on the cache it leaves behind."""
import math
import os
import re

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

README = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "README.md")


def test_readme_example_runs_and_matches_the_oracle():
    import oracle.attention as oatt
    from gpu_util import assert_close, out_f64, to_host
    import paged_kv_cache_342_b200 as pa
    text = open(README).read()
    code = re.search(r"```python\n(.*?)```", text, re.S).group(1)
    ns = {}
    exec(compile(code, "README.md", "exec"), ns)
    import torch
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    info, dec = ns["info"], ns["dec"]
    lens = info.lens.astype(np.int64).copy()
    tables = info.tables.copy()
    assert list(lens) == [701, 1201, 36]
    want = oatt.paged_decode_attention(
        to_host(ns["q"], "bf16"), to_host(ns["k_cache"], "bf16"), to_host(ns["v_cache"], "bf16"),
        tables, lens, 1 / math.sqrt(128), dec.block_size, dec.num_kv_heads, "bf16")
    assert_close(out_f64(ns["out"]), want, "bf16", "README example")
