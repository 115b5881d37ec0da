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
