"""The five synthetic decode workloads at full size, one decode step each through
the C ABI (the launch configuration bench.py times), against the oracle:

  * block-manager output (slots, copy-on-write pairs, tables, lengths): bit-exact;
  * the cache after the step's copies and writes: bit-exact on every block the step
    touched and on a random sample of the rest (the whole pool for the small
    workloads);
  * attention: every (sequence, head) for the tiny and 7B-shaped workloads,
    a sample of sequences / kv-head groups elsewhere; all other outputs must be
    finite and bounded by the largest |V| in the pool.
"""
import math

import numpy as np
import pytest
import torch

from gpu_util import TORCH_DT, assert_close, out_f64, to_dev, to_host
from oracle.step import build_context, decode_step
from workloads import CONFIGS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    assert torch.cuda.is_available()
    m.pa_device_error_read()
    return m


def _sample(cfg, name):
    S, Hq, Hkv = cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads
    G = Hq // Hkv
    if name in ("tiny_fp32", "7b_bf16"):
        return None, None
    g = np.random.default_rng(123)
    if name == "gqa_long_bf16":
        kv = [0, Hkv - 1]
        return list(range(S)), [h for k in kv for h in range(k * G, (k + 1) * G)]
    seqs = sorted(set(g.choice(S, 24, replace=False).tolist()))
    return seqs, None


# seed 0 is the parity case of every workload; seeds 1-3 are spot checks of other draws
@pytest.mark.parametrize("name,fork_step,seed", [
    ("tiny_fp32", False, 0), ("7b_bf16", False, 0), ("13b_fp16", False, 0),
    ("gqa_long_bf16", False, 0), ("prefix_cow_bf16", False, 0), ("prefix_cow_bf16", True, 0),
    ("tiny_fp32", False, 1), ("tiny_fp32", False, 2), ("tiny_fp32", False, 3),
    ("7b_bf16", False, 1), ("13b_fp16", False, 2), ("prefix_cow_bf16", False, 3)])
def test_workload_step(pa, name, fork_step, seed):
    from paged_kv_cache_342_b200.runtime import PagedDecoder
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, seed, fork_step=fork_step)
    dt = cfg.dtype
    S = cfg.num_seqs
    lens_after = inp.context_lens + 1
    max_blocks = int(math.ceil(int(lens_after.max()) / cfg.block_size)) + 1

    # ---- product path -------------------------------------------------------
    kd, vd = to_dev(inp.k_pool, dt), to_dev(inp.v_pool, dt)
    dec = PagedDecoder(kd, vd, cfg.num_heads, cfg.scale, max_blocks, inp.free_order,
                       cfg.partition_size)
    if inp.prefix is None:
        for s in range(S):
            dec.admit(s, int(inp.context_lens[s]))
        build_pairs = np.zeros((0, 2), np.int32)
    else:
        p = inp.prefix
        build_pairs = dec.admit_shared_prefix(p.groups, p.samples, p.prefix_len, p.private_lens)
        dec.apply_copies(build_pairs)
    dec.bind(range(S))
    out = torch.full((S, cfg.num_heads, cfg.head_dim), float("nan"), dtype=TORCH_DT[dt],
                     device="cuda")
    meta = dec.step(to_dev(inp.q, dt), to_dev(inp.new_k, dt), to_dev(inp.new_v, dt), out)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    slots_c = meta.slots.copy()
    pairs_c = meta.pairs.copy()
    tables_c, lens_c = meta.tables.copy(), meta.lens.copy()

    # ---- oracle (in place on the host pool: the device has its own copy) -----
    seqs, heads = _sample(cfg, name)
    bm, k, v, o_build = build_context(inp, copy_pool=False)
    assert [tuple(x) for x in build_pairs.tolist()] == o_build
    res = decode_step(bm, k, v, inp, max_blocks, seqs=seqs, heads=heads)

    assert np.array_equal(slots_c, res["slots"])
    assert np.array_equal(pairs_c.reshape(-1, 2), res["pairs"])
    assert np.array_equal(tables_c, res["tables"]) and np.array_equal(lens_c, res["seq_lens"])
    if fork_step:
        assert len(pairs_c) == 224
    # kernels of the step: copies (if any), the cache write, the partition grid, then
    # the merge - or, for a grouped batch, the clear of its arrival counters before it
    several = -(-meta.max_len // meta.partition_size) > 1
    assert meta.kernels == (1 if meta.num_cow else 0) + 2 + (1 if several else 0)

    # ---- caches ---------------------------------------------------------------
    touched = set((res["slots"] // cfg.block_size).tolist()) | set(res["pairs"][:, 1].tolist())
    touched |= set(np.asarray(o_build, np.int64).reshape(-1, 2)[:, 1].tolist())
    rest = np.random.default_rng(7).choice(cfg.num_blocks, min(64, cfg.num_blocks), replace=False)
    check = sorted(touched | set(rest.tolist())) if cfg.num_blocks > 4096 else None
    for dev, host in ((kd, k), (vd, v)):
        if check is None:
            assert np.array_equal(to_host(dev, dt), host)
        else:
            idx = torch.tensor(check, device="cuda")
            assert np.array_equal(to_host(dev.index_select(0, idx), dt), host[check])

    # ---- attention --------------------------------------------------------------
    got = out_f64(out)
    want = res["out"]
    rows = ~np.isnan(want[:, :, 0])
    assert rows.any()
    assert_close(got[rows], want[rows], dt, name)
    assert np.isfinite(got).all()
    vmax = float(np.abs(out_f64(vd.view(-1)[: 1 << 24])).max()) * 4.0 + 1.0
    assert np.abs(got).max() <= vmax
