"""Logit trajectories that move the online softmax's running max in every way the
kernels distinguish: slow rises (block maxima a few units above the last max, which a
lazy running max keeps without rescaling), steady rises that cross the lazy bound every
other block, a sudden jump of 40 (base 2), a fall, and a flat stretch.  Every query
head of a kv head shares one direction, so the trajectory is the same for all of them.
Every kernel (CUDA cores for MHA, tensor cores for groups of 8 and 16, on fp8 caches
the tcgen05 kernel with its q split into two or three e4m3 terms and its P into two),
bf16, f16 and fp8 caches, several partition sizes; compared with the float64 oracle on
the stored values."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as oatt
from oracle import fp8
from oracle.numerics import to_f64
from gpu_util import TORCH_DT, assert_close, out_f64, tables_from_order, to_dev
from workloads import normal_fill, round_to_storage

pytestmark = pytest.mark.gpu

LOG2E = 1.0 / math.log(2.0)


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    assert torch.cuda.is_available()
    m.pa_device_error_read()
    return m


def trajectory(L, seed):
    """Target base-2 logits for tokens 0..L-1."""
    g = np.random.default_rng([seed, 77])
    t = np.arange(L, dtype=np.float64)
    lam = np.where(t < 96, 0.45 * t, 0.0)                                # crosses 8 every ~18 tokens
    lam = np.where((t >= 96) & (t < 160), 43.0 + 0.02 * (t - 96), lam)   # jump of ~40
    lam = np.where((t >= 160) & (t < 260), 44.0 - 0.3 * (t - 160), lam)  # fall
    lam = np.where(t >= 260, 10.0 + 7.5 * ((t - 260) // 16), lam)        # +7.5 per block
    return lam + 0.05 * g.standard_normal(L)


def build(lens, Hq, Hkv, D, bs, seed):
    """K rows along each kv head's query direction so that q.k * scale follows the
    trajectory; V is N(0,1).  Returns float32 K, V, q and the block tables."""
    lens = np.asarray(lens, np.int64)
    S = lens.size
    G = Hq // Hkv
    NB = int(sum(-(-int(L) // bs) for L in lens)) + 2
    scale = 1.0 / math.sqrt(D)
    g = np.random.default_rng([seed, 78])
    qdir = g.standard_normal((S, Hkv, D))
    q = np.repeat(qdir, G, axis=1).astype(np.float32)                  # [S, Hq, D]
    order = g.permutation(NB).astype(np.int32)
    tables = tables_from_order(lens, bs, order, int(-(-lens.max() // bs)) + 1)
    k = (0.3 * g.standard_normal((NB, Hkv, bs, D))).astype(np.float32)
    for s, L in enumerate(lens):
        lam = trajectory(int(L), seed + s)
        for h in range(Hkv):
            u = qdir[s, h]
            coef = lam / (scale * LOG2E * float(u @ u))
            for tpos in range(int(L)):
                blk, off = tables[s, tpos // bs], tpos % bs
                k[blk, h, off] = coef[tpos] * u
    v = normal_fill((NB, Hkv, bs, D), "f32", 1.0, seed, 2)
    return k, v, q, tables, scale


CASES = [
    # Hq, Hkv, D, bs, partition, lens
    (2, 2, 128, 16, 64, (700, 333, 1, 97)),     # CUDA cores, many partitions
    (2, 2, 128, 16, 2048, (700, 333, 1, 97)),   # CUDA cores, one partition
    (16, 2, 128, 16, 64, (700, 333, 1, 97)),    # tensor cores, group 8
    (16, 2, 128, 16, 4096, (700, 333, 1, 97)),
    (16, 2, 128, 32, 128, (700, 161, 40)),      # tensor cores, block 32
    (32, 2, 128, 16, 256, (700, 333, 1, 97)),   # tensor cores, group 16
]


@pytest.mark.parametrize("qdt", ["bf16", "f16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"h{c[0]}/{c[1]}-b{c[3]}-p{c[4]}")
def test_logit_trajectory_16bit_cache(pa, case, qdt):
    Hq, Hkv, D, bs, ps, lens = case
    k, v, q, tables, scale = build(lens, Hq, Hkv, D, bs, 5)
    ks, vs, qs = (round_to_storage(x, qdt) for x in (k, v, q))
    lens = np.asarray(lens, np.int64)
    S, max_len = lens.size, int(lens.max())
    out = torch.full((S, Hq, D), float("nan"), dtype=TORCH_DT[qdt], device="cuda")
    wsb = pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda") if wsb else None
    pa.pa_decode_attention(out, to_dev(qs, qdt), to_dev(ks, qdt), to_dev(vs, qdt),
                           torch.from_numpy(tables).cuda(),
                           torch.from_numpy(lens.astype(np.int32)).cuda(), scale, bs, Hkv,
                           max_len, ps, ws)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    want = oatt.paged_decode_attention(qs, ks, vs, tables, lens, scale, bs, Hkv, qdt)
    assert_close(out_f64(out), want, qdt, "logit trajectory")


@pytest.mark.parametrize("qdt", ["bf16", "f16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"h{c[0]}/{c[1]}-b{c[3]}-p{c[4]}")
def test_logit_trajectory_fp8_cache(pa, case, qdt):
    Hq, Hkv, D, bs, ps, lens = case
    k, v, q, tables, scale = build(lens, Hq, Hkv, D, bs, 6)
    k_scale = float(np.abs(k).max()) / 448.0
    v_scale = 4.0 / 448.0
    kc, vc = fp8.quantize(k, k_scale), fp8.quantize(v, v_scale)
    qs = round_to_storage(q, qdt)
    lens = np.asarray(lens, np.int64)
    S, max_len = lens.size, int(lens.max())
    out = torch.full((S, Hq, D), float("nan"), dtype=TORCH_DT[qdt], device="cuda")
    wsb = pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    pa.pa_decode_attention_fp8(out, to_dev(qs, qdt), torch.from_numpy(kc).cuda(),
                               torch.from_numpy(vc).cuda(), torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens.astype(np.int32)).cuda(), scale, bs, Hkv,
                               max_len, k_scale, v_scale, ps, ws if wsb else None)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    want = oatt.paged_decode_attention(to_f64(qs, qdt), fp8.dequantize(kc, k_scale),
                                       fp8.dequantize(vc, v_scale), tables, lens, scale, bs,
                                       Hkv, "f64")
    assert_close(out_f64(out), want, qdt, "logit trajectory, fp8 cache")
