"""The fp8 (e4m3) cache: the quantizing write is bit-exact against the oracle's
codec, and decode over the fp8 cache matches the float64 oracle on the dequantized
values (per-tensor scales; stored = e4m3(x * (1/scale)), value = code * scale)."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as oatt
from oracle import fp8
from gpu_util import TORCH_DT, assert_close, out_f64, tables_from_order, to_dev
from oracle.numerics import to_f64
from workloads import normal_fill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    assert torch.cuda.is_available()
    m.pa_device_error_read()
    return m


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("D,bs,Hkv", [(128, 16, 4), (64, 8, 2), (256, 32, 2)])
def test_fp8_write_is_bit_exact(pa, dtype, D, bs, Hkv):
    NB, T = 24, 29
    key = normal_fill((T, Hkv, D), dtype, 3.0, 4, 1)
    val = normal_fill((T, Hkv, D), dtype, 40.0, 4, 2)      # some values saturate
    ks, vs = 0.0271, 0.05
    slots = np.random.default_rng(4).choice(NB * bs, T, replace=False).astype(np.int64)
    slots[3] = -1
    kc = torch.full((NB, Hkv, bs, D), 0x5A, dtype=torch.uint8, device="cuda")
    vc = torch.full_like(kc, 0x21)
    pa.pa_reshape_and_cache_fp8(to_dev(key, dtype), to_dev(val, dtype), kc, vc,
                                torch.from_numpy(slots).cuda(), ks, vs)
    want_k = np.full((NB, Hkv, bs, D), 0x5A, np.uint8)
    want_v = np.full_like(want_k, 0x21)
    for t, slot in enumerate(slots):
        if slot < 0:
            continue
        b, o = divmod(int(slot), bs)
        want_k[b, :, o, :] = fp8.quantize(to_f64(key[t], dtype).astype(np.float32), ks)
        want_v[b, :, o, :] = fp8.quantize(to_f64(val[t], dtype).astype(np.float32), vs)
    assert np.array_equal(kc.cpu().numpy(), want_k)
    assert np.array_equal(vc.cpu().numpy(), want_v)
    assert pa.pa_device_error_read() == 0


FP8_CASES = [
    # q dtype, Hq, Hkv, D, bs, partition, lens
    ("bf16", 4, 4, 128, 16, 64, (1, 15, 16, 17, 200, 333, 0)),
    ("f16", 8, 2, 128, 8, 32, (5, 64, 65, 400)),          # group 4
    ("bf16", 16, 2, 128, 16, 512, (1, 700, 33)),           # group 8: tensor cores
    ("f16", 16, 2, 128, 32, 128, (1, 300, 64, 0)),         # tensor cores, block 32
    ("bf16", 32, 2, 256, 16, 64, (5, 200, 129)),           # group 16, head_dim 256
    ("f16", 8, 2, 128, 16, 64, (9, 90)),                   # group 4: CUDA cores
    ("f16", 2, 2, 256, 32, 64, (3, 100, 250)),
    ("bf16", 4, 4, 128, 4, 16, (7, 18, 10)),
    # the tcgen05 kernel (head_dim 128, groups of 8 or 16): 128-token tiles
    ("bf16", 32, 2, 128, 16, 256, (1, 127, 128, 129, 1000)),   # group 16
    ("f16", 32, 2, 128, 32, 64, (5, 333, 64, 65)),            # group 16, partitions < a tile
    ("f16", 16, 2, 128, 16, 384, (383, 384, 385, 1153)),      # partitions of three tiles
    ("bf16", 32, 4, 128, 16, 512, (1100, 700)),               # 4 kv heads x group 8
    ("bf16", 16, 2, 128, 16, 4096, (4096, 17)),               # one partition of 32 tiles
    ("bf16", 16, 2, 128, 32, 2048, (2048, 1)),
]


@pytest.mark.parametrize("case", FP8_CASES, ids=lambda c: f"{c[0]}-h{c[1]}/{c[2]}-d{c[3]}-b{c[4]}")
def test_fp8_decode_matches_oracle(pa, case):
    dtype, Hq, Hkv, D, bs, ps, lens = case
    lens = np.asarray(lens, np.int64)
    S = lens.size
    NB = int(sum(-(-int(L) // bs) for L in lens)) + 3
    g = np.random.default_rng(8)
    # N(0,1) K/V stored with scale 8/448 (the oracle's codec makes the codes)
    ks = vs = 8.0 / 448.0
    kcodes = fp8.quantize(normal_fill((NB, Hkv, bs, D), "f32", 1.0, 8, 1), ks)
    vcodes = fp8.quantize(normal_fill((NB, Hkv, bs, D), "f32", 1.0, 8, 2), vs)
    q = normal_fill((S, Hq, D), dtype, 1.0, 8, 3)
    order = g.permutation(NB).astype(np.int32)
    tables = tables_from_order(lens, bs, order, int(-(-lens.max() // bs)) + 1)
    max_len = int(lens.max())
    out = torch.full((S, Hq, D), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
    wsb = pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    scale = 1 / math.sqrt(D)
    pa.pa_decode_attention_fp8(out, to_dev(q, dtype), torch.from_numpy(kcodes).cuda(),
                               torch.from_numpy(vcodes).cuda(), torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens.astype(np.int32)).cuda(), scale, bs, Hkv,
                               max_len, ks, vs, ps, ws if wsb else None)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    want = oatt.paged_decode_attention(to_f64(q, dtype), fp8.dequantize(kcodes, ks),
                                       fp8.dequantize(vcodes, vs), tables, lens, scale, bs, Hkv,
                                       "f64")
    assert_close(out_f64(out), want, dtype, "fp8 cache")


def test_fp8_decode_all_codes(pa):
    """Every finite e4m3 code appears in the cache (magnitudes up to 448 * scale); the
    output is compared at the tolerance of its own magnitude (bf16 rounding of |out|)."""
    S, Hq, Hkv, D, bs = 3, 4, 4, 128, 16
    lens = np.array([256, 100, 37])
    NB = 24
    g = np.random.default_rng(9)
    codes = [g.integers(0, 256, (NB, Hkv, bs, D)).astype(np.uint8) for _ in range(2)]
    for c in codes:
        c[(c & 0x7F) == 0x7F] = 0x3F                    # no NaN codes
    ks, vs = 0.002, 0.004
    q = normal_fill((S, Hq, D), "bf16", 1.0, 9, 3)
    tables = tables_from_order(lens, bs, g.permutation(NB).astype(np.int32), 17)
    out = torch.empty((S, Hq, D), dtype=torch.bfloat16, device="cuda")
    pa.pa_decode_attention_fp8(out, to_dev(q, "bf16"), torch.from_numpy(codes[0]).cuda(),
                               torch.from_numpy(codes[1]).cuda(), torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens.astype(np.int32)).cuda(), 1 / math.sqrt(D),
                               bs, Hkv, 256, ks, vs, 64,
                               torch.empty(pa.pa_decode_workspace_bytes(S, Hq, D, 256, 64),
                                           dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    want = oatt.paged_decode_attention(to_f64(q, "bf16"), fp8.dequantize(codes[0], ks),
                                       fp8.dequantize(codes[1], vs), tables, lens,
                                       1 / math.sqrt(D), bs, Hkv, "f64")
    got = out_f64(out)
    assert np.isfinite(got).all()
    assert np.all(np.abs(got - want) <= 2e-2 + 2.0 ** -8 * np.abs(want))


def test_fp8_decode_step_through_the_runtime(pa):
    """A whole decode step on an fp8 cache: write the new token (quantized), attend."""
    from paged_kv_cache_342_b200.runtime import PagedDecoder
    S, Hq, Hkv, D, bs, NB = 6, 8, 8, 128, 16, 96
    g = np.random.default_rng(12)
    lens = g.integers(20, 200, S)
    ks = vs = 8.0 / 448
    pool_k = fp8.quantize(normal_fill((NB, Hkv, bs, D), "f32", 1.0, 12, 1), ks)
    pool_v = fp8.quantize(normal_fill((NB, Hkv, bs, D), "f32", 1.0, 12, 2), vs)
    kd, vd = torch.from_numpy(pool_k).cuda(), torch.from_numpy(pool_v).cuda()
    dec = PagedDecoder(kd, vd, Hq, 1 / math.sqrt(D), 16, g.permutation(NB), 64,
                       kv_scales=(ks, vs), query_dtype=torch.bfloat16)
    for s in range(S):
        dec.admit(s, int(lens[s]))
    dec.bind(range(S))
    q = normal_fill((S, Hq, D), "bf16", 1.0, 12, 3)
    nk = normal_fill((S, Hkv, D), "bf16", 1.0, 12, 4)
    nv = normal_fill((S, Hkv, D), "bf16", 1.0, 12, 5)
    out = torch.empty((S, Hq, D), dtype=torch.bfloat16, device="cuda")
    meta = dec.step(to_dev(q, "bf16"), to_dev(nk, "bf16"), to_dev(nv, "bf16"), out)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    tables, sl = meta.tables.copy(), meta.lens.copy()
    slots = meta.slots.copy()
    # oracle: quantize the new token into its slot, attend over dequantized values
    for s, slot in enumerate(slots):
        b, o = divmod(int(slot), bs)
        pool_k[b, :, o, :] = fp8.quantize(to_f64(nk[s], "bf16").astype(np.float32), ks)
        pool_v[b, :, o, :] = fp8.quantize(to_f64(nv[s], "bf16").astype(np.float32), vs)
    assert np.array_equal(kd.cpu().numpy(), pool_k) and np.array_equal(vd.cpu().numpy(), pool_v)
    want = oatt.paged_decode_attention(to_f64(q, "bf16"), fp8.dequantize(pool_k, ks),
                                       fp8.dequantize(pool_v, vs), tables, sl, 1 / math.sqrt(D),
                                       bs, Hkv, "f64")
    assert_close(out_f64(out), want, "bf16", "fp8 step")


@pytest.mark.parametrize("Hq,Hkv,bs,ps,qdt", [(16, 2, 16, 512, "bf16"), (32, 2, 32, 64, "f16"),
                                             (16, 2, 32, 256, "f16")])
def test_fp8_tensor_cores_never_read_unused_slots(pa, Hq, Hkv, bs, ps, qdt):
    """Every slot no sequence owns - the tail of each last block and the blocks in no
    table - holds the NaN code 0x7F: the tiles' rows past the end must not reach O."""
    lens = np.array([1, 130, 700, 129], np.int64)
    S, D = lens.size, 128
    NB = int(sum(-(-int(L) // bs) for L in lens)) + 4
    ks = vs = 8.0 / 448.0
    kc = fp8.quantize(normal_fill((NB, Hkv, bs, D), "f32", 1.0, 13, 1), ks)
    vc = fp8.quantize(normal_fill((NB, Hkv, bs, D), "f32", 1.0, 13, 2), vs)
    order = np.random.default_rng(13).permutation(NB).astype(np.int32)
    tables = tables_from_order(lens, bs, order, int(-(-lens.max() // bs)) + 1)
    used = np.zeros((NB, bs), bool)
    for srow, L in zip(tables, lens):
        for t in range(int(L)):
            used[srow[t // bs], t % bs] = True
    for c in (kc, vc):
        c.transpose(0, 2, 1, 3)[~used] = 0x7F
    q = normal_fill((S, Hq, D), qdt, 1.0, 13, 3)
    out = torch.full((S, Hq, D), float("nan"), dtype=TORCH_DT[qdt], device="cuda")
    wsb = pa.pa_decode_workspace_bytes(S, Hq, D, int(lens.max()), ps)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    pa.pa_decode_attention_fp8(out, to_dev(q, qdt), torch.from_numpy(kc).cuda(),
                               torch.from_numpy(vc).cuda(), torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens.astype(np.int32)).cuda(), 1 / math.sqrt(D),
                               bs, Hkv, int(lens.max()), ks, vs, ps, ws if wsb else None)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    want = oatt.paged_decode_attention(to_f64(q, qdt), fp8.dequantize(kc, ks),
                                       fp8.dequantize(vc, vs), tables, lens, 1 / math.sqrt(D),
                                       bs, Hkv, "f64")
    assert_close(out_f64(out), want, qdt, "fp8 cache, NaN in unused slots")


def test_fp8_tensor_cores_out_of_range_table_entry(pa):
    """A table entry outside the pool is skipped (its rows count as absent) and
    reported; every output stays finite."""
    S, Hq, Hkv, D, bs, NB = 2, 16, 2, 128, 16, 16
    kc = fp8.quantize(normal_fill((NB, Hkv, bs, D), "f32", 1.0, 14, 1), 8.0 / 448)
    q = normal_fill((S, Hq, D), "bf16", 1.0, 14, 2)
    tables = np.array([[3, 5, NB + 7], [1, -4, 2]], np.int32)
    lens = np.array([40, 40], np.int32)
    out = torch.empty((S, Hq, D), dtype=torch.bfloat16, device="cuda")
    kd = torch.from_numpy(kc).cuda()
    pa.pa_decode_attention_fp8(out, to_dev(q, "bf16"), kd, kd, torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens).cuda(), 0.1, bs, Hkv, 40, 8.0 / 448,
                               8.0 / 448, 512, None)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == pa.DEVERR_TABLE
    assert torch.isfinite(out).all()


def _random_codes(shape, seed, stream):
    """e4m3 codes with magnitudes up to 30 (exponent field <= 11) and random signs;
    no NaN codes.  Any such byte is a valid cache entry."""
    g = np.random.default_rng([seed, stream])
    return (g.integers(0, 0x60, shape) | (g.integers(0, 2, shape) << 7)).astype(np.uint8)


def test_fp8_many_rows_on_the_mma_kernel(pa):
    """152 (sequence, kv head) rows of up to 8 partitions of 64 tokens: more rows than
    the tcgen05 kernel takes (it serves few rows, split evenly over the SMs), so the
    mma.sync tensor-core kernel runs it, one CTA per (row, partition), and the dense
    merge combines the partitions."""
    S, Hq, Hkv, D, bs, ps = 19, 64, 8, 128, 16, 64
    g = np.random.default_rng(15)
    lens = np.concatenate([[512, 449, 1, 64, 65], g.integers(380, 513, S - 5)]).astype(np.int64)
    NB = int(sum(-(-int(L) // bs) for L in lens)) + 3
    kc, vc = _random_codes((NB, Hkv, bs, D), 15, 1), _random_codes((NB, Hkv, bs, D), 15, 2)
    ks, vs = 1.0 / 64, 1.0 / 32
    q = normal_fill((S, Hq, D), "bf16", 1.0, 15, 3)
    tables = tables_from_order(lens, bs, g.permutation(NB).astype(np.int32),
                               int(-(-lens.max() // bs)) + 1)
    max_len = int(lens.max())
    out = torch.full((S, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps), dtype=torch.uint8,
                     device="cuda")
    pa.pa_decode_attention_fp8(out, to_dev(q, "bf16"), torch.from_numpy(kc).cuda(),
                               torch.from_numpy(vc).cuda(), torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens.astype(np.int32)).cuda(), 1 / math.sqrt(D),
                               bs, Hkv, max_len, ks, vs, ps, ws)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    want = oatt.paged_decode_attention(to_f64(q, "bf16"), fp8.dequantize(kc, ks),
                                       fp8.dequantize(vc, vs), tables, lens, 1 / math.sqrt(D),
                                       bs, Hkv, "f64")
    assert_close(out_f64(out), want, "bf16", "several partitions per CTA")


@pytest.mark.parametrize("S,Hq,Hkv", [(19, 40, 5), (12, 64, 8)], ids=["95-rows-tcgen05", "96-rows-mma"])
def test_fp8_rows_at_the_kernel_boundary(pa, S, Hq, Hkv):
    """95 (sequence, kv head) rows, the most the tcgen05 kernel takes, and 96, the
    fewest the mma.sync kernel takes: both match the oracle."""
    D, bs, ps = 128, 16, 64
    g = np.random.default_rng(S)
    lens = g.integers(1, 700, S).astype(np.int64)
    lens[0] = 700
    NB = int(sum(-(-int(L) // bs) for L in lens)) + 3
    kc, vc = _random_codes((NB, Hkv, bs, D), S, 1), _random_codes((NB, Hkv, bs, D), S, 2)
    ks, vs = 1.0 / 64, 1.0 / 32
    q = normal_fill((S, Hq, D), "bf16", 1.0, S, 3)
    tables = tables_from_order(lens, bs, g.permutation(NB).astype(np.int32),
                               int(-(-lens.max() // bs)) + 1)
    max_len = int(lens.max())
    out = torch.full((S, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps), dtype=torch.uint8,
                     device="cuda")
    pa.pa_decode_attention_fp8(out, to_dev(q, "bf16"), torch.from_numpy(kc).cuda(),
                               torch.from_numpy(vc).cuda(), torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens.astype(np.int32)).cuda(), 1 / math.sqrt(D),
                               bs, Hkv, max_len, ks, vs, ps, ws)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    want = oatt.paged_decode_attention(to_f64(q, "bf16"), fp8.dequantize(kc, ks),
                                       fp8.dequantize(vc, vs), tables, lens, 1 / math.sqrt(D),
                                       bs, Hkv, "f64")
    assert_close(out_f64(out), want, "bf16", f"{S * Hkv} rows")


def test_fp8_tensor_cores_balanced_split_any_workspace(pa):
    """Few (sequence, kv head) rows: the tensor-core kernel cuts all partitions into
    equal ranges (CTAs combine each range's partitions and leave one partial per
    range; the merge skips the empty slots).  The workspace needs no initialisation:
    calls on a workspace of 0xff bytes, of zeros, and right after another call give
    the same bits, and match the oracle."""
    S, Hq, Hkv, D, bs, ps = 6, 64, 8, 128, 16, 128
    lens = np.array([3000, 2500, 700, 129, 1, 4096], np.int64)
    g = np.random.default_rng(21)
    NB = int(sum(-(-int(L) // bs) for L in lens)) + 3
    kc, vc = _random_codes((NB, Hkv, bs, D), 21, 1), _random_codes((NB, Hkv, bs, D), 21, 2)
    ks, vs = 1.0 / 64, 1.0 / 32
    q = normal_fill((S, Hq, D), "f16", 1.0, 21, 3)
    tables = tables_from_order(lens, bs, g.permutation(NB).astype(np.int32),
                               int(-(-lens.max() // bs)) + 1)
    max_len = int(lens.max())
    args = (to_dev(q, "f16"), torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda(),
            torch.from_numpy(tables).cuda(), torch.from_numpy(lens.astype(np.int32)).cuda(),
            1 / math.sqrt(D), bs, Hkv, max_len, ks, vs, ps)
    nbytes = pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps)
    outs = []
    for fill in (0xFF, 0x00, None):
        ws = (torch.full((nbytes,), fill, dtype=torch.uint8, device="cuda") if fill is not None
              else ws)  # None: the previous call's workspace as it was left
        out = torch.full((S, Hq, D), float("nan"), dtype=torch.float16, device="cuda")
        pa.pa_decode_attention_fp8(out, *args, ws)
        torch.cuda.synchronize()
        assert pa.pa_device_error_read() == 0
        outs.append(out)
    want = oatt.paged_decode_attention(to_f64(q, "f16"), fp8.dequantize(kc, ks),
                                       fp8.dequantize(vc, vs), tables, lens, 1 / math.sqrt(D),
                                       bs, Hkv, "f64")
    assert_close(out_f64(outs[0]), want, "f16", "balanced split")
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_fp8_long_context_gqa_full_size(pa):
    """The long-context GQA workload at full size on an fp8 cache (random codes, the
    stated 512-token partitions, the library's launch), sampled against the oracle:
    two (sequence, kv head) pairs exactly, every output finite."""
    from workloads import CONFIGS, make_inputs
    cfg = CONFIGS["gqa_long_bf16"]
    inp = make_inputs(cfg, 0, pool=False)
    lens = (inp.context_lens + 1).astype(np.int64)
    S, Hq, Hkv, D, bs, NB = (cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_dim,
                             cfg.block_size, cfg.num_blocks)
    width = int(-(-lens.max() // bs)) + 1
    tables = tables_from_order(lens, bs, inp.free_order, width)
    kc, vc = _random_codes((NB, Hkv, bs, D), 16, 1), _random_codes((NB, Hkv, bs, D), 16, 2)
    ks, vs = 1.0 / 64, 1.0 / 32
    max_len, ps = int(lens.max()), cfg.partition_size
    out = torch.full((S, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps), dtype=torch.uint8,
                     device="cuda")
    kd, vd = torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda()
    pa.pa_decode_attention_fp8(out, to_dev(inp.q, "bf16"), kd, vd, torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens.astype(np.int32)).cuda(), cfg.scale, bs, Hkv,
                               max_len, ks, vs, ps, ws)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    got = out_f64(out)
    assert np.isfinite(got).all()
    G = Hq // Hkv
    for s_, g_ in ((int(np.argmin(lens)), 0), (int(np.argmax(lens)), Hkv - 1)):
        nb = int(-(-lens[s_] // bs))
        blocks = tables[s_, :nb]
        sub_k = fp8.dequantize(kc[blocks, g_:g_ + 1], ks)
        sub_v = fp8.dequantize(vc[blocks, g_:g_ + 1], vs)
        want = oatt.paged_decode_attention(
            to_f64(inp.q[s_:s_ + 1, g_ * G:(g_ + 1) * G], "bf16"), sub_k, sub_v,
            np.arange(nb, dtype=np.int32)[None, :], lens[s_:s_ + 1], cfg.scale, bs, 1, "f64")
        assert_close(got[s_:s_ + 1, g_ * G:(g_ + 1) * G], want, "bf16",
                     f"sequence {s_}, kv head {g_}")
