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


@pytest.mark.parametrize("dtype,Hq,Hkv,bs", [("bf16", 16, 2, 16), ("f16", 4, 4, 16),
                                          ("f32", 8, 2, 8)])
def test_library_partition_choice_matches_the_oracle(pa, dtype, Hq, Hkv, bs):
    lens = (3000, 1, 1500, 2049, 700)
    # the device's own choice, and the choices for smaller machines (longer partitions)
    sizes = {pa.pa_decode_partition_size(PA_CODE[dtype], len(lens), Hq, Hkv, 128, bs,
                                         max(lens), n) for n in (0, 1, 2)}
    assert 0 not in sizes
    for ps in sorted(sizes):
        got, want = run_case(pa, dtype, Hq, Hkv, 128, bs, ps, lens, seed=8)
        assert_close(got, want, dtype, f"partition {ps}")


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


# ---------------------------------------------------------------------------
# prefix groups: shared partitions computed once per group
# ---------------------------------------------------------------------------

def run_grouped_case(pa, dtype, Hq, Hkv, D, bs, ps, prefix_len, tails, group_sizes, mm,
                     seed=3, ws_fill=None, calls=1):
    """Groups of sequences forked from one prefix through the block manager, with
    private tails written into their own blocks; compare the grouped call with the
    oracle (and with the plain call).  ws_fill: a byte value, or "random", written over
    the workspace first; calls: grouped calls made back to back on that workspace (the
    result is the last one's, and every call must give the same bits)."""
    from oracle.allocator import BlockManager
    sizes = list(group_sizes)
    S = sum(sizes)
    lens = np.array([prefix_len + t for t in tails], np.int64)
    assert len(lens) == S
    NB = len(sizes) * (-(-prefix_len // bs)) + int(sum(-(-t // bs) + 1 for t in tails)) + 4
    bm = BlockManager(NB, bs, np.random.default_rng([seed, 9]).permutation(NB))
    sid = 0
    for n in sizes:
        bm.add(sid, prefix_len)
        for i in range(1, n):
            bm.fork(sid, sid + i)
        sid += n
    for s in range(S):
        for _ in range(int(tails[s])):
            bm.append_slot(s)
    width = max(len(t) for t in bm.tables.values()) + 1
    rows, sl = bm.block_tables(range(S), width)
    tables, sl = np.array(rows, np.int32), np.array(sl, np.int32)
    k = normal_fill((NB, Hkv, bs, D), dtype, 1.0, seed, 1)
    v = normal_fill((NB, Hkv, bs, D), dtype, 1.0, seed, 2)
    q = normal_fill((S, Hq, D), dtype, 1.0, seed, 3)
    pp, chunks = bm.prefix_groups(range(S), ps, mm)
    cm = np.full((max(len(chunks), 1), mm), -1, np.int32)
    cp = np.zeros(max(len(chunks), 1), np.int32)
    for i, (members, parts) in enumerate(chunks):
        cm[i, :len(members)] = members
        cp[i] = parts
    max_len = int(sl.max())
    scale = 1 / math.sqrt(D)
    kd, vd, qd = to_dev(k, dtype), to_dev(v, dtype), to_dev(q, dtype)
    td, ld = torch.from_numpy(tables).cuda(), torch.from_numpy(sl).cuda()
    wsb = pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    if ws_fill == "random":
        ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8,
                               generator=torch.Generator().manual_seed(seed)))
    elif ws_fill is not None:
        ws.fill_(ws_fill)
    own = [min(p_, (int(L) - 1) // ps) if L > 0 else 0 for p_, L in zip(pp, sl)]
    first = min(own) if chunks else 0
    results = []
    for _ in range(calls):
        out = torch.full((S, Hq, D), float("nan"), dtype=TORCH_DT[dtype], device="cuda")
        pa.pa_decode_attention_grouped(out, qd, kd, vd, td, ld, scale, bs, Hkv, max_len,
                                       torch.from_numpy(np.array(pp, np.int32)).cuda(),
                                       torch.from_numpy(cm).cuda(), torch.from_numpy(cp).cuda(),
                                       len(chunks), max([c[1] for c in chunks], default=0), ps,
                                       ws if wsb else None, first_part=first)
        results.append(out)
    for r in results[1:]:
        assert torch.equal(r.view(torch.int16), results[0].view(torch.int16))
    plain = torch.full_like(out, float("nan"))
    pa.pa_decode_attention(plain, qd, kd, vd, td, ld, scale, bs, Hkv, max_len, ps,
                           ws if wsb else None)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    want = oatt.paged_decode_attention(q, k, v, tables, sl, scale, bs, Hkv, dtype)
    return out_f64(out), out_f64(plain), want, chunks


GROUP_CASES = [
    # dtype, Hq, Hkv, D, bs, partition, prefix, tails, group sizes, members per chunk
    ("bf16", 4, 4, 128, 16, 64, 300, [1, 5, 40, 0, 17, 3, 90, 1], [8], 8),
    ("f16", 2, 2, 64, 16, 32, 130, [2, 0, 1, 33, 70], [3, 2], 8),       # prefix not whole
    ("bf16", 4, 2, 128, 32, 64, 256, [1, 9, 64, 2, 3, 1], [6], 4),     # group 2 heads/kv
    ("bf16", 16, 2, 128, 16, 64, 200, [1, 20, 3], [3], 1),             # GQA 8 + 1 member
    ("f16", 4, 4, 256, 16, 64, 129, [1] * 11 + [40], [12], 8),         # 2 chunks
    ("bf16", 2, 2, 128, 16, 64, 64, [0, 0, 5], [3], 8),                 # tails of length 0
    # a group beside two sequences of no group (their own prefixes): in the one grid the
    # group's shared partitions, then every sequence's own partitions from partition 0
    ("bf16", 8, 8, 128, 16, 64, 200, [3, 50, 0, 7, 130, 9], [4, 1, 1], 8),
    # long shared partitions and one-token tails: the group CTAs finish last, so they
    # combine their members' rows (8 members of one head; 4 members of 4 heads)
    ("bf16", 8, 8, 128, 16, 512, 4100, [1] * 16, [16], 8),
    ("bf16", 8, 2, 128, 16, 256, 2100, [1, 0, 2, 1], [4], 4),
]


@pytest.mark.parametrize("case", GROUP_CASES, ids=lambda c: f"{c[0]}-h{c[1]}/{c[2]}-d{c[3]}-b{c[4]}-p{c[5]}-g{c[8]}")
def test_grouped_matches_oracle_and_plain(pa, case):
    dtype, Hq, Hkv, D, bs, ps, prefix, tails, sizes, mm = case
    got, plain, want, chunks = run_grouped_case(pa, dtype, Hq, Hkv, D, bs, ps, prefix, tails,
                                                sizes, mm)
    assert_close(got, want, dtype, "grouped")
    assert_close(plain, want, dtype, "plain")
    assert np.abs(got - plain).max() <= 2e-2


@pytest.mark.parametrize("fill", [0xFF, 0x00, "random"])
def test_grouped_result_does_not_depend_on_workspace_contents(pa, fill):
    """The grouped grid combines each row in the CTA that writes its last partial, on
    arrival counters in the workspace that the call clears first: whatever the
    workspace held, and on back-to-back calls, the bits are the same."""
    case = GROUP_CASES[0]
    got, _, want, _ = run_grouped_case(pa, *case, ws_fill=fill, calls=2)
    ref, *_ = run_grouped_case(pa, *case)
    assert np.array_equal(got, ref)
    assert_close(got, want, case[0], "grouped")


def test_grouped_call_uses_groups(pa):
    """The shared-prefix case really forms chunks (so the group kernel ran)."""
    *_, chunks = run_grouped_case(pa, *GROUP_CASES[0])
    # 300-token prefix at block 16 = 18 full shared blocks = 288 tokens = 4 partitions of 64
    assert len(chunks) == 1 and chunks[0] == (list(range(8)), 4)


def test_grouped_first_part_too_high_is_reported(pa):
    """A first_part above a sequence's own first partition leaves a hole: reported."""
    dtype, Hq, Hkv, D, bs, ps = "bf16", 4, 4, 128, 16, 64
    from oracle.allocator import BlockManager
    bm = BlockManager(64, bs)
    bm.add(0, 300)
    bm.fork(0, 1)
    bm.add(2, 100)                     # no group: computes from partition 0
    rows, sl = bm.block_tables([0, 1, 2], 24)
    pp, chunks = bm.prefix_groups([0, 1, 2], ps, 8)
    k = to_dev(normal_fill((64, Hkv, bs, D), dtype, 1.0, 2, 1), dtype)
    q = to_dev(normal_fill((3, Hq, D), dtype, 1.0, 2, 2), dtype)
    cm = np.full((1, 8), -1, np.int32)
    cm[0, :2] = chunks[0][0]
    out = torch.empty((3, Hq, D), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(pa.pa_decode_workspace_bytes(3, Hq, D, 300, ps), dtype=torch.uint8,
                     device="cuda")
    pa.pa_decode_attention_grouped(out, q, k, k, torch.tensor(rows, dtype=torch.int32).cuda(),
                                   torch.tensor(sl, dtype=torch.int32).cuda(), 0.1, bs, Hkv, 300,
                                   torch.tensor(pp, dtype=torch.int32).cuda(),
                                   torch.from_numpy(cm).cuda(),
                                   torch.tensor([chunks[0][1]], dtype=torch.int32).cuda(), 1,
                                   chunks[0][1], ps, ws, first_part=2)
    assert pa.pa_device_error_read() == pa.DEVERR_GROUP


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (16, 2)])
def test_decode_right_after_a_kernel_that_writes_its_inputs(pa, Hq, Hkv):
    # the decode kernels are launched to overlap the end of the kernel before them on
    # the stream; here that kernel writes q and the cache, so an early read would show
    S, D, bs = 3, 128, 16
    lens = np.array([700, 33, 1500], np.int32)
    NB = int(sum(blocks_for(int(L), bs) for L in lens)) + 2
    order = np.random.default_rng(4).permutation(NB).astype(np.int32)
    tables = tables_from_order(lens, bs, order, int(max(blocks_for(int(L), bs) for L in lens)))
    k = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 21, 1), "bf16")
    v = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 21, 2), "bf16")
    qs = [to_dev(normal_fill((S, Hq, D), "bf16", 1.0, 21, 3 + i), "bf16") for i in range(6)]
    t_d, l_d = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    wsb = pa.pa_decode_workspace_bytes(S, Hq, D, int(lens.max()), 256)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")

    def decode(q, out):
        pa.pa_decode_attention(out, q, k, v, t_d, l_d, 1 / math.sqrt(D), bs, Hkv,
                               int(lens.max()), 256, ws)

    refs = []
    for q in qs:
        out = torch.empty_like(q)
        decode(q, out)
        refs.append(out)
    torch.cuda.synchronize()
    q_live = torch.zeros_like(qs[0])
    outs = []
    for i, q in enumerate(qs):
        torch.mul(q, 1.0, out=q_live)          # a kernel writing q just before the decode
        k.mul_(1.0)                             # and one rewriting the cache in place
        out = torch.empty_like(q)
        decode(q_live, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert pa.pa_device_error_read() == 0
    for i in range(len(qs)):
        assert torch.equal(outs[i], refs[i]), f"iteration {i}"


@pytest.mark.parametrize("Hq,Hkv,ps", [(4, 4, 512), (16, 2, 64), (8, 2, 32)])
def test_sequence_order_does_not_change_the_result(pa, Hq, Hkv, ps):
    # pa_decode with seq_order: the grid takes the sequences in another order; every
    # output is bit-identical to the plain call's
    S, D, bs = 7, 128, 16
    lens = np.array([300, 5, 1000, 64, 0, 129, 700], np.int64)
    NB = int(sum(blocks_for(int(L), bs) for L in lens)) + 3
    order = np.random.default_rng(6).permutation(NB).astype(np.int32)
    width = int(max(blocks_for(int(L), bs) for L in lens)) + 1
    tables = tables_from_order(lens, bs, order, width)
    k = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 41, 1), "bf16")
    v = to_dev(normal_fill((NB, Hkv, bs, D), "bf16", 1.0, 41, 2), "bf16")
    q = to_dev(normal_fill((S, Hq, D), "bf16", 1.0, 41, 3), "bf16")
    t_d = torch.from_numpy(tables).cuda()
    l_d = torch.from_numpy(lens.astype(np.int32)).cuda()
    max_len = int(lens.max())
    wsb = pa.pa_decode_workspace_bytes(S, Hq, D, max_len, ps)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(q)
    pa.pa_decode_attention(ref, q, k, v, t_d, l_d, 1 / math.sqrt(D), bs, Hkv, max_len, ps,
                           ws if wsb else None)
    for perm in (np.argsort(-lens, kind="stable"), np.random.default_rng(2).permutation(S)):
        out = torch.full_like(q, float("nan"))
        pa.pa_decode(out, q, k, v, t_d, l_d, 1 / math.sqrt(D), bs, Hkv, max_len, ps,
                     ws if wsb else None, seq_order=torch.from_numpy(perm.astype(np.int32)).cuda())
        torch.cuda.synchronize()
        assert pa.pa_device_error_read() == 0
        assert torch.equal(out, ref)
    # an entry out of range skips its row and is reported; the other rows are unchanged
    bad = np.arange(S, dtype=np.int32)
    bad[3] = S + 5
    out = torch.full_like(q, float("nan"))
    pa.pa_decode(out, q, k, v, t_d, l_d, 1 / math.sqrt(D), bs, Hkv, max_len, ps,
                 ws if wsb else None, seq_order=torch.from_numpy(bad).cuda())
    assert pa.pa_device_error_read() & pa.DEVERR_ORDER
    rows = [s for s in range(S) if s != 3]
    assert torch.equal(out[rows], ref[rows])
