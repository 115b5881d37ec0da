"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each check is a function that returns the largest disagreement it saw, so that
``test_oracle_mutations.py`` can plant plausible mistakes in copies of the oracle
and show that at least one check catches each of them.

Sources of the pinned facts (page title, section):
  [BLOG] "How PagedAttention Powers vLLM's KV Cache" (hassanahmed.net)
  [LAB]  "PagedAttention" explainer (divagr.pages.dev/attention-lab/paged)
"""
import math

import numpy as np
import pytest
import torch

import oracle.attention as oatt
import oracle.cache_ops as ocache
from oracle.allocator import AllocError, BlockManager
from oracle.waste import batch_memory, contiguous_reservation, paged_growth
from workloads import CONFIGS, make_inputs, normal_fill, storage_to_torch

pytestmark = pytest.mark.filterwarnings("ignore")


# ---------------------------------------------------------------------------
# helpers: a paged cache written token by token from contiguous per-sequence K/V
# ---------------------------------------------------------------------------

def _paged_from_contiguous(Ks, Vs, block_size, num_blocks, free_order, Hkv, D, dtype,
                           bm_cls=BlockManager, reshape=None):
    """Admit each sequence empty and append its tokens one by one through the block
    manager, writing each token's K/V into the slot the manager returns."""
    reshape = reshape or ocache.reshape_and_cache
    store = Ks[0].dtype
    k = np.zeros((num_blocks, Hkv, block_size, D), store)
    v = np.zeros_like(k)
    bm = bm_cls(num_blocks, block_size, free_order)
    for s, (K, V) in enumerate(zip(Ks, Vs)):
        bm.add(s, 0)
        for t in range(K.shape[0]):
            slot, src, dst = bm.append_slot(s)
            reshape(K[t:t + 1], V[t:t + 1], k, v, [slot], block_size)
    width = max(len(t) for t in bm.tables.values())
    rows, lens = bm.block_tables(range(len(Ks)), width)
    return k, v, np.array(rows, np.int32), np.array(lens, np.int32)


def _draw_contiguous(lens, Hq, Hkv, D, dtype, seed):
    Ks = [normal_fill((L, Hkv, D), dtype, 1.0, seed, 100 + 2 * i) for i, L in enumerate(lens)]
    Vs = [normal_fill((L, Hkv, D), dtype, 1.0, seed, 101 + 2 * i) for i, L in enumerate(lens)]
    q = normal_fill((len(lens), Hq, D), dtype, 1.0, seed, 99)
    return Ks, Vs, q


def check_against_sdpa(att=oatt, lens=(5, 13, 7, 18, 10), Hq=4, Hkv=4, D=64, bs=4,
                       dtype="f32", seed=0, scale=0.125, reshape=None):
    """Largest |oracle - torch SDPA| over all (seq, head); SDPA runs in float64 on the
    contiguous K/V (query head h reads kv head h // (Hq/Hkv) via repeat_interleave),
    widened from the stored bits by torch's casts."""
    Ks, Vs, q = _draw_contiguous(lens, Hq, Hkv, D, dtype, seed)
    nb = sum(-(-L // bs) for L in lens) + 3
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    k, v, tables, seq_lens = _paged_from_contiguous(Ks, Vs, bs, nb, order, Hkv, D, dtype,
                                                    reshape=reshape)
    out = att.paged_decode_attention(q, k, v, tables, seq_lens, scale, bs, Hkv, dtype)
    worst = 0.0
    G = Hq // Hkv
    # the SDPA side widens the stored bits with torch's own casts, not the oracle's
    wide = lambda a: storage_to_torch(a, dtype).double()
    for s, L in enumerate(lens):
        Kt = wide(Ks[s]).permute(1, 0, 2)                               # [Hkv, L, D]
        Vt = wide(Vs[s]).permute(1, 0, 2)
        Kt, Vt = Kt.repeat_interleave(G, 0), Vt.repeat_interleave(G, 0)
        qt = wide(q[s]).unsqueeze(1)                                    # [Hq, 1, D]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt.unsqueeze(0), Kt.unsqueeze(0), Vt.unsqueeze(0), scale=scale)[0, :, 0, :]
        worst = max(worst, float(np.abs(out[s] - ref.numpy()).max()))
    return worst


def check_against_loops(att=oatt, seed=3):
    """Largest |oracle - textbook formula in pure Python loops| on a tiny case:
    out_d = sum_t exp(s_t) v_td / sum_t exp(s_t), s_t = scale * sum_d q_d k_td."""
    lens, Hq, Hkv, D, bs, scale = (3, 6, 1), 2, 2, 8, 2, 0.3
    Ks, Vs, q = _draw_contiguous(lens, Hq, Hkv, D, "f32", seed)
    nb = 8
    order = np.arange(nb, dtype=np.int32)[::-1].copy()
    k, v, tables, seq_lens = _paged_from_contiguous(Ks, Vs, bs, nb, order, Hkv, D, "f32")
    out = att.paged_decode_attention(q, k, v, tables, seq_lens, scale, bs, Hkv, "f32")
    worst = 0.0
    for s, L in enumerate(lens):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            e = [math.exp(scale * sum(float(q[s, h, d]) * float(Ks[s][t, g, d]) for d in range(D)))
                 for t in range(L)]
            z = sum(e)
            for d in range(D):
                ref = sum(e[t] * float(Vs[s][t, g, d]) for t in range(L)) / z
                worst = max(worst, abs(out[s, h, d] - ref))
    return worst


def check_partition_invariance(att=oatt, seed=1):
    """Largest relative gap between the partitioned + merged form and the plain form."""
    g = np.random.default_rng(seed)
    worst = 0.0
    for L in (1, 17, 300, 1000):
        q = g.standard_normal(64)
        K = g.standard_normal((L, 64)) * 2.0
        V = g.standard_normal((L, 64))
        ref = att.softmax_attention(q, K, V, 0.125)
        for ps in (16, 64, 512, 1 << 20):
            o = att.partitioned_attention(q, K, V, 0.125, ps)
            worst = max(worst, float(np.abs(o - ref).max() / np.abs(ref).max()))
    return worst


def check_block_permutation(att=oatt, seed=2):
    """Max |out - out'| when physical blocks are permuted and the tables rewritten."""
    cfg = CONFIGS["tiny_fp32"]
    inp = make_inputs(cfg, seed)
    bm = BlockManager(cfg.num_blocks, cfg.block_size, inp.free_order)
    lens = inp.context_lens + 1
    for s in range(cfg.num_seqs):
        bm.add(s, int(lens[s]))
    rows, sl = bm.block_tables(range(cfg.num_seqs), 5)
    tables, sl = np.array(rows, np.int32), np.array(sl, np.int32)
    out = att.paged_decode_attention(inp.q, inp.k_pool, inp.v_pool, tables, sl, cfg.scale,
                                     cfg.block_size, cfg.num_kv_heads, cfg.dtype)
    perm = np.random.default_rng(seed + 10).permutation(cfg.num_blocks)
    k2 = np.empty_like(inp.k_pool)
    v2 = np.empty_like(inp.v_pool)
    k2[perm] = inp.k_pool
    v2[perm] = inp.v_pool
    t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1).astype(np.int32)
    out2 = att.paged_decode_attention(inp.q, k2, v2, t2, sl, cfg.scale, cfg.block_size,
                                      cfg.num_kv_heads, cfg.dtype)
    return float(np.abs(out - out2).max())


def check_prefix_sharing(att=oatt, bm_cls=BlockManager, seed=4, prefix=10, bs=4):
    """Max |out_shared - out_duplicated|: two sequences with a common prefix, once
    sharing the prefix blocks through fork (with copy-on-write on divergence), once
    storing the prefix twice."""
    Hkv, D = 2, 16
    X = normal_fill((prefix, Hkv, D), "f32", 1.0, seed, 1)
    XV = normal_fill((prefix, Hkv, D), "f32", 1.0, seed, 2)
    Y = [normal_fill((n, Hkv, D), "f32", 1.0, seed, 3 + i) for i, n in enumerate((3, 6))]
    YV = [normal_fill((n, Hkv, D), "f32", 1.0, seed, 5 + i) for i, n in enumerate((3, 6))]
    q = normal_fill((2, Hkv, D), "f32", 1.0, seed, 7)
    nb = 16

    def write(bm, k, v, s, K, V):
        for t in range(K.shape[0]):
            slot, src, dst = bm.append_slot(s)
            if src >= 0:
                ocache.copy_blocks(k, v, [(src, dst)])
            ocache.reshape_and_cache(K[t:t + 1], V[t:t + 1], k, v, [slot], bs)

    outs = []
    for shared in (True, False):
        k = np.zeros((nb, Hkv, bs, D), np.float32)
        v = np.zeros_like(k)
        bm = bm_cls(nb, bs)
        bm.add(0, 0)
        write(bm, k, v, 0, X, XV)
        if shared:
            bm.fork(0, 1)
        else:
            bm.add(1, 0)
            write(bm, k, v, 1, X, XV)
        write(bm, k, v, 0, Y[0], YV[0])
        write(bm, k, v, 1, Y[1], YV[1])
        rows, sl = bm.block_tables([0, 1], 6)
        outs.append(att.paged_decode_attention(q, k, v, np.array(rows, np.int32),
                                               np.array(sl, np.int32), 0.25, bs, Hkv, "f32"))
    return float(np.abs(outs[0] - outs[1]).max())


# ---------------------------------------------------------------------------
# attention pins
# ---------------------------------------------------------------------------

def test_matches_sdpa_mha_fp32():
    assert check_against_sdpa() < 1e-12


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_matches_sdpa_gqa_half(dtype):
    assert check_against_sdpa(lens=(1, 16, 33, 50), Hq=8, Hkv=2, D=32, bs=8,
                              dtype=dtype, scale=1 / math.sqrt(32)) < 1e-12


def test_matches_textbook_loops():
    assert check_against_loops() < 1e-12


def test_single_token_is_its_value():
    g = np.random.default_rng(0)
    q, K, V = g.standard_normal(32), g.standard_normal((1, 32)), g.standard_normal((1, 32))
    assert np.array_equal(oatt.softmax_attention(q, K, V, 0.3), V[0])


def test_identical_keys_give_mean_value():
    g = np.random.default_rng(1)
    q, V = g.standard_normal(32), g.standard_normal((37, 32))
    K = np.tile(g.standard_normal(32), (37, 1))
    np.testing.assert_allclose(oatt.softmax_attention(q, K, V, 0.3), V.mean(0), rtol=0,
                               atol=1e-13)


def test_dominant_logit_selects_its_value():
    g = np.random.default_rng(2)
    D, L = 16, 50
    q = np.zeros(D)
    q[0] = 1.0
    K = g.standard_normal((L, D)) * 0.1
    K[23, 0] = 60.0
    V = g.standard_normal((L, D))
    out = oatt.softmax_attention(q, K, V, 1.0)
    assert np.abs(out - V[23]).max() <= 1e-15 * np.abs(V).max()


def test_empty_sequence_gives_zeros():
    q = np.ones((1, 2, 8), np.float32)
    k = np.ones((2, 2, 4, 8), np.float32)
    out = oatt.paged_decode_attention(q, k, k, np.array([[-1]], np.int32),
                                      np.array([0], np.int32), 1.0, 4, 2, "f32")
    assert np.array_equal(out, np.zeros((1, 2, 8)))


def test_partition_size_invariance():
    assert check_partition_invariance() < 1e-12


def test_block_permutation_invariance():
    assert check_block_permutation() == 0.0


def test_prefix_sharing_invariance():
    assert check_prefix_sharing() == 0.0


def test_page_table_reading_order(golden):
    """[LAB] 'Keep pages in order': logical 0->6, 1->1, 2->8 reads blocks 6, 1, 8.
    Each page is stored as one slot holding its phrase id (block size 1), so the walk
    through the table must spell the sentence in logical order."""
    ex = golden["page_table"]
    phrases = {int(b): text for b, text in ex["contents_printed"].items()}
    cache = np.full((ex["pool_blocks"], 1, 1, 1), -1.0, np.float32)
    for b in phrases:
        cache[b, 0, 0, 0] = b
    table = ex["table_printed"]
    rows = oatt.gather_sequence(cache, table, len(table), 1, 0)
    order = [int(r) for r in rows[:, 0]]
    assert order == table
    assert " ".join(phrases[b] for b in order) == ex["reading_order_implied"]


# ---------------------------------------------------------------------------
# cache-op pins
# ---------------------------------------------------------------------------

def test_reshape_and_cache_matches_flat_slot_view():
    """A slot number indexes the (block, offset) pair of the cache seen as
    [num_blocks * block_size] token rows; numpy's own reshape defines that view."""
    g = np.random.default_rng(5)
    NB, Hkv, bs, D, T = 6, 3, 4, 8, 9
    k = g.standard_normal((NB, Hkv, bs, D)).astype(np.float32)
    v = g.standard_normal((NB, Hkv, bs, D)).astype(np.float32)
    key = g.standard_normal((T, Hkv, D)).astype(np.float32)
    val = g.standard_normal((T, Hkv, D)).astype(np.float32)
    slots = g.choice(NB * bs, T, replace=False).astype(np.int64)
    slots[4] = -1
    k0, v0 = k.copy(), v.copy()
    ocache.reshape_and_cache(key, val, k, v, slots, bs)
    flat_k = k0.transpose(0, 2, 1, 3).reshape(NB * bs, Hkv, D).copy()
    flat_v = v0.transpose(0, 2, 1, 3).reshape(NB * bs, Hkv, D).copy()
    keep = slots >= 0
    flat_k[slots[keep]] = key[keep]
    flat_v[slots[keep]] = val[keep]
    assert np.array_equal(k, flat_k.reshape(NB, bs, Hkv, D).transpose(0, 2, 1, 3))
    assert np.array_equal(v, flat_v.reshape(NB, bs, Hkv, D).transpose(0, 2, 1, 3))


def test_copy_blocks_copies_whole_blocks_only():
    g = np.random.default_rng(6)
    k = g.integers(0, 1 << 16, (8, 2, 4, 8)).astype(np.uint16)
    v = g.integers(0, 1 << 16, (8, 2, 4, 8)).astype(np.uint16)
    k0, v0 = k.copy(), v.copy()
    ocache.copy_blocks(k, v, [(1, 5), (1, 6), (3, 0)])
    expect_k = k0.copy()
    expect_k[[5, 6, 0]] = k0[[1, 1, 3]]
    assert np.array_equal(k, expect_k)
    assert np.array_equal(v[[5, 6, 0]], v0[[1, 1, 3]])
    untouched = [1, 2, 3, 4, 7]
    assert np.array_equal(v[untouched], v0[untouched])


# ---------------------------------------------------------------------------
# allocator pins: worked examples and invariants
# ---------------------------------------------------------------------------

def test_reservation_example(golden):
    ex = golden["reservation"]
    r = contiguous_reservation(ex["used"], ex["reserved"])
    assert r["empty"] == ex["empty_printed"]
    assert round(100 * r["wasted_fraction"]) == ex["wasted_percent_printed"]


def test_page_growth_example(golden):
    ex = golden["page_growth"]
    r = paged_growth(ex["tokens_printed"], ex["tokens_per_page"])
    assert r["logical_pages"] == ex["logical_pages_printed"]
    assert r["pages"] == ex["pages_implied"] and r["empty_slots"] == ex["empty_slots_implied"]
    assert r["slots"] == 12


def test_batch_memory_example(golden):
    ex = golden["batch"]
    r = batch_memory(ex["lengths_printed"], ex["block_size_implied"], ex["reservation_printed"])
    assert r["contiguous_slots"] == ex["contiguous_slots_printed"]
    assert r["paged_slots"] == ex["paged_slots_printed"]
    assert r["stored_tokens"] == ex["stored_tokens_printed"]
    assert round(100 * r["saving_fraction"]) == ex["saving_percent_printed"]
    assert r["blocks"] == [2, 4, 2, 5, 3]


def test_paged_waste_under_four_percent_at_block_16(golden):
    """[BLOG]: the only waste is each sequence's last partial block; 'under 4%' holds
    for the 7B-shaped lengths at the default block size 16."""
    from workloads import draw_lengths
    lens, _ = draw_lengths(CONFIGS["7b_bf16"], 0)
    r = batch_memory(lens.tolist(), golden["paged_waste_bound"]["default_block_size_printed"],
                     2048)
    assert 100 * r["paged_waste_fraction"] < golden["paged_waste_bound"]["waste_percent_bound_printed"]


def _invariants(bm: BlockManager):
    counts = [0] * bm.num_blocks
    for t in bm.tables.values():
        for b in t:
            counts[b] += 1
    assert counts == bm.ref
    free = set(bm.free)
    assert len(free) == len(bm.free)
    used = {b for b in range(bm.num_blocks) if bm.ref[b] > 0}
    assert free.isdisjoint(used) and free | used == set(range(bm.num_blocks))
    for s, t in bm.tables.items():
        L = bm.lens[s]
        assert len(t) == -(-L // bm.block_size)
        assert len(t) * bm.block_size - L < bm.block_size


def random_ops(bm: BlockManager, g: np.random.Generator, n_ops: int, check=None):
    live, next_id = [], 0
    log = []
    for _ in range(n_ops):
        op = g.integers(0, 10)
        try:
            if op < 2 or not live:
                n = int(g.integers(0, 3 * bm.block_size))
                bm.add(next_id, n)
                log.append(("add", next_id, n))
                live.append(next_id)
                next_id += 1
            elif op < 4:
                p = live[int(g.integers(0, len(live)))]
                bm.fork(p, next_id)
                log.append(("fork", p, next_id))
                live.append(next_id)
                next_id += 1
            elif op < 9:
                s = live[int(g.integers(0, len(live)))]
                log.append(("append", s, bm.append_slot(s)))
            elif g.integers(0, 2):
                s = live.pop(int(g.integers(0, len(live))))
                bm.free_seq(s)
                log.append(("free", s))
            else:
                s = live[int(g.integers(0, len(live)))]
                n = int(g.integers(0, bm.lens[s] + 1))
                bm.truncate([s], [n])
                log.append(("truncate", s, n))
        except AllocError as e:
            log.append(("error", e.code))
        if check:
            check(bm)
    return log


def test_allocator_invariants_random():
    g = np.random.default_rng(7)
    for trial in range(20):
        bm = BlockManager(24, 4, g.permutation(24))
        random_ops(bm, g, 300, _invariants)


def test_append_after_full_shared_block_needs_no_copy():
    bm = BlockManager(8, 4)
    bm.add(0, 8)              # two full blocks
    bm.fork(0, 1)
    slot, src, dst = bm.append_slot(1)
    assert (src, dst) == (-1, -1) and bm.tables[1][:2] == bm.tables[0]
    assert len(bm.tables[1]) == 3 and slot == bm.tables[1][2] * 4


def test_write_into_shared_block_copies_first():
    bm = BlockManager(8, 4, [3, 1, 4, 0, 5, 2, 6, 7])
    bm.add(0, 6)              # blocks 3, 1; last block half full
    bm.fork(0, 1)
    slot, src, dst = bm.append_slot(1)
    assert (src, dst) == (1, 4) and bm.ref[1] == 1 and bm.ref[4] == 1
    assert slot == 4 * 4 + 2
    slot0, src0, _ = bm.append_slot(0)   # now sole owner of block 1: no copy
    assert src0 == -1 and slot0 == 1 * 4 + 2


def test_full_pool_fails_without_changing_state():
    bm = BlockManager(3, 4)
    bm.add(0, 12)
    before = bm.stats(), dict(bm.tables), list(bm.free)
    with pytest.raises(AllocError) as e:
        bm.append_slot(0)
    assert e.value.code == "NO_FREE_BLOCKS"
    assert (bm.stats(), dict(bm.tables), list(bm.free)) == before
    with pytest.raises(AllocError):
        bm.add(1, 1)
    bm.fork(0, 1)
    with pytest.raises(AllocError):
        bm.append_slots([0, 1])
    assert bm.lens == {0: 12, 1: 12}


def test_fork_step_copy_count_prefix_workload():
    """32 groups x 8 samples on a 1030-token prefix (last block 6/16 full, shared by 8):
    the first 7 samples of each group copy, the 8th writes in place: 224 copies."""
    from oracle.step import build_context
    cfg = CONFIGS["prefix_cow_bf16"]
    inp = make_inputs(cfg, 0, fork_step=True, pool=False)
    bm, _, _, build_pairs = build_context(inp, copy_pool=False)
    assert build_pairs == []
    res = bm.append_slots(range(cfg.num_seqs))
    pairs = [(r[1], r[2]) for r in res if r[1] >= 0]
    assert len(pairs) == 224
    assert len({d for _, d in pairs}) == 224 and not ({d for _, d in pairs} & {s for s, _ in pairs})
    _invariants(bm)


def test_truncate_then_append_reuses_the_released_block():
    """Dropping a token that opened a block returns that block; appending again takes
    it back (LIFO pool) - a rolled-back decode step leaves the state as it was."""
    bm = BlockManager(8, 4, [5, 2, 7, 0, 1, 3, 4, 6])
    bm.add(0, 8)
    before = (bm.stats(), list(bm.free), [list(t) for t in bm.tables.values()])
    slot, _, _ = bm.append_slot(0)
    assert slot == 7 * 4
    bm.truncate([0], [8])
    after = (bm.stats(), list(bm.free), [list(t) for t in bm.tables.values()])
    assert before[1:] == after[1:] and before[0]["logical_tokens"] == after[0]["logical_tokens"]
    with pytest.raises(AllocError):
        bm.truncate([0], [9])


def test_truncate_keeps_shared_blocks_shared():
    bm = BlockManager(8, 4)
    bm.add(0, 6)
    bm.fork(0, 1)
    bm.truncate([1], [3])            # still inside block 0: nothing released
    assert bm.ref[0] == 2 and bm.ref[1] == 1 and len(bm.tables[1]) == 1
    _, src, dst = bm.append_slot(1)  # writing into the shared block copies it
    assert src == 0 and bm.ref[0] == 1
    _invariants(bm)


# ---------------------------------------------------------------------------
# widening of stored values: oracle.numerics.to_f64 against the IEEE-754 binary
# formats decoded from their definition and against torch's own dtype casts
# ([LAB] "Measure memory use across requests": paging leaves the attention
# equation unchanged, so the stored bits must widen to exactly their value)
# ---------------------------------------------------------------------------

def _decode_binary(bits: int, exp_bits: int, man_bits: int) -> float:
    """Value of an IEEE-754 binary pattern from the format's definition: sign bit,
    biased exponent, fraction; exponent 0 is subnormal, all ones is inf / NaN."""
    sign = -1.0 if (bits >> (exp_bits + man_bits)) & 1 else 1.0
    e = (bits >> man_bits) & ((1 << exp_bits) - 1)
    f = bits & ((1 << man_bits) - 1)
    bias = (1 << (exp_bits - 1)) - 1
    if e == (1 << exp_bits) - 1:
        return sign * math.inf if f == 0 else math.nan
    if e == 0:
        return sign * math.ldexp(f, 1 - bias - man_bits)
    return sign * math.ldexp((1 << man_bits) + f, e - bias - man_bits)


def _same_f64(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Element-wise exact equality of float64 values, NaN equal to NaN, -0 != +0."""
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    both_nan = np.isnan(a) & np.isnan(b)
    return both_nan | (a.view(np.uint64) == b.view(np.uint64))


# hand values: (dtype, bit pattern, value)
_HAND_VALUES = [
    ("bf16", 0x3F80, 1.0), ("bf16", 0xC000, -2.0), ("bf16", 0x0001, 2.0 ** -133),
    ("bf16", 0x0080, 2.0 ** -126), ("bf16", 0x7F7F, (2 - 2.0 ** -7) * 2.0 ** 127),
    ("bf16", 0x7F80, math.inf), ("bf16", 0xFF80, -math.inf), ("bf16", 0x7FC0, math.nan),
    ("bf16", 0x8000, -0.0), ("bf16", 0x3E00, 0.125), ("bf16", 0x4049, 3.140625),
    ("f16", 0x3C00, 1.0), ("f16", 0xC000, -2.0), ("f16", 0x0001, 2.0 ** -24),
    ("f16", 0x0400, 2.0 ** -14), ("f16", 0x7BFF, 65504.0), ("f16", 0x7C00, math.inf),
    ("f16", 0xFC00, -math.inf), ("f16", 0x7E00, math.nan), ("f16", 0x8000, -0.0),
    ("f16", 0x3555, 0.333251953125),
    ("f32", 0x3F800000, 1.0), ("f32", 0x00000001, 2.0 ** -149),
    ("f32", 0x7F7FFFFF, (2 - 2.0 ** -23) * 2.0 ** 127), ("f32", 0xFF800000, -math.inf),
]


def _storage_from_bits(bits: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bits.astype(np.uint16)
    if dtype == "f16":
        return bits.astype(np.uint16).view(np.float16)
    return bits.astype(np.uint32).view(np.float32)


def check_widening(fn=None, seed=12) -> int:
    """Number of stored bit patterns whose widened value differs from (a) the format's
    definition, (b) torch's cast of the same bits, or (c) the hand values.  Covers all
    65 536 bf16 and f16 patterns and 40 000 float32 patterns (random plus specials)."""
    if fn is None:
        from oracle import numerics
        fn = numerics.to_f64
    bad = 0
    all16 = np.arange(1 << 16, dtype=np.uint32)
    g = np.random.default_rng(seed)
    f32 = np.concatenate([g.integers(0, 1 << 32, 40000 - 8, dtype=np.uint64).astype(np.uint32),
                          np.array([0, 0x80000000, 1, 0x807FFFFF, 0x7F800000, 0x7FC00000,
                                    0x3F800000, 0xBF800000], np.uint32)])
    for dtype, bits, (eb, mb), tview in (("bf16", all16, (8, 7), torch.bfloat16),
                                         ("f16", all16, (5, 10), torch.float16),
                                         ("f32", f32, (8, 23), torch.float32)):
        got = np.asarray(fn(_storage_from_bits(bits, dtype), dtype), np.float64)
        if got.shape != bits.shape:
            return bits.size
        definition = np.array([_decode_binary(int(b), eb, mb) for b in bits])
        if dtype == "f32":
            t = torch.from_numpy(bits.astype(np.uint32).view(np.int32)).view(torch.float32)
        else:
            t = torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(tview)
        by_torch = t.double().numpy()
        bad += int((~_same_f64(got, definition)).sum()) + int((~_same_f64(got, by_torch)).sum())
    for dtype, b, value in _HAND_VALUES:
        got = np.asarray(fn(_storage_from_bits(np.array([b], np.uint32), dtype), dtype))
        bad += int(not _same_f64(got, np.array([value]))[0])
    return bad


def test_widening_matches_the_formats_exactly():
    assert check_widening() == 0


def test_format_decoder_matches_hand_values():
    """The definition decoder above, checked by itself on the hand values."""
    for dtype, b, value in _HAND_VALUES:
        eb, mb = {"bf16": (8, 7), "f16": (5, 10), "f32": (8, 23)}[dtype]
        assert _same_f64(np.array([_decode_binary(b, eb, mb)]), np.array([value]))[0]


# ---------------------------------------------------------------------------
# moving sequences between two pools (swap out / in): the block manager's move
# ---------------------------------------------------------------------------

class _Contents:
    """What each sequence has written, and what each physical slot holds.

    Token ids are unique integers.  Writes follow the block manager's slots and
    copy-on-write pairs; a move copies the blocks its pairs name.  Reading a
    sequence back through its block table must give exactly the tokens that
    sequence was given ([BLOG] "The bonus contiguous storage can't give you:
    sharing": sharing and copy-on-write never change what a sequence reads)."""

    def __init__(self, pools):
        self.mem = {id(p): np.full((p.num_blocks, p.block_size), -1, np.int64) for p in pools}
        self.tokens = {}
        self.next_tok = 0

    def _fresh(self, n):
        t = list(range(self.next_tok, self.next_tok + n))
        self.next_tok += n
        return t

    def add(self, bm, s, n):
        bm.add(s, n)
        toks = self._fresh(n)
        mem = self.mem[id(bm)]
        for t, tok in enumerate(toks):
            mem[bm.tables[s][t // bm.block_size], t % bm.block_size] = tok
        self.tokens[s] = toks

    def fork(self, bm, p, c):
        bm.fork(p, c)
        self.tokens[c] = list(self.tokens[p])

    def append(self, bm, s):
        slot, src, dst = bm.append_slot(s)
        mem = self.mem[id(bm)]
        if src >= 0:
            mem[dst] = mem[src]
        tok = self._fresh(1)[0]
        mem[slot // bm.block_size, slot % bm.block_size] = tok
        self.tokens[s].append(tok)

    def free(self, bm, s):
        bm.free_seq(s)
        del self.tokens[s]

    def move(self, src_bm, dst_bm, ids):
        pairs = src_bm.move_to(dst_bm, ids)
        ms, md = self.mem[id(src_bm)], self.mem[id(dst_bm)]
        for a, b in pairs:
            md[b] = ms[a]
        return pairs

    def check(self, bm):
        mem = self.mem[id(bm)]
        for s, table in bm.tables.items():
            L = bm.lens[s]
            read = [int(mem[table[t // bm.block_size], t % bm.block_size]) for t in range(L)]
            assert read == self.tokens[s], s


def check_moves(bm_cls=BlockManager, seed=21, trials=6, n_ops=250):
    """Random add / fork / append / free / move-out / move-in sequences over two pools.
    After every op: the invariants on both pools (counts = table entries, free and
    used partition each pool, ceil(L/bs) blocks), every sequence reads back exactly
    its own tokens, and each move's pairs are the moved set's distinct blocks in
    first-appearance order with distinct fresh destinations."""
    g = np.random.default_rng(seed)
    for _ in range(trials):
        bs = int(g.choice([1, 2, 4]))
        A = bm_cls(40, bs, g.permutation(40))
        B = bm_cls(30, bs, g.permutation(30))
        C = _Contents([A, B])
        where, nid = {}, 0
        for _ in range(n_ops):
            r = int(g.integers(0, 10))
            pool = A if g.integers(0, 3) else B
            mine = [s for s, p in where.items() if p is pool]
            try:
                if r < 2 or not mine:
                    C.add(pool, nid, int(g.integers(0, 3 * bs + 1)))
                    where[nid] = pool
                    nid += 1
                elif r < 4:
                    C.fork(pool, mine[int(g.integers(0, len(mine)))], nid)
                    where[nid] = pool
                    nid += 1
                elif r < 6:
                    C.append(pool, mine[int(g.integers(0, len(mine)))])
                elif r < 7:
                    s = mine[int(g.integers(0, len(mine)))]
                    C.free(pool, s)
                    del where[s]
                else:
                    other = B if pool is A else A
                    k = int(g.integers(1, min(4, len(mine)) + 1))
                    ids = [int(x) for x in g.choice(mine, k, replace=False)]
                    old = {s: list(pool.tables[s]) for s in ids}
                    free_before = other.free_list()
                    pairs = C.move(pool, other, ids)
                    distinct = list(dict.fromkeys(b for s in ids for b in old[s]))
                    assert [a for a, _ in pairs] == distinct
                    assert [b for _, b in pairs] == free_before[:len(distinct)]
                    m = dict(pairs)
                    for s in ids:
                        assert other.tables[s] == [m[b] for b in old[s]]
                        where[s] = other
            except AllocError:
                pass
            for p in (A, B):
                _invariants(p)
                C.check(p)
    return True


def test_moves_keep_invariants_and_contents():
    assert check_moves()


def test_move_hand_case_shared_block_becomes_private():
    """Worked by hand.  Pool A pops 5, 3, 7, 0, ...; pool B pops 2, 0, 1, 3.
    seq 0 holds 10 tokens at 4 per block: blocks 5, 3, 7 (7 half full).  seqs 1 and 2
    fork from it (every count 3).  seq 2 appends: block 7 is shared, so it copies
    7 -> 0 (7 drops to 2).  Moving seqs 0 and 1 to B: their distinct blocks 5, 3, 7
    get B's 2, 0, 1, shared by both (count 2 each).  In A, seq 2 keeps 5 and 3, now
    private (count 1), and block 7 reaches zero and goes back on top of A's stack."""
    A = BlockManager(8, 4, [5, 3, 7, 0, 1, 2, 4, 6])
    B = BlockManager(4, 4, [2, 0, 1, 3])
    A.add(0, 10)
    A.fork(0, 1)
    A.fork(0, 2)
    assert A.tables[0] == [5, 3, 7] and A.ref[5] == A.ref[3] == A.ref[7] == 3
    slot, src, dst = A.append_slot(2)
    assert (src, dst) == (7, 0) and slot == 0 * 4 + 2 and A.ref[7] == 2
    pairs = A.move_to(B, [0, 1])
    assert pairs == [(5, 2), (3, 0), (7, 1)]
    assert B.tables[0] == B.tables[1] == [2, 0, 1] and B.lens == {0: 10, 1: 10}
    assert [B.ref[b] for b in (2, 0, 1)] == [2, 2, 2] and B.free_list() == [3]
    assert A.tables == {2: [5, 3, 0]} and A.lens == {2: 11}
    assert [A.ref[b] for b in (5, 3, 0, 7)] == [1, 1, 1, 0]
    assert A.free_list() == [7, 1, 2, 4, 6]
    _invariants(A)
    _invariants(B)


# ---------------------------------------------------------------------------
# prefix groups: a fork forest worked by hand
# ---------------------------------------------------------------------------

def _fork_forest(bm_cls=BlockManager):
    """Block size 4, a 32-block pool taken in index order.
      seq 10: 20 tokens (5 full blocks); 11 and 12 fork from it.
      11 appends 1 token (a fresh sixth block).  12 is truncated to 9 tokens and
      appends one: its third block was shared, so it copies (tables diverge after
      2 blocks).  50 forks from 10 at the end.
      seq 20: 12 tokens (3 full blocks); 21 forks and appends 1 (a fresh block).
      seq 30: 3 tokens (1 block); 31 forks from it.
      seq 40: 16 tokens, alone.
    Batch order [40, 10, 20, 11, 30, 12, 21, 31, 50] (positions 0..8)."""
    bm = bm_cls(32, 4)
    bm.add(10, 20)
    bm.fork(10, 11)
    bm.fork(10, 12)
    bm.append_slot(11)
    bm.truncate([12], [9])
    bm.append_slot(12)
    bm.add(20, 12)
    bm.fork(20, 21)
    bm.append_slot(21)
    bm.add(30, 3)
    bm.fork(30, 31)
    bm.add(40, 16)
    bm.fork(10, 50)
    return bm, [40, 10, 20, 11, 30, 12, 21, 31, 50]


# (partition_size, max_members) -> (prefix_parts per position, chunks)
# group of 10 (positions 1, 3, 5, 8): common prefix 2 blocks = 8 tokens;
# group of 20 (positions 2, 6): 3 blocks = 12 tokens; group of 30 (4, 7): 1 block
# = 4 tokens; 40 (position 0) is alone.  parts = floor(common tokens / partition).
_FOREST_EXPECTED = {
    (8, 2): ([0, 1, 1, 1, 0, 1, 1, 0, 1], [([1, 3], 1), ([5, 8], 1), ([2, 6], 1)]),
    (8, 8): ([0, 1, 1, 1, 0, 1, 1, 0, 1], [([1, 3, 5, 8], 1), ([2, 6], 1)]),
    (4, 3): ([0, 2, 3, 2, 1, 2, 3, 1, 2],
             [([1, 3, 5], 2), ([8], 2), ([2, 6], 3), ([4, 7], 1)]),
    (16, 8): ([0] * 9, []),
}


def check_prefix_groups(bm_cls=BlockManager) -> int:
    """Number of (partition, max_members) cases whose groups differ from the hand
    values above."""
    bm, ids = _fork_forest(bm_cls)
    bad = 0
    for (ps, mm), (parts, chunks) in _FOREST_EXPECTED.items():
        got_parts, got_chunks = bm.prefix_groups(ids, ps, mm)
        got = (list(got_parts), [(list(m), int(p)) for m, p in got_chunks])
        bad += int(got != (parts, chunks))
    return bad


def test_prefix_groups_of_a_hand_built_fork_forest():
    bm, _ = _fork_forest()
    assert bm.tables[10] == [0, 1, 2, 3, 4] and bm.tables[11] == [0, 1, 2, 3, 4, 5]
    assert bm.tables[12] == [0, 1, 6] and bm.tables[50] == [0, 1, 2, 3, 4]
    assert bm.tables[20] == [7, 8, 9] and bm.tables[21] == [7, 8, 9, 10]
    assert bm.tables[30] == bm.tables[31] == [11] and bm.tables[40] == [12, 13, 14, 15]
    assert check_prefix_groups() == 0
