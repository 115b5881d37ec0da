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
from oracle.numerics import to_f64
from oracle.waste import batch_memory, contiguous_reservation, paged_growth
from workloads import CONFIGS, make_inputs, normal_fill

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
    contiguous K/V (query head h reads kv head h // (Hq/Hkv) via repeat_interleave)."""
    Ks, Vs, q = _draw_contiguous(lens, Hq, Hkv, D, dtype, seed)
    nb = sum(-(-L // bs) for L in lens) + 3
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    k, v, tables, seq_lens = _paged_from_contiguous(Ks, Vs, bs, nb, order, Hkv, D, dtype,
                                                    reshape=reshape)
    out = att.paged_decode_attention(q, k, v, tables, seq_lens, scale, bs, Hkv, dtype)
    worst = 0.0
    G = Hq // Hkv
    for s, L in enumerate(lens):
        Kt = torch.from_numpy(to_f64(Ks[s], dtype)).permute(1, 0, 2)   # [Hkv, L, D]
        Vt = torch.from_numpy(to_f64(Vs[s], dtype)).permute(1, 0, 2)
        Kt, Vt = Kt.repeat_interleave(G, 0), Vt.repeat_interleave(G, 0)
        qt = torch.from_numpy(to_f64(q[s], dtype)).unsqueeze(1)        # [Hq, 1, D]
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
