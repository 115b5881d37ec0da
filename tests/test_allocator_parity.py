"""The C++ block manager in libpa.so against the oracle's model, bit for bit:
slots, copy-on-write pairs, block tables, reference counts, free-pool order and
statistics after every operation; errors leave both unchanged.  Host only."""
import numpy as np
import pytest

from oracle.allocator import AllocError, BlockManager
from workloads import CONFIGS, make_inputs


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_342_b200 as m
    return m


def same_state(c, o: BlockManager):
    assert c.stats() == o.stats()
    assert c.free_list() == o.free_list()
    for b in range(o.num_blocks):
        assert c.refcount(b) == o.ref[b]
    for s, t in o.tables.items():
        assert c.seq_blocks(s) == t
        assert c.seq_len(s) == o.lens[s]


def run_both(pa, c, o, op, *args):
    """Apply one op to both; both must succeed with equal results or fail alike."""
    err_c = err_o = None
    res_c = res_o = None
    try:
        res_c = getattr(c, op)(*args)
    except pa.PagedAttentionError as e:
        err_c = e.code
    try:
        res_o = getattr(o, {"free": "free_seq"}.get(op, op))(*args)
    except AllocError as e:
        err_o = e.code
    assert err_c == err_o, (op, args, err_c, err_o)
    return res_c, res_o


@pytest.mark.parametrize("seed", range(6))
def test_random_op_sequences(pa, seed):
    g = np.random.default_rng(seed)
    nb, bs = int(g.integers(8, 40)), int(g.choice([1, 2, 4, 16]))
    order = g.permutation(nb)
    c, o = pa.BlockAllocator(nb, bs, order), BlockManager(nb, bs, order)
    live, next_id = [], 0
    for step in range(400):
        op = int(g.integers(0, 12))
        if op < 2 or not live:
            n = int(g.integers(0, 3 * bs + 1))
            run_both(pa, c, o, "add", next_id, n)
            if next_id in o.tables:
                live.append(next_id)
            next_id += 1
        elif op < 4:
            p = live[int(g.integers(0, len(live)))]
            run_both(pa, c, o, "fork", p, next_id)
            if next_id in o.tables:
                live.append(next_id)
            next_id += 1
        elif op < 8:
            s = live[int(g.integers(0, len(live)))]
            rc, ro = run_both(pa, c, o, "append_slot", s)
            assert rc == ro
        elif op < 10:
            k = int(g.integers(1, 6))
            ids = [live[int(i)] for i in g.integers(0, len(live), k)]
            rc, ro = run_both(pa, c, o, "append_slots", ids)
            if ro is not None:
                slots, pairs = rc
                assert slots.tolist() == [r[0] for r in ro]
                assert [tuple(p) for p in pairs.tolist()] == [(r[1], r[2]) for r in ro if r[1] >= 0]
        elif op < 11:
            if g.integers(0, 2):
                s = live.pop(int(g.integers(0, len(live))))
                run_both(pa, c, o, "free", s)
            else:
                k = int(g.integers(1, 4))
                ids = [live[int(i)] for i in g.integers(0, len(live), k)]
                ids = list(dict.fromkeys(ids))
                lens = [int(g.integers(0, o.lens[i] + 2)) for i in ids]   # may be too long
                run_both(pa, c, o, "truncate", ids, lens)
        else:
            run_both(pa, c, o, "free", 10_000 + step)      # unknown id
            run_both(pa, c, o, "fork", 10_000 + step, 20_000 + step)
            if live:
                run_both(pa, c, o, "add", live[0], 3)        # exists
        same_state(c, o)
    ids = sorted(o.tables)
    if ids:
        width = max(len(o.tables[s]) for s in ids) + 2
        t_c, l_c = c.build_block_tables(ids, width)
        rows, lens = o.block_tables(ids, width)
        assert t_c.tolist() == rows and l_c.tolist() == lens


def test_failed_batch_changes_nothing(pa):
    c, o = pa.BlockAllocator(5, 4), BlockManager(5, 4)
    for m in (c, o):
        m.add(0, 6)          # 2 blocks, last half full
        m.fork(0, 1)
        m.add(2, 8)          # 2 full blocks
    # seq 0: copy (1 block), seq 1: in place, seq 2: new block, seq 2 again: in place
    # -> needs 2 blocks, pool has 1
    run_both(pa, c, o, "append_slots", [0, 1, 2, 2, 2, 2, 2])
    same_state(c, o)
    rc, ro = run_both(pa, c, o, "append_slots", [0, 1])
    same_state(c, o)


@pytest.mark.parametrize("name", ["tiny_fp32", "7b_bf16", "13b_fp16", "gqa_long_bf16"])
def test_workload_context_and_step(pa, name):
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, 0, pool=False)
    c = pa.BlockAllocator(cfg.num_blocks, cfg.block_size, inp.free_order)
    o = BlockManager(cfg.num_blocks, cfg.block_size, inp.free_order)
    for s in range(cfg.num_seqs):
        c.add(s, int(inp.context_lens[s]))
        o.add(s, int(inp.context_lens[s]))
    slots, pairs = c.append_slots(range(cfg.num_seqs))
    ro = o.append_slots(range(cfg.num_seqs))
    assert slots.tolist() == [r[0] for r in ro] and len(pairs) == 0
    assert c.stats() == o.stats() and c.free_list() == o.free_list()


@pytest.mark.parametrize("fork_step", [False, True])
def test_prefix_workload(pa, fork_step):
    from oracle.step import build_context
    from paged_kv_cache_342_b200.runtime import PagedDecoder  # noqa: F401 (import check)
    cfg = CONFIGS["prefix_cow_bf16"]
    inp = make_inputs(cfg, 0, fork_step=fork_step, pool=False)
    o, _, _, build_pairs = build_context(inp, copy_pool=False)
    c = pa.BlockAllocator(cfg.num_blocks, cfg.block_size, inp.free_order)
    p = inp.prefix
    cp = []
    for gi in range(p.groups):
        c.add(gi * p.samples, p.prefix_len)
        for i in range(1, p.samples):
            c.fork(gi * p.samples, gi * p.samples + i)
    for s in range(cfg.num_seqs):
        for _ in range(int(p.private_lens[s])):
            _, src, dst = c.append_slot(s)
            if src >= 0:
                cp.append((src, dst))
    assert cp == build_pairs
    slots, pairs = c.append_slots(range(cfg.num_seqs))
    ro = o.append_slots(range(cfg.num_seqs))
    assert slots.tolist() == [r[0] for r in ro]
    assert [tuple(x) for x in pairs.tolist()] == [(r[1], r[2]) for r in ro if r[1] >= 0]
    if fork_step:
        assert len(pairs) == 224
    assert c.stats() == o.stats()
    assert c.stats()["cow_copies"] == len(build_pairs) + len(pairs)


def test_stats_match_worked_batch_example(pa, golden):
    ex = golden["batch"]
    c = pa.BlockAllocator(64, ex["block_size_implied"])
    for i, n in enumerate(ex["lengths_printed"]):
        c.add(i, n)
    st = c.stats()
    assert st["allocated_slots"] == ex["paged_slots_printed"]
    assert st["logical_tokens"] == ex["stored_tokens_printed"]


def test_bad_create_arguments(pa):
    with pytest.raises(pa.PagedAttentionError):
        pa.BlockAllocator(4, 4, [0, 1, 1, 2])        # not a permutation
    with pytest.raises(pa.PagedAttentionError):
        pa.BlockAllocator(0, 4)


def _compare_groups(c, o, ids, ps, mm):
    pp, cm, cp, mp = c.prefix_groups(ids, ps, mm)
    opp, ochunks = o.prefix_groups(ids, ps, mm)
    assert pp.tolist() == opp
    assert [(row[row >= 0].tolist(), int(parts)) for row, parts in zip(cm, cp)] == \
        [(list(m), p) for m, p in ochunks]
    assert mp == max([p for _, p in ochunks], default=0)
    return ochunks


@pytest.mark.parametrize("seed", range(4))
def test_prefix_groups_random_forks(pa, seed):
    """Fork forests with appends, copies and frees: both sides find the same groups."""
    g = np.random.default_rng(100 + seed)
    bs = int(g.choice([2, 4, 16]))
    nb = 400
    c, o = pa.BlockAllocator(nb, bs), BlockManager(nb, bs)
    live, nid = [], 0
    for _ in range(60):
        r = g.integers(0, 10)
        if r < 3 or not live:
            n = int(g.integers(0, 6 * bs))
            c.add(nid, n), o.add(nid, n)
            live.append(nid)
            nid += 1
        elif r < 6:
            p = live[int(g.integers(0, len(live)))]
            c.fork(p, nid), o.fork(p, nid)
            live.append(nid)
            nid += 1
        elif r < 9:
            s = live[int(g.integers(0, len(live)))]
            for _ in range(int(g.integers(1, 2 * bs))):
                assert c.append_slot(s) == o.append_slot(s)
        else:
            s = live.pop(int(g.integers(0, len(live))))
            c.free(s), o.free_seq(s)
    ids = list(g.permutation(live))
    for ps in (bs, 2 * bs, 4 * bs):
        for mm in (1, 2, 3, 8):
            _compare_groups(c, o, ids, ps, mm)


def test_prefix_groups_of_the_shared_prefix_workload(pa):
    from oracle.step import build_context
    cfg = CONFIGS["prefix_cow_bf16"]
    inp = make_inputs(cfg, 0, pool=False)
    o, _, _, _ = build_context(inp, copy_pool=False)
    c = pa.BlockAllocator(cfg.num_blocks, cfg.block_size, inp.free_order)
    p = inp.prefix
    for gi in range(p.groups):
        c.add(gi * p.samples, p.prefix_len)
        for i in range(1, p.samples):
            c.fork(gi * p.samples, gi * p.samples + i)
    for s in range(cfg.num_seqs):
        for _ in range(int(p.private_lens[s])):
            c.append_slot(s)
    chunks = _compare_groups(c, o, list(range(cfg.num_seqs)), 512, 8)
    # 1030-token prefix = 64 full blocks shared by all 8 samples -> 2 partitions of 512
    assert len(chunks) == 32 and all(len(m) == 8 and parts == 2 for m, parts in chunks)


# ---------------------------------------------------------------------------
# moving sequences between pools (swap out to a host pool and back)
# ---------------------------------------------------------------------------

def _pools(pa, nb_dev, nb_host, bs, seed):
    g = np.random.default_rng(seed)
    od, oh = g.permutation(nb_dev), g.permutation(nb_host)
    return (pa.BlockAllocator(nb_dev, bs, od), pa.BlockAllocator(nb_host, bs, oh),
            BlockManager(nb_dev, bs, od), BlockManager(nb_host, bs, oh))


@pytest.mark.parametrize("seed", range(4))
def test_moves_between_two_pools(pa, seed):
    g = np.random.default_rng(200 + seed)
    bs = int(g.choice([2, 4, 16]))
    cd, ch, od, oh = _pools(pa, 64, 48, bs, seed)
    where = {}          # seq -> "d" or "h"
    nid = 0
    for step in range(250):
        r = int(g.integers(0, 10))
        on_dev = [s for s, w in where.items() if w == "d"]
        on_host = [s for s, w in where.items() if w == "h"]
        try_ops = []
        if r < 2 or not on_dev:
            n = int(g.integers(0, 4 * bs))
            e1 = e2 = None
            try:
                cd.add(nid, n)
            except pa.PagedAttentionError as e:
                e1 = e.code
            try:
                od.add(nid, n)
            except AllocError as e:
                e2 = e.code
            assert e1 == e2
            if e1 is None:
                where[nid] = "d"
            nid += 1
        elif r < 4:
            p = on_dev[int(g.integers(0, len(on_dev)))]
            cd.fork(p, nid), od.fork(p, nid)
            where[nid] = "d"
            nid += 1
        elif r < 6:
            s = on_dev[int(g.integers(0, len(on_dev)))]
            rc, ro = run_both(pa, cd, od, "append_slot", s)
            assert rc == ro
        elif r < 8:          # swap out a random subset of the device sequences
            k = int(g.integers(1, min(4, len(on_dev)) + 1))
            ids = [int(x) for x in g.choice(on_dev, k, replace=False)]
            err_c = err_o = None
            try:
                pc = cd.move_to(ch, ids)
            except pa.PagedAttentionError as e:
                err_c = e.code
            try:
                po = od.move_to(oh, ids)
            except AllocError as e:
                err_o = e.code
            assert err_c == err_o
            if err_c is None:
                assert [tuple(x) for x in pc.tolist()] == po
                for s in ids:
                    where[s] = "h"
        elif on_host:        # swap back in
            k = int(g.integers(1, min(3, len(on_host)) + 1))
            ids = [int(x) for x in g.choice(on_host, k, replace=False)]
            err_c = err_o = None
            try:
                pc = ch.move_to(cd, ids)
            except pa.PagedAttentionError as e:
                err_c = e.code
            try:
                po = oh.move_to(od, ids)
            except AllocError as e:
                err_o = e.code
            assert err_c == err_o
            if err_c is None:
                assert [tuple(x) for x in pc.tolist()] == po
                for s in ids:
                    where[s] = "d"
        same_state(cd, od)
        same_state(ch, oh)


def test_move_keeps_sharing_inside_the_moved_set(pa):
    cd, ch, od, oh = _pools(pa, 16, 16, 4, 0)
    for m in (cd, od):
        m.add(0, 10)          # 3 blocks
        m.fork(0, 1)
        m.fork(0, 2)
    pc = cd.move_to(ch, [0, 1])       # seq 2 stays: shared blocks copied once
    po = od.move_to(oh, [0, 1])
    assert [tuple(x) for x in pc.tolist()] == po and len(po) == 3
    assert ch.seq_blocks(0) == ch.seq_blocks(1)
    assert all(ch.refcount(b) == 2 for b in ch.seq_blocks(0))
    assert all(cd.refcount(b) == 1 for b in cd.seq_blocks(2))
    same_state(cd, od)
    same_state(ch, oh)


def test_full_pool_swap_out_lets_the_batch_continue(pa):
    """Preemption on the host: the pool runs dry mid-step, the latest sequence is
    swapped out to the host pool, and the step goes through for the others."""
    dev, host = pa.BlockAllocator(6, 4), pa.BlockAllocator(8, 4)
    for s in range(3):
        dev.add(s, 8)                 # 2 full blocks each: pool empty
    with pytest.raises(pa.PagedAttentionError) as e:
        dev.append_slots([0, 1, 2])   # each needs a new block
    assert e.value.code == "NO_FREE_BLOCKS"
    assert dev.stats()["free_blocks"] == 0 and dev.seq_len(0) == 8   # unchanged
    pairs = dev.move_to(host, [2])   # preempt the latest sequence
    assert len(pairs) == 2 and dev.stats()["free_blocks"] == 2
    slots, _ = dev.append_slots([0, 1])
    assert len(slots) == 2 and host.seq_len(2) == 8
    dev.free(0)                      # a sequence finishes: room to swap back in
    back = host.move_to(dev, [2])
    assert len(back) == 2 and dev.seq_len(2) == 8 and host.stats()["num_seqs"] == 0


# ---------------------------------------------------------------------------
# automatic prefix caching
# ---------------------------------------------------------------------------

def _prompt(g, prefixes, bs):
    """A prompt = one of a few shared prefixes + a random tail (token ids)."""
    base = prefixes[int(g.integers(0, len(prefixes)))]
    cut = int(g.integers(0, len(base) + 1))
    tail = g.integers(0, 50, int(g.integers(0, 3 * bs))).tolist()
    return base[:cut] + tail


@pytest.mark.parametrize("seed", range(6))
def test_prefix_cache_random_ops(pa, seed):
    g = np.random.default_rng(300 + seed)
    bs = int(g.choice([2, 4, 8]))
    nb = int(g.integers(12, 40))
    order = g.permutation(nb)
    c, o = pa.BlockAllocator(nb, bs, order), BlockManager(nb, bs, order)
    prefixes = [g.integers(0, 50, int(g.integers(bs, 6 * bs))).tolist() for _ in range(3)]
    live, nid = [], 0
    for step in range(300):
        r = int(g.integers(0, 12))
        if r < 4 or not live:
            toks = _prompt(g, prefixes, bs)
            rc, ro = run_both(pa, c, o, "add_prompt", nid, toks)
            assert rc == ro
            if nid in o.tables:
                live.append(nid)
            nid += 1
        elif r < 6:
            s = live[int(g.integers(0, len(live)))]
            rc, ro = run_both(pa, c, o, "append_slot", s)
            assert rc == ro
        elif r < 7:
            p = live[int(g.integers(0, len(live)))]
            run_both(pa, c, o, "fork", p, nid)
            if nid in o.tables:
                live.append(nid)
            nid += 1
        elif r < 9:
            s = live.pop(int(g.integers(0, len(live))))
            run_both(pa, c, o, "free", s)
        elif r < 10:
            s = live[int(g.integers(0, len(live)))]
            run_both(pa, c, o, "truncate", [s], [int(g.integers(0, o.lens[s] + 1))])
        else:
            n = int(g.integers(0, 2 * bs))
            run_both(pa, c, o, "add", nid, n)
            if nid in o.tables:
                live.append(nid)
            nid += 1
        same_state(c, o)
    assert o.cache_hits > 0 and o.cache_evictions > 0      # both paths were exercised


def test_identical_system_prompts_are_stored_once(pa):
    """[GLOSS] prompt sharing: identical system prompts are stored once and mapped into
    several requests.  Two requests with the same 40-token prompt at block 16: the
    second reuses both full blocks and only its partial last block is new."""
    prompt = list(range(100, 140))
    for m in (pa.BlockAllocator(16, 16), BlockManager(16, 16)):
        first = m.add_prompt(0, prompt)
        second = m.add_prompt(1, prompt + [7, 8])
        t0 = m.seq_blocks(0) if hasattr(m, "seq_blocks") else m.tables[0]
        t1 = m.seq_blocks(1) if hasattr(m, "seq_blocks") else m.tables[1]
        assert (first, second) == (0, 32)
        assert t0[:2] == t1[:2] and t0[2] != t1[2]
        st = m.stats()
        assert st["cached_blocks"] == 2 and st["cache_hits"] == 2 and st["used_blocks"] == 4


def test_released_cached_blocks_are_reused_before_eviction(pa):
    for m in (pa.BlockAllocator(4, 4), BlockManager(4, 4)):
        m.add_prompt(0, list(range(8)))          # 2 cached blocks
        (m.free_seq if isinstance(m, BlockManager) else m.free)(0)
        st = m.stats()
        assert st["evictable_blocks"] == 2 and st["free_blocks"] == 2
        assert m.add_prompt(1, list(range(8)) + [9]) == 8    # hits both, no eviction
        assert m.stats()["cache_evictions"] == 0
        m.add(2, 4)                               # takes the last free block
        with pytest.raises(Exception):
            m.add(3, 4)                           # nothing free, nothing evictable
