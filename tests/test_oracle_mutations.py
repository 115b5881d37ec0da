"""Plant plausible mistakes in the CPU oracle and show that a pin catches each one.

Every mutation is applied to the oracle modules with pytest's monkeypatch (on the
CPU only) and is undone after its test.  A mutation "is caught" when one of the pin
checks from ``test_oracle_pins`` reports a disagreement above its tolerance.
"""
import numpy as np
import pytest

import oracle.allocator as oalloc
import oracle.attention as oatt
import oracle.cache_ops as ocache
from test_oracle_pins import (check_against_loops, check_against_sdpa,
                              check_partition_invariance, check_prefix_sharing)


def _caught_attention():
    gqa = check_against_sdpa(lens=(1, 16, 33, 50), Hq=8, Hkv=2, D=32, bs=8, dtype="bf16",
                             scale=32 ** -0.5)
    return max(check_against_sdpa(), gqa, check_against_loops()) > 1e-6


def test_unmutated_oracle_passes():
    assert not _caught_attention()


def test_catches_table_ignored(monkeypatch):
    orig = oatt.gather_sequence

    def bad(cache, table_row, seq_len, block_size, kv_head):
        return orig(cache, list(range(len(table_row))), seq_len, block_size, kv_head)
    monkeypatch.setattr(oatt, "gather_sequence", bad)
    assert _caught_attention()


def test_catches_last_token_dropped(monkeypatch):
    orig = oatt.gather_sequence

    def bad(cache, table_row, seq_len, block_size, kv_head):
        return orig(cache, table_row, max(seq_len - 1, 1), block_size, kv_head)
    monkeypatch.setattr(oatt, "gather_sequence", bad)
    assert _caught_attention()


def test_catches_missing_scale(monkeypatch):
    orig = oatt.softmax_attention
    monkeypatch.setattr(oatt, "softmax_attention", lambda q, K, V, scale: orig(q, K, V, 1.0))
    assert _caught_attention()


def test_catches_swapped_key_value(monkeypatch):
    orig = oatt.softmax_attention
    monkeypatch.setattr(oatt, "softmax_attention", lambda q, K, V, scale: orig(q, V, K, scale))
    assert _caught_attention()


def test_catches_sign_error(monkeypatch):
    orig = oatt.softmax_attention
    monkeypatch.setattr(oatt, "softmax_attention", lambda q, K, V, scale: orig(-q, K, V, scale))
    assert _caught_attention()


def test_catches_interleaved_gqa_grouping(monkeypatch):
    def bad(q, k_cache, v_cache, block_tables, seq_lens, scale, block_size, num_kv_heads,
            dtype, seqs=None, heads=None):
        S, Hq, D = q.shape
        out = np.zeros((S, Hq, D))
        for s in range(S):
            for h in range(Hq):
                g = h % num_kv_heads          # wrong: interleaved instead of consecutive
                K = oatt.to_f64(oatt.gather_sequence(k_cache, block_tables[s], int(seq_lens[s]),
                                                     block_size, g), dtype)
                V = oatt.to_f64(oatt.gather_sequence(v_cache, block_tables[s], int(seq_lens[s]),
                                                     block_size, g), dtype)
                out[s, h] = oatt.softmax_attention(oatt.to_f64(q[s, h], dtype), K, V, scale)
        return out
    monkeypatch.setattr(oatt, "paged_decode_attention", bad)
    gqa = check_against_sdpa(lens=(1, 16, 33, 50), Hq=8, Hkv=2, D=32, bs=8, dtype="bf16",
                             scale=32 ** -0.5)
    assert gqa > 1e-6


def test_catches_unweighted_merge(monkeypatch):
    def bad(states):
        return sum(l * o for _, l, o in states) / sum(l for _, l, _ in states)
    monkeypatch.setattr(oatt, "merge_partitions", bad)
    assert check_partition_invariance() > 1e-6


def test_catches_slot_offset_error(monkeypatch):
    def bad(key, value, k_cache, v_cache, slot_mapping, block_size):
        for t, slot in enumerate(np.asarray(slot_mapping)):
            if slot < 0:
                continue
            blk, off = divmod(int(slot), block_size)
            k_cache[blk, :, (off + 1) % block_size, :] = key[t]
            v_cache[blk, :, (off + 1) % block_size, :] = value[t]
    monkeypatch.setattr(ocache, "reshape_and_cache", bad)
    assert check_against_sdpa(reshape=bad) > 1e-6


def test_catches_missing_copy_on_write(monkeypatch):
    class NoCow(oalloc.BlockManager):
        def append_slot(self, seq_id):
            table, n = self.tables[seq_id], self.lens[seq_id]
            off = n % self.block_size
            if off == 0:
                table.append(self._pop())
            self.lens[seq_id] = n + 1
            return table[-1] * self.block_size + off, -1, -1
    assert check_prefix_sharing(bm_cls=NoCow) > 0.0


# ---- block manager: refcount and table bookkeeping mistakes ------------------------

def _caught_allocator(bm_cls) -> bool:
    """Random add/fork/append/free/truncate sequences under the allocator invariants
    (counts = table entries, free and used partition the pool, ceil(L/bs) blocks)."""
    from test_oracle_pins import _invariants, random_ops
    g = np.random.default_rng(11)
    try:
        for _ in range(5):
            random_ops(bm_cls(24, 4, g.permutation(24)), g, 200, _invariants)
    except AssertionError:
        return True
    return False


def test_unmutated_allocator_passes():
    assert not _caught_allocator(oalloc.BlockManager)


def test_catches_fork_without_reference_counts():
    class Bad(oalloc.BlockManager):
        def fork(self, parent, child):
            if parent not in self.tables:
                raise oalloc.AllocError(oalloc.UNKNOWN_SEQ, str(parent))
            self.tables[child] = list(self.tables[parent])
            self.lens[child] = self.lens[parent]
    assert _caught_allocator(Bad)


def test_catches_free_that_leaks_blocks():
    class Bad(oalloc.BlockManager):
        def free_seq(self, seq_id):
            self.tables.pop(seq_id)
            del self.lens[seq_id]
    assert _caught_allocator(Bad)


def test_catches_block_taken_one_token_early():
    class Bad(oalloc.BlockManager):
        def append_slot(self, seq_id):
            table, n = self.tables[seq_id], self.lens[seq_id]
            if n % self.block_size == self.block_size - 1 and self._available():
                table.append(self._pop())          # the last slot of a block is never used
                self.lens[seq_id] = n + 1
                return table[-1] * self.block_size, -1, -1
            return super().append_slot(seq_id)
    assert _caught_allocator(Bad)


def test_catches_copy_on_write_that_keeps_the_shared_reference():
    class Bad(oalloc.BlockManager):
        def _release(self, b):
            if self.ref[b] > 1:
                return                             # the writer's reference is never dropped
            super()._release(b)
    assert _caught_allocator(Bad)


# ---- widening of stored values -------------------------------------------------------

def _widening_caught(bad) -> bool:
    from test_oracle_pins import check_widening
    return check_widening(fn=bad) > 0


def test_unmutated_widening_passes():
    from oracle.numerics import to_f64
    assert not _widening_caught(to_f64)


def test_catches_bf16_shifted_by_15():
    from oracle.numerics import to_f64

    def bad(x, dtype):
        if dtype == "bf16":
            bits = np.asarray(x, np.uint16).astype(np.uint32) << np.uint32(15)
            return bits.view(np.float32).astype(np.float64)
        return to_f64(x, dtype)
    assert _widening_caught(bad)


def test_catches_bf16_bits_read_as_f16():
    from oracle.numerics import to_f64

    def bad(x, dtype):
        if dtype == "bf16":
            return np.asarray(x, np.uint16).view(np.float16).astype(np.float64)
        return to_f64(x, dtype)
    assert _widening_caught(bad)


def test_catches_f16_through_bf16_rounding():
    from oracle.numerics import to_f64

    def bad(x, dtype):
        if dtype == "f16":       # an extra trip through a 7-bit significand
            f = np.asarray(x, np.float16).astype(np.float32).view(np.uint32)
            return (f & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)
        return to_f64(x, dtype)
    assert _widening_caught(bad)


def test_catches_subnormals_flushed_to_zero():
    from oracle.numerics import to_f64

    def bad(x, dtype):
        v = to_f64(x, dtype)
        tiny = {"bf16": 2.0 ** -126, "f16": 2.0 ** -14, "f32": 2.0 ** -126}[dtype]
        return np.where(np.abs(v) < tiny, 0.0, v)
    assert _widening_caught(bad)


def test_catches_sign_dropped():
    from oracle.numerics import to_f64
    assert _widening_caught(lambda x, dtype: np.abs(to_f64(x, dtype)))


# ---- moves between pools ---------------------------------------------------------------

def _moves_caught(bm_cls) -> bool:
    from test_oracle_pins import check_moves
    try:
        check_moves(bm_cls, trials=4, n_ops=200)
    except AssertionError:
        return True
    return False


def _hand_move_caught(bm_cls) -> bool:
    import test_oracle_pins as pins
    orig = pins.BlockManager
    pins.BlockManager = bm_cls
    try:
        pins.test_move_hand_case_shared_block_becomes_private()
    except (AssertionError, oalloc.AllocError):
        return True
    finally:
        pins.BlockManager = orig
    return False


def test_unmutated_moves_pass():
    assert not _moves_caught(oalloc.BlockManager)
    assert not _hand_move_caught(oalloc.BlockManager)


def test_catches_move_without_release():
    class Bad(oalloc.BlockManager):
        def move_to(self, other, seq_ids):
            keep = list(self.ref)
            pairs = super().move_to(other, seq_ids)
            for b in range(self.num_blocks):       # this pool's references never drop
                if keep[b] and not self.ref[b] and b in self.free:
                    self.free.remove(b)
                self.ref[b] = keep[b]
            return pairs
    assert _moves_caught(Bad)


def test_catches_move_that_loses_sharing():
    class Bad(oalloc.BlockManager):
        def move_to(self, other, seq_ids):
            pairs = []
            for s in list(seq_ids):                 # one private copy per reference
                pairs += super().move_to(other, [s])
            return pairs
    assert _hand_move_caught(Bad)


def test_catches_move_pairs_in_block_order():
    class Bad(oalloc.BlockManager):
        def move_to(self, other, seq_ids):
            ids = list(seq_ids)
            distinct = sorted({b for s in ids for b in self.tables[s]})
            mapping = {b: other._pop() for b in distinct}
            for nb in mapping.values():
                other.ref[nb] = 0
            for s in ids:
                table = self.tables.pop(s)
                other.tables[s] = [mapping[b] for b in table]
                other.lens[s] = self.lens.pop(s)
                for b in table:
                    other.ref[mapping[b]] += 1
                    self._release(b)
            return [(b, mapping[b]) for b in distinct]
    assert _moves_caught(Bad) or _hand_move_caught(Bad)


def test_catches_move_that_copies_nothing():
    class Bad(oalloc.BlockManager):
        def move_to(self, other, seq_ids):
            pairs = super().move_to(other, seq_ids)
            return [(a, b) for a, b in pairs][:-1]  # the last distinct block is not copied
    assert _moves_caught(Bad)


# ---- prefix groups -------------------------------------------------------------------

def _groups_caught(bm_cls) -> bool:
    from test_oracle_pins import check_prefix_groups
    return check_prefix_groups(bm_cls) > 0


def test_unmutated_prefix_groups_pass():
    assert not _groups_caught(oalloc.BlockManager)


def test_catches_common_prefix_of_first_two_members_only():
    class Bad(oalloc.BlockManager):
        def prefix_groups(self, seq_ids, partition_size, max_members):
            ids = list(seq_ids)
            by_first, order = {}, []
            for pos, s in enumerate(ids):
                t = self.tables[s]
                if t:
                    if t[0] not in by_first:
                        by_first[t[0]] = []
                        order.append(t[0])
                    by_first[t[0]].append(pos)
            parts_of, chunks = [0] * len(ids), []
            for first in order:
                members = by_first[first]
                if len(members) < 2:
                    continue
                a, b = self.tables[ids[members[0]]], self.tables[ids[members[1]]]
                common = 0
                while common < min(len(a), len(b)) and a[common] == b[common]:
                    common += 1
                parts = common * self.block_size // partition_size
                if parts:
                    for m in members:
                        parts_of[m] = parts
                    for i in range(0, len(members), max_members):
                        chunks.append((members[i:i + max_members], parts))
            return parts_of, chunks
    assert _groups_caught(Bad)


def test_catches_partial_partition_rounded_up():
    class Bad(oalloc.BlockManager):
        def prefix_groups(self, seq_ids, partition_size, max_members):
            # a common prefix that ends inside a partition claims that partition too
            pp, chunks = super().prefix_groups(seq_ids, 1, max_members)
            ceil = lambda p: -(-p // partition_size)
            return [ceil(p) for p in pp], [(m, ceil(p)) for m, p in chunks]
    assert _groups_caught(Bad)


def test_catches_chunks_not_split():
    class Bad(oalloc.BlockManager):
        def prefix_groups(self, seq_ids, partition_size, max_members):
            return super().prefix_groups(seq_ids, partition_size, 1 << 30)
    assert _groups_caught(Bad)


def test_catches_singletons_grouped():
    class Bad(oalloc.BlockManager):
        def prefix_groups(self, seq_ids, partition_size, max_members):
            pp, chunks = super().prefix_groups(seq_ids, partition_size, max_members)
            ids = list(seq_ids)
            for pos, s in enumerate(ids):
                t = self.tables[s]
                parts = len(t) * self.block_size // partition_size
                if pp[pos] == 0 and parts and not any(
                        self.tables[o] and self.tables[o][0] == t[0] for o in ids if o != s):
                    pp[pos] = parts
                    chunks.append(([pos], parts))
            return pp, chunks
    assert _groups_caught(Bad)
