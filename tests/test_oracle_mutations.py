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
