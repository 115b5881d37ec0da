"""Block manager model in plain Python (oracle; test infrastructure only).

Sources (page title, section):
  [BLOG] "How PagedAttention Powers vLLM's KV Cache":
    "PagedAttention: paging, borrowed from the operating system" - when a sequence
      needs room it takes a free physical block from a shared pool and appends it to
      its block table; a finished sequence's blocks go back to the pool; nothing is
      reserved up front.
    "The bonus contiguous storage can't give you: sharing" - block tables of several
      sequences may point at one physical block, which carries a reference count;
      before a sequence writes past the shared region it copies that block
      (copy-on-write); parallel sampling branches share the prompt's blocks.
  [LAB] "PagedAttention" explainer:
    "Add pages as the request grows" / "Block allocation" - a new block only when
      the current one is full, so only the last block has unused slots.
    "Share matching prefixes" / "Shared blocks and copy-on-write" - writing into a
      shared block needs a private copy; appending after a full shared block only
      needs a new block.

Readings where the pages are silent (the C-ABI allocator follows the same ones):
  * free pool order: a LIFO stack whose successive pops return free_order[0],
    free_order[1], ...; a block whose count drops to zero is pushed on top;
  * a finished sequence releases its blocks in logical order; truncating a sequence
    (dropping its last tokens, e.g. a rejected draft token) releases the blocks past
    the new length the same way and never copies;
  * copy-on-write fires when the block the next token goes into has count > 1;
    the writer gets a fresh block, the shared block's count drops by one;
  * a failing call leaves the state unchanged; a batch of appends is all or nothing;
  * block-table rows are padded with -1.

Automatic prefix caching ([BLOG] "The bonus contiguous storage can't give you:
sharing": prefix caching is built on top of copy-on-write; the mechanism is not
given, so this is the reading taken):
  * a prompt admitted with its token ids reuses a cached block for every leading
    full block whose tokens - and whose whole prefix - match an earlier prompt's;
  * the cache key of a full block is (cache id of the previous block, its tokens);
    a block registered in the cache gets a fresh cache id, so a key can only match
    when the entire prefix matches (no hashing, no collisions);
  * the first block that misses, and every block after it, is a fresh block that is
    registered (the caller writes its K/V before anyone attends over it); the last
    partial block is fresh and not registered;
  * a cached block whose count drops to zero becomes evictable (least recently
    released first) instead of free; a pop takes a free block if there is one, else
    evicts the least recently released cached block;
  * a cached block's content is immutable: a write into it (an append after the
    sequence was truncated into it) copies it when shared and uncaches it when not.
"""
from __future__ import annotations

import copy


class AllocError(Exception):
    def __init__(self, code: str, msg: str = ""):
        super().__init__(f"{code}: {msg}")
        self.code = code


NO_FREE_BLOCKS = "NO_FREE_BLOCKS"
UNKNOWN_SEQ = "UNKNOWN_SEQ"
SEQ_EXISTS = "SEQ_EXISTS"
INVALID_ARG = "INVALID_ARG"


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise AllocError(INVALID_ARG, "pool and block size must be positive")
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise AllocError(INVALID_ARG, "free_order must be a permutation of the pool")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = order[::-1]          # top of the stack is the end of the list
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.cow_copies = 0
        self.blocks_allocated = 0
        # prefix cache
        self.evictable: list[int] = []        # least recently released first
        self.cache: dict = {}                 # (parent cache id, tokens) -> block
        self.cache_of: dict = {}              # block -> (key, cache id)
        self.next_cache_id = 1
        self.cache_hits = 0
        self.cache_evictions = 0

    # -- helpers -------------------------------------------------------------
    def _available(self) -> int:
        return len(self.free) + len(self.evictable)

    def _pop(self) -> int:
        if self.free:
            b = self.free.pop()
        else:
            b = self.evictable.pop(0)
            key, _ = self.cache_of.pop(b)
            del self.cache[key]
            self.cache_evictions += 1
        self.ref[b] = 1
        self.blocks_allocated += 1
        return b

    def _release(self, b: int) -> None:
        """One reference to b goes away."""
        self.ref[b] -= 1
        if self.ref[b] == 0:
            (self.evictable if b in self.cache_of else self.free).append(b)

    def _uncache(self, b: int) -> None:
        key, _ = self.cache_of.pop(b)
        del self.cache[key]

    def _blocks_for(self, n_tokens: int) -> int:
        return (n_tokens + self.block_size - 1) // self.block_size

    # -- operations ----------------------------------------------------------
    def add(self, seq_id: int, n_tokens: int) -> None:
        """A new sequence with n_tokens cached tokens: ceil(n/bs) fresh blocks."""
        if seq_id in self.tables:
            raise AllocError(SEQ_EXISTS, str(seq_id))
        if n_tokens < 0:
            raise AllocError(INVALID_ARG, "negative length")
        need = self._blocks_for(n_tokens)
        if need > self._available():
            raise AllocError(NO_FREE_BLOCKS, f"need {need}, have {self._available()}")
        self.tables[seq_id] = [self._pop() for _ in range(need)]
        self.lens[seq_id] = n_tokens

    def add_prompt(self, seq_id: int, tokens) -> int:
        """Admit a sequence by its prompt token ids, reusing cached full blocks.
        Returns the number of leading tokens whose blocks came from the cache."""
        if seq_id in self.tables:
            raise AllocError(SEQ_EXISTS, str(seq_id))
        tokens = [int(t) for t in tokens]
        bs = self.block_size
        full = len(tokens) // bs
        keys, hits, parent = [], [], 0
        for j in range(full):
            key = (parent, tuple(tokens[j * bs:(j + 1) * bs]))
            keys.append(key)
            if parent is not None and key in self.cache:
                b = self.cache[key]
                hits.append(b)
                parent = self.cache_of[b][1]
            else:
                parent = None             # the chain is broken: no later block can match
        fresh = len(keys) - len(hits) + (1 if len(tokens) % bs else 0)
        claimable = sum(1 for b in hits if self.ref[b] == 0)
        if fresh > self._available() - claimable:
            raise AllocError(NO_FREE_BLOCKS, f"need {fresh}")
        table = []
        for b in hits:                    # claim the cached blocks first
            if self.ref[b] == 0:
                self.evictable.remove(b)
            self.ref[b] += 1
            table.append(b)
        self.cache_hits += len(hits)
        parent = self.cache_of[hits[-1]][1] if hits else 0
        for key in keys[len(hits):]:      # then fresh, registered blocks
            b = self._pop()
            key = (parent, key[1])
            cid = self.next_cache_id
            self.next_cache_id += 1
            self.cache[key] = b
            self.cache_of[b] = (key, cid)
            parent = cid
            table.append(b)
        if len(tokens) % bs:
            table.append(self._pop())     # the partial last block is never cached
        self.tables[seq_id] = table
        self.lens[seq_id] = len(tokens)
        return len(hits) * bs

    def fork(self, parent: int, child: int) -> None:
        """child shares every block of parent (each count + 1)."""
        if parent not in self.tables:
            raise AllocError(UNKNOWN_SEQ, str(parent))
        if child in self.tables:
            raise AllocError(SEQ_EXISTS, str(child))
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def append_slot(self, seq_id: int):
        """Room for one more token: returns (slot, cow_src, cow_dst), -1 = no copy."""
        if seq_id not in self.tables:
            raise AllocError(UNKNOWN_SEQ, str(seq_id))
        table, n = self.tables[seq_id], self.lens[seq_id]
        off = n % self.block_size
        src = dst = -1
        if off == 0:
            if not self._available():
                raise AllocError(NO_FREE_BLOCKS, "append")
            table.append(self._pop())
        elif self.ref[table[-1]] > 1:
            if not self._available():
                raise AllocError(NO_FREE_BLOCKS, "copy-on-write")
            src = table[-1]
            dst = self._pop()
            self._release(src)
            table[-1] = dst
            self.cow_copies += 1
        elif table[-1] in self.cache_of:
            self._uncache(table[-1])     # sole owner writes into a cached block
        self.lens[seq_id] = n + 1
        return table[-1] * self.block_size + off, src, dst

    def append_slots(self, seq_ids):
        """One append per listed sequence, in order; all or nothing."""
        saved = copy.deepcopy(self.__dict__)
        try:
            return [self.append_slot(s) for s in seq_ids]
        except AllocError:
            self.__dict__.clear()
            self.__dict__.update(saved)
            raise

    def truncate(self, seq_ids, new_lens) -> None:
        """Shorten each listed sequence to its new length (<= current); blocks past
        ceil(new_len / bs) are released in logical order.  All or nothing."""
        pairs = list(zip(seq_ids, new_lens))
        for s, n in pairs:
            if s not in self.tables:
                raise AllocError(UNKNOWN_SEQ, str(s))
        if len({s for s, _ in pairs}) != len(pairs):
            raise AllocError(INVALID_ARG, "sequence ids repeat")
        for s, n in pairs:
            if n < 0 or n > self.lens[s]:
                raise AllocError(INVALID_ARG, f"cannot truncate {s} to {n}")
        for s, n in pairs:
            keep = self._blocks_for(n)
            table = self.tables[s]
            for b in table[keep:]:
                self._release(b)
            del table[keep:]
            self.lens[s] = n

    def move_to(self, other: "BlockManager", seq_ids):
        """Move sequences into another pool (e.g. device pool -> host swap pool).

        Every distinct block the moved sequences reference gets one fresh block in
        ``other`` (taken in order of first appearance: sequence order, then logical
        order), so sharing inside the moved set is kept; references to blocks shared
        with sequences that stay behind become private copies.  In this pool each
        moved reference is dropped in the same order (a block reaching zero goes
        back on the free stack).  Returns the (this_block, other_block) pairs to copy.
        All or nothing; ids must be distinct.
        """
        ids = list(seq_ids)
        if len(set(ids)) != len(ids):
            raise AllocError(INVALID_ARG, "sequence ids repeat")
        for s in ids:
            if s not in self.tables:
                raise AllocError(UNKNOWN_SEQ, str(s))
            if s in other.tables:
                raise AllocError(SEQ_EXISTS, str(s))
        if other.block_size != self.block_size:
            raise AllocError(INVALID_ARG, "block sizes differ")
        distinct = []
        for s in ids:
            for b in self.tables[s]:
                if b not in distinct:
                    distinct.append(b)
        if len(distinct) > other._available():
            raise AllocError(NO_FREE_BLOCKS, f"need {len(distinct)}, have {other._available()}")
        mapping = {b: other._pop() for b in distinct}
        for nb in mapping.values():
            other.ref[nb] = 0                # counted below, one per table entry
        for s in ids:
            table = self.tables.pop(s)
            other.tables[s] = [mapping[b] for b in table]
            other.lens[s] = self.lens.pop(s)
            for b in table:
                other.ref[mapping[b]] += 1
                self._release(b)
        return [(b, mapping[b]) for b in distinct]

    def free_seq(self, seq_id: int) -> None:
        if seq_id not in self.tables:
            raise AllocError(UNKNOWN_SEQ, str(seq_id))
        for b in self.tables.pop(seq_id):
            self._release(b)
        del self.lens[seq_id]

    # -- sharing structure ---------------------------------------------------
    def prefix_groups(self, seq_ids, partition_size: int, max_members: int):
        """Batch positions whose block tables begin with the same physical blocks.

        Sequences are grouped by their first block (first appearance order); a group
        needs at least two members and a common table prefix (in blocks) covering at
        least one whole partition.  Members are split, in order, into chunks of at most
        ``max_members``.  Returns (prefix_parts per position, [(members, parts)] chunks)
        where parts = floor(common_prefix_blocks * block_size / partition_size).
        """
        ids = list(seq_ids)
        by_first, order = {}, []
        for pos, s in enumerate(ids):
            t = self.tables[s]
            if not t:
                continue
            if t[0] not in by_first:
                by_first[t[0]] = []
                order.append(t[0])
            by_first[t[0]].append(pos)
        prefix_parts = [0] * len(ids)
        chunks = []
        for first in order:
            members = by_first[first]
            if len(members) < 2:
                continue
            tabs = [self.tables[ids[m]] for m in members]
            common = 0
            while all(common < len(t) for t in tabs) and \
                    all(t[common] == tabs[0][common] for t in tabs):
                common += 1
            parts = common * self.block_size // partition_size
            if parts == 0:
                continue
            for m in members:
                prefix_parts[m] = parts
            for i in range(0, len(members), max_members):
                chunks.append((members[i:i + max_members], parts))
        return prefix_parts, chunks

    # -- views ---------------------------------------------------------------
    def block_tables(self, seq_ids, max_blocks: int):
        rows, lens = [], []
        for s in seq_ids:
            t = self.tables[s]
            if len(t) > max_blocks:
                raise AllocError(INVALID_ARG, "table wider than max_blocks")
            rows.append(t + [-1] * (max_blocks - len(t)))
            lens.append(self.lens[s])
        return rows, lens

    def free_list(self):
        """Free blocks in the order the next pops return them."""
        return self.free[::-1]

    def stats(self) -> dict:
        bs = self.block_size
        used = self.num_blocks - len(self.free) - len(self.evictable)
        return dict(
            num_blocks=self.num_blocks, block_size=bs, free_blocks=len(self.free),
            used_blocks=used, shared_blocks=sum(1 for r in self.ref if r > 1),
            total_refs=sum(self.ref), num_seqs=len(self.tables),
            logical_tokens=sum(self.lens.values()), allocated_slots=used * bs,
            tail_waste_slots=sum(len(t) * bs - self.lens[s] for s, t in self.tables.items()),
            cow_copies=self.cow_copies, blocks_allocated=self.blocks_allocated,
            cached_blocks=len(self.cache_of), evictable_blocks=len(self.evictable),
            cache_hits=self.cache_hits, cache_evictions=self.cache_evictions)
