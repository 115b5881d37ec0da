// Host block manager for the paged KV cache (C ABI in include/pa.h).
//
// Behaviour from "How PagedAttention Powers vLLM's KV Cache" (hassanahmed.net),
// sections "PagedAttention: paging, borrowed from the operating system" (blocks
// from a shared free pool, appended on demand, returned when a sequence ends) and
// "The bonus contiguous storage can't give you: sharing" (reference counts,
// copy-on-write, parallel samples sharing a prompt), and from the "PagedAttention"
// attention-lab explainer (divagr.pages.dev), sections "Add pages as the request
// grows" and "Share matching prefixes" (a new block only when the last is full;
// after a full shared block only a new block, no copy).
//
// Pool order (not fixed by the pages): a LIFO stack; pops return free_order[0],
// free_order[1], ...; a released block goes on top; a freed sequence releases its
// blocks in logical order.  Every failing call leaves the state unchanged.
//
// Automatic prefix caching (built on the sharing machinery, as the same blog's
// sharing section says): full prompt blocks are registered under the exact key
// (cache id of the previous block, the block's token ids); a released cached block
// becomes evictable (least recently released first) instead of free; a pop takes a
// free block first, then evicts; a write into a cached block copies it when shared
// and uncaches it when not.
#include <cstdint>
#include <cstring>
#include <iterator>
#include <list>
#include <map>
#include <new>
#include <unordered_map>
#include <utility>
#include <vector>

#include "../../include/pa.h"

namespace {

struct Seq {
  std::vector<int32_t> blocks;  // logical order
  int64_t len = 0;
  // scratch of batched calls, valid while mark equals the allocator's epoch
  uint64_t mark = 0;
  int64_t sim_len = 0;
  int32_t sim_last = -1;
};

}  // namespace

struct pa_alloc {
  using CacheKey = std::pair<int64_t, std::vector<int32_t>>;  // (parent cache id, tokens)

  int64_t num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_stack;  // back() is the top
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Seq> seqs;
  int64_t cow_copies = 0;
  int64_t blocks_allocated = 0;
  int64_t shared_blocks = 0;  // maintained incrementally: count of ref > 1
  // prefix cache
  std::list<int32_t> evictable;  // cached blocks with ref 0, least recently released first
  std::vector<std::list<int32_t>::iterator> evict_pos;
  std::vector<int64_t> cache_id;  // 0 = not cached
  std::vector<CacheKey> cache_key;
  std::map<CacheKey, int32_t> cache;
  int64_t next_cache_id = 1, cache_hits = 0, cache_evictions = 0;
  // scratch of batched calls: each call takes a new epoch, so per-sequence and
  // per-block marks from earlier calls read as unset without clearing anything
  uint64_t epoch = 0;
  std::vector<uint64_t> block_mark;
  std::vector<int32_t> block_val;
  std::vector<Seq*> batch;

  // Looks every id up once; false if one is unknown.
  bool resolve(const int64_t* ids, int n) {
    batch.resize(static_cast<size_t>(n));
    for (int i = 0; i < n; ++i) {
      auto it = seqs.find(ids[i]);
      if (it == seqs.end()) return false;
      batch[static_cast<size_t>(i)] = &it->second;
    }
    return true;
  }

  int64_t available() const {
    return static_cast<int64_t>(free_stack.size() + evictable.size());
  }
  void uncache(int32_t b) {
    cache.erase(cache_key[b]);
    cache_key[b] = CacheKey();
    cache_id[b] = 0;
  }
  int32_t pop() {
    int32_t b;
    if (!free_stack.empty()) {
      b = free_stack.back();
      free_stack.pop_back();
    } else {
      b = evictable.front();
      evictable.pop_front();
      uncache(b);
      ++cache_evictions;
    }
    ref[b] = 1;
    ++blocks_allocated;
    return b;
  }
  void inc(int32_t b) {
    if (++ref[b] == 2) ++shared_blocks;
  }
  void dec(int32_t b) {
    if (ref[b]-- == 2) --shared_blocks;
    if (ref[b] == 0) {
      if (cache_id[b]) {
        evictable.push_back(b);
        evict_pos[b] = std::prev(evictable.end());
      } else {
        free_stack.push_back(b);
      }
    }
  }
};

namespace {

inline int64_t blocks_for(int64_t n, int bs) { return (n + bs - 1) / bs; }

// Length of the common prefix of two block lists of at least n entries: whole
// 16-entry chunks by memcmp, then entry by entry inside the first differing chunk.
inline size_t common_prefix(const int32_t* x, const int32_t* y, size_t n) {
  constexpr size_t kChunk = 16;
  size_t c = 0;
  while (c + kChunk <= n && std::memcmp(x + c, y + c, kChunk * sizeof(int32_t)) == 0) c += kChunk;
  while (c < n && x[c] == y[c]) ++c;
  return c;
}

// Blocks one append to `s` takes from the pool, given the (possibly simulated)
// reference count of its last block.
inline bool append_needs_block(const Seq& s, int bs, int32_t last_ref) {
  if (s.len % bs == 0) return true;
  return last_ref > 1;
}

}  // namespace

extern "C" {

int pa_alloc_create(int64_t num_blocks, int block_size, const int32_t* free_order,
                    pa_alloc_t** out) {
  if (!out || num_blocks <= 0 || block_size <= 0 || num_blocks > INT32_MAX)
    return PA_ERR_INVALID_ARG;
  *out = nullptr;
  pa_alloc* a = new (std::nothrow) pa_alloc();
  if (!a) return PA_ERR_INVALID_ARG;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->ref.assign(static_cast<size_t>(num_blocks), 0);
  a->block_mark.assign(static_cast<size_t>(num_blocks), 0);
  a->block_val.assign(static_cast<size_t>(num_blocks), 0);
  a->evict_pos.assign(static_cast<size_t>(num_blocks), a->evictable.end());
  a->cache_id.assign(static_cast<size_t>(num_blocks), 0);
  a->cache_key.assign(static_cast<size_t>(num_blocks), pa_alloc::CacheKey());
  a->free_stack.resize(static_cast<size_t>(num_blocks));
  if (free_order) {
    std::vector<uint8_t> seen(static_cast<size_t>(num_blocks), 0);
    for (int64_t i = 0; i < num_blocks; ++i) {
      int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return PA_ERR_INVALID_ARG;
      }
      seen[b] = 1;
      a->free_stack[static_cast<size_t>(num_blocks - 1 - i)] = b;
    }
  } else {
    for (int64_t i = 0; i < num_blocks; ++i)
      a->free_stack[static_cast<size_t>(num_blocks - 1 - i)] = static_cast<int32_t>(i);
  }
  *out = a;
  return PA_OK;
}

int pa_alloc_destroy(pa_alloc_t* a) {
  delete a;
  return PA_OK;
}

int pa_seq_add(pa_alloc_t* a, int64_t seq_id, int64_t num_tokens) {
  if (!a || num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (a->seqs.count(seq_id)) return PA_ERR_SEQ_EXISTS;
  int64_t need = blocks_for(num_tokens, a->block_size);
  if (need > a->available()) return PA_ERR_NO_FREE_BLOCKS;
  Seq s;
  s.blocks.reserve(static_cast<size_t>(need + 1));
  for (int64_t i = 0; i < need; ++i) s.blocks.push_back(a->pop());
  s.len = num_tokens;
  a->seqs.emplace(seq_id, std::move(s));
  return PA_OK;
}

int pa_seq_add_prompt(pa_alloc_t* a, int64_t seq_id, const int32_t* token_ids, int64_t n,
                      int64_t* cached_tokens) {
  if (!a || n < 0 || (n > 0 && !token_ids) || !cached_tokens) return PA_ERR_INVALID_ARG;
  if (a->seqs.count(seq_id)) return PA_ERR_SEQ_EXISTS;
  const int bs = a->block_size;
  const int64_t full = n / bs;
  // plan: the leading full blocks found in the cache, in order
  std::vector<int32_t> hits;
  int64_t parent = 0;
  for (int64_t j = 0; j < full; ++j) {
    pa_alloc::CacheKey key(parent, std::vector<int32_t>(token_ids + j * bs, token_ids + (j + 1) * bs));
    auto it = a->cache.find(key);
    if (it == a->cache.end()) break;  // the chain is broken: nothing later can match
    hits.push_back(it->second);
    parent = a->cache_id[it->second];
  }
  const int64_t fresh = full - static_cast<int64_t>(hits.size()) + (n % bs ? 1 : 0);
  int64_t claimable = 0;
  for (int32_t b : hits) claimable += a->ref[b] == 0;
  if (fresh > a->available() - claimable) return PA_ERR_NO_FREE_BLOCKS;
  Seq s;
  s.blocks.reserve(static_cast<size_t>(full + 2));
  for (int32_t b : hits) {  // claim the cached blocks first
    if (a->ref[b] == 0) {
      a->evictable.erase(a->evict_pos[b]);
      a->evict_pos[b] = a->evictable.end();
      a->ref[b] = 1;
    } else {
      a->inc(b);
    }
    s.blocks.push_back(b);
  }
  a->cache_hits += static_cast<int64_t>(hits.size());
  for (int64_t j = static_cast<int64_t>(hits.size()); j < full; ++j) {  // fresh, registered
    const int32_t b = a->pop();
    pa_alloc::CacheKey key(parent, std::vector<int32_t>(token_ids + j * bs, token_ids + (j + 1) * bs));
    const int64_t cid = a->next_cache_id++;
    a->cache.emplace(key, b);
    a->cache_key[b] = std::move(key);
    a->cache_id[b] = cid;
    parent = cid;
    s.blocks.push_back(b);
  }
  if (n % bs) s.blocks.push_back(a->pop());  // the partial last block is never cached
  s.len = n;
  a->seqs.emplace(seq_id, std::move(s));
  *cached_tokens = static_cast<int64_t>(hits.size()) * bs;
  return PA_OK;
}

int pa_seq_fork(pa_alloc_t* a, int64_t parent, int64_t child) {
  if (!a) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end()) return PA_ERR_UNKNOWN_SEQ;
  if (a->seqs.count(child)) return PA_ERR_SEQ_EXISTS;
  Seq c = it->second;  // copy of the table and length
  for (int32_t b : c.blocks) a->inc(b);
  a->seqs.emplace(child, std::move(c));
  return PA_OK;
}

static int64_t append_one(pa_alloc* a, Seq& s, int32_t* src, int32_t* dst) {
  const int bs = a->block_size;
  const int64_t off = s.len % bs;
  *src = -1;
  *dst = -1;
  if (off == 0) {
    s.blocks.push_back(a->pop());
  } else {
    int32_t last = s.blocks.back();
    if (a->ref[last] > 1) {
      int32_t fresh = a->pop();
      a->dec(last);  // stays > 0: it was shared
      s.blocks.back() = fresh;
      *src = last;
      *dst = fresh;
      ++a->cow_copies;
    } else if (a->cache_id[last]) {
      a->uncache(last);  // the sole owner writes into a cached block
    }
  }
  ++s.len;
  return static_cast<int64_t>(s.blocks.back()) * bs + off;
}

int pa_seq_append_slot(pa_alloc_t* a, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                       int32_t* cow_dst) {
  if (!a || !slot || !cow_src || !cow_dst) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_UNKNOWN_SEQ;
  Seq& s = it->second;
  bool need = append_needs_block(s, a->block_size, s.blocks.empty() ? 0 : a->ref[s.blocks.back()]);
  if (need && a->available() == 0) return PA_ERR_NO_FREE_BLOCKS;
  *slot = append_one(a, s, cow_src, cow_dst);
  return PA_OK;
}

int pa_seq_append_slots(pa_alloc_t* a, const int64_t* seq_ids, int n, int64_t* slots,
                        int32_t* cow_pairs, int* num_cow) {
  if (!a || n < 0 || (n > 0 && (!seq_ids || !slots || !cow_pairs)) || !num_cow)
    return PA_ERR_INVALID_ARG;
  // Dry run: count the blocks the batch takes, simulating lengths and the
  // reference counts that earlier copies in the batch drop (block_val).
  if (!a->resolve(seq_ids, n)) return PA_ERR_UNKNOWN_SEQ;
  const uint64_t ep = ++a->epoch;
  int64_t need = 0;
  const int bs = a->block_size;
  for (int i = 0; i < n; ++i) {
    Seq& s = *a->batch[static_cast<size_t>(i)];
    if (s.mark != ep) {
      s.mark = ep;
      s.sim_len = s.len;
      s.sim_last = s.blocks.empty() ? -1 : s.blocks.back();
    }
    if (s.sim_len % bs == 0) {
      ++need;
      s.sim_last = -1;  // a fresh, private block
    } else if (s.sim_last >= 0) {
      const int32_t last = s.sim_last;
      const int32_t drop = a->block_mark[last] == ep ? a->block_val[last] : 0;
      if (a->ref[last] - drop > 1) {
        ++need;
        a->block_mark[last] = ep;
        a->block_val[last] = drop + 1;
        s.sim_last = -1;
      }
    }
    ++s.sim_len;
  }
  if (need > a->available()) return PA_ERR_NO_FREE_BLOCKS;
  int nc = 0;
  for (int i = 0; i < n; ++i) {
    int32_t src, dst;
    slots[i] = append_one(a, *a->batch[static_cast<size_t>(i)], &src, &dst);
    if (src >= 0) {
      cow_pairs[2 * nc] = src;
      cow_pairs[2 * nc + 1] = dst;
      ++nc;
    }
  }
  *num_cow = nc;
  return PA_OK;
}

int pa_seq_truncate(pa_alloc_t* a, const int64_t* seq_ids, const int64_t* new_lens, int n) {
  if (!a || n < 0 || (n > 0 && (!seq_ids || !new_lens))) return PA_ERR_INVALID_ARG;
  // validate first: all or nothing
  if (!a->resolve(seq_ids, n)) return PA_ERR_UNKNOWN_SEQ;
  const uint64_t ep = ++a->epoch;
  for (int i = 0; i < n; ++i) {
    Seq& s = *a->batch[static_cast<size_t>(i)];
    if (new_lens[i] < 0 || new_lens[i] > s.len) return PA_ERR_INVALID_ARG;
    if (s.mark == ep) return PA_ERR_INVALID_ARG;  // ids must be distinct
    s.mark = ep;
  }
  for (int i = 0; i < n; ++i) {
    Seq& s = *a->batch[static_cast<size_t>(i)];
    const size_t keep = static_cast<size_t>(blocks_for(new_lens[i], a->block_size));
    for (size_t j = keep; j < s.blocks.size(); ++j) a->dec(s.blocks[j]);
    if (keep < s.blocks.size()) s.blocks.resize(keep);
    s.len = new_lens[i];
  }
  return PA_OK;
}

int pa_seqs_move(pa_alloc_t* from, pa_alloc_t* to, const int64_t* seq_ids, int n,
                 int32_t* pairs_out, int64_t cap, int64_t* num_pairs) {
  if (!from || !to || from == to || n < 0 || !num_pairs || (n > 0 && !seq_ids))
    return PA_ERR_INVALID_ARG;
  if (from->block_size != to->block_size) return PA_ERR_INVALID_ARG;
  std::unordered_map<int64_t, int> seen;
  for (int i = 0; i < n; ++i) {
    if (seen[seq_ids[i]]++) return PA_ERR_INVALID_ARG;  // ids must be distinct
    if (!from->seqs.count(seq_ids[i])) return PA_ERR_UNKNOWN_SEQ;
    if (to->seqs.count(seq_ids[i])) return PA_ERR_SEQ_EXISTS;
  }
  // distinct blocks of the moved set, in order of first appearance
  std::vector<int32_t> distinct;
  std::unordered_map<int32_t, int32_t> index;
  for (int i = 0; i < n; ++i)
    for (int32_t b : from->seqs.find(seq_ids[i])->second.blocks)
      if (index.emplace(b, static_cast<int32_t>(distinct.size())).second) distinct.push_back(b);
  const int64_t nd = static_cast<int64_t>(distinct.size());
  if (nd > 0 && (!pairs_out || cap < nd)) return PA_ERR_INVALID_ARG;
  if (nd > to->available()) return PA_ERR_NO_FREE_BLOCKS;
  std::vector<int32_t> fresh(distinct.size());
  for (size_t k = 0; k < distinct.size(); ++k) {
    fresh[k] = to->pop();
    to->ref[fresh[k]] = 0;  // counted below, one per table entry
    pairs_out[2 * k] = distinct[k];
    pairs_out[2 * k + 1] = fresh[k];
  }
  for (int i = 0; i < n; ++i) {
    auto it = from->seqs.find(seq_ids[i]);
    Seq moved;
    moved.len = it->second.len;
    moved.blocks.reserve(it->second.blocks.size() + 1);
    for (int32_t b : it->second.blocks) {
      const int32_t nb = fresh[static_cast<size_t>(index[b])];
      moved.blocks.push_back(nb);
      to->inc(nb);
      from->dec(b);
    }
    from->seqs.erase(it);
    to->seqs.emplace(seq_ids[i], std::move(moved));
  }
  *num_pairs = nd;
  return PA_OK;
}

int pa_seq_free(pa_alloc_t* a, int64_t seq_id) {
  if (!a) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_UNKNOWN_SEQ;
  for (int32_t b : it->second.blocks) a->dec(b);
  a->seqs.erase(it);
  return PA_OK;
}

int pa_seq_len(const pa_alloc_t* a, int64_t seq_id, int64_t* len) {
  if (!a || !len) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_UNKNOWN_SEQ;
  *len = it->second.len;
  return PA_OK;
}

int pa_seq_blocks(const pa_alloc_t* a, int64_t seq_id, int32_t* out, int64_t cap, int64_t* n) {
  if (!a || !n || cap < 0 || (cap > 0 && !out)) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_UNKNOWN_SEQ;
  const auto& b = it->second.blocks;
  *n = static_cast<int64_t>(b.size());
  int64_t m = cap < *n ? cap : *n;
  if (m > 0) std::memcpy(out, b.data(), static_cast<size_t>(m) * sizeof(int32_t));
  return PA_OK;
}

int pa_build_block_tables(const pa_alloc_t* a, const int64_t* seq_ids, int num_seqs,
                          int32_t* tables, int max_blocks_per_seq, int32_t* seq_lens) {
  if (!a || num_seqs < 0 || max_blocks_per_seq < 0) return PA_ERR_INVALID_ARG;
  if (num_seqs > 0 && (!seq_ids || !tables || !seq_lens)) return PA_ERR_INVALID_ARG;
  pa_alloc* m = const_cast<pa_alloc*>(a);  // scratch only; the pool is not changed
  if (!m->resolve(seq_ids, num_seqs)) return PA_ERR_UNKNOWN_SEQ;
  for (int i = 0; i < num_seqs; ++i) {  // validate first: all or nothing
    const Seq& s = *m->batch[static_cast<size_t>(i)];
    if (static_cast<int64_t>(s.blocks.size()) > max_blocks_per_seq || s.len > INT32_MAX)
      return PA_ERR_INVALID_ARG;
  }
  for (int i = 0; i < num_seqs; ++i) {
    const Seq& s = *m->batch[static_cast<size_t>(i)];
    int32_t* row = tables + static_cast<int64_t>(i) * max_blocks_per_seq;
    size_t nb = s.blocks.size();
    if (nb) std::memcpy(row, s.blocks.data(), nb * sizeof(int32_t));
    for (int64_t j = static_cast<int64_t>(nb); j < max_blocks_per_seq; ++j) row[j] = -1;
    seq_lens[i] = static_cast<int32_t>(s.len);
  }
  return PA_OK;
}

int pa_build_prefix_groups(const pa_alloc_t* a, const int64_t* seq_ids, int num_seqs,
                           int partition_size, int max_members, int32_t* prefix_parts,
                           int32_t* chunk_members, int32_t* chunk_parts, int* num_chunks,
                           int* max_chunk_parts) {
  if (!a || num_seqs < 0 || partition_size <= 0 || max_members < 1 || !num_chunks ||
      !max_chunk_parts)
    return PA_ERR_INVALID_ARG;
  if (num_seqs > 0 && (!seq_ids || !prefix_parts || !chunk_members || !chunk_parts))
    return PA_ERR_INVALID_ARG;
  pa_alloc* m = const_cast<pa_alloc*>(a);  // scratch only; the pool is not changed
  if (!m->resolve(seq_ids, num_seqs)) return PA_ERR_UNKNOWN_SEQ;
  const std::vector<Seq*>& seqs = m->batch;
  // group positions by first physical block, in order of first appearance: block_val
  // holds a block's group while block_mark is this call's epoch
  const uint64_t ep = ++m->epoch;
  std::vector<int> gid(static_cast<size_t>(num_seqs), -1);
  std::vector<int> count;
  for (int i = 0; i < num_seqs; ++i) {
    prefix_parts[i] = 0;
    if (seqs[i]->blocks.empty()) continue;
    const int32_t b0 = seqs[i]->blocks[0];
    if (m->block_mark[b0] != ep) {
      m->block_mark[b0] = ep;
      m->block_val[b0] = static_cast<int32_t>(count.size());
      count.push_back(0);
    }
    gid[i] = m->block_val[b0];
    ++count[static_cast<size_t>(gid[i])];
  }
  // members of each group contiguous, in position order (a counting sort)
  std::vector<int> start(count.size() + 1, 0);
  for (size_t g = 0; g < count.size(); ++g) start[g + 1] = start[g] + count[g];
  std::vector<int> fill(start.begin(), start.end() - 1), flat(static_cast<size_t>(start.back()));
  for (int i = 0; i < num_seqs; ++i)
    if (gid[i] >= 0) flat[static_cast<size_t>(fill[static_cast<size_t>(gid[i])]++)] = i;
  int nc = 0, maxp = 0;
  for (size_t gi = 0; gi < count.size(); ++gi) {
    const int* g = flat.data() + start[gi];
    const size_t size = static_cast<size_t>(count[gi]);
    if (size < 2) continue;
    const auto& t0 = seqs[static_cast<size_t>(g[0])]->blocks;
    size_t common = t0.size();
    for (size_t k = 1; k < size && common > 0; ++k) {
      const auto& t = seqs[static_cast<size_t>(g[k])]->blocks;
      common = common_prefix(t0.data(), t.data(), common < t.size() ? common : t.size());
    }
    const int parts = static_cast<int>(static_cast<int64_t>(common) * a->block_size / partition_size);
    if (parts == 0) continue;
    for (size_t k = 0; k < size; ++k) prefix_parts[g[k]] = parts;
    for (size_t k = 0; k < size; k += static_cast<size_t>(max_members)) {
      int32_t* row = chunk_members + static_cast<int64_t>(nc) * max_members;
      for (int j = 0; j < max_members; ++j) {
        const size_t idx = k + static_cast<size_t>(j);
        row[j] = idx < size ? g[idx] : -1;
      }
      chunk_parts[nc] = parts;
      ++nc;
    }
    if (parts > maxp) maxp = parts;
  }
  *num_chunks = nc;
  *max_chunk_parts = maxp;
  return PA_OK;
}

int pa_block_refcount(const pa_alloc_t* a, int32_t block, int32_t* refcount) {
  if (!a || !refcount || block < 0 || block >= a->num_blocks) return PA_ERR_INVALID_ARG;
  *refcount = a->ref[block];
  return PA_OK;
}

int pa_alloc_free_list(const pa_alloc_t* a, int32_t* out, int64_t cap, int64_t* n) {
  if (!a || !n || cap < 0 || (cap > 0 && !out)) return PA_ERR_INVALID_ARG;
  const auto& fs = a->free_stack;
  *n = static_cast<int64_t>(fs.size());
  int64_t m = cap < *n ? cap : *n;
  for (int64_t i = 0; i < m; ++i) out[i] = fs[fs.size() - 1 - static_cast<size_t>(i)];
  return PA_OK;
}

int pa_alloc_stats(const pa_alloc_t* a, pa_stats_t* st) {
  if (!a || !st) return PA_ERR_INVALID_ARG;
  std::memset(st, 0, sizeof(*st));
  st->num_blocks = a->num_blocks;
  st->block_size = a->block_size;
  st->free_blocks = static_cast<int64_t>(a->free_stack.size());
  st->used_blocks = a->num_blocks - st->free_blocks - static_cast<int64_t>(a->evictable.size());
  st->shared_blocks = a->shared_blocks;
  st->num_seqs = static_cast<int64_t>(a->seqs.size());
  for (const auto& kv : a->seqs) {
    const Seq& s = kv.second;
    st->total_refs += static_cast<int64_t>(s.blocks.size());
    st->logical_tokens += s.len;
    st->tail_waste_slots += static_cast<int64_t>(s.blocks.size()) * a->block_size - s.len;
  }
  st->allocated_slots = st->used_blocks * a->block_size;
  st->cow_copies = a->cow_copies;
  st->blocks_allocated = a->blocks_allocated;
  st->cached_blocks = static_cast<int64_t>(a->cache.size());
  st->evictable_blocks = static_cast<int64_t>(a->evictable.size());
  st->cache_hits = a->cache_hits;
  st->cache_evictions = a->cache_evictions;
  return PA_OK;
}

}  // extern "C"
