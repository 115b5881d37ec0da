// Decode-step runtime: the host side of one decode step of a bound batch in native
// code, on top of the library's own entry points (block manager, cache kernels,
// decode attention).  The order of a step follows [BLOG] "How PagedAttention Powers
// vLLM's KV Cache" ("PagedAttention: paging, borrowed from the operating system",
// "The bonus contiguous storage can't give you: sharing"): room for the new token
// from the block manager (a copy first where its block is shared), the token's K/V
// written into its slot, then attention over every cached token.
//
// Buffers of a bound batch (laid out by pa_decoder_bind, never inside a step):
//   - two staging sets, each one page-locked host buffer (the decoder's own) and one
//     device buffer of the same layout (slots, copy pairs, lengths, block tables,
//     prefix groups); step k fills set k % 2 while the kernels of step k - 1 still
//     read the other, and one cudaMemcpyAsync on the decoder's copy stream moves the
//     whole set;
//   - the decode workspace for the bound batch at full table capacity;
//   - for steps fed from host memory, two device sets of q / new K / new V / out.
// All device memory comes from one caller-owned buffer (pa_decoder_device_bytes
// gives its size); the library allocates no device memory.
// Events order everything across the caller's stream and the decoder's streams;
// host waits happen only where a host buffer is about to be rewritten.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/pa.h"

namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int elem_size(int dtype) {
  switch (dtype) {
    case PA_F32: return 4;
    case PA_BF16:
    case PA_F16: return 2;
    case PA_FP8_E4M3: return 1;
    default: return 0;
  }
}

// Makes the decoder's device current for the scope of a call.
class DeviceGuard {
 public:
  explicit DeviceGuard(int dev) {
    int cur = -1;
    ok_ = cudaGetDevice(&cur) == cudaSuccess;
    if (ok_ && cur != dev) {
      ok_ = cudaSetDevice(dev) == cudaSuccess;
      if (ok_) prev_ = cur;
    }
  }
  ~DeviceGuard() {
    if (prev_ >= 0) cudaSetDevice(prev_);
  }
  bool ok() const { return ok_; }

 private:
  int prev_ = -1;
  bool ok_ = false;
};

struct StageSet {
  uint8_t* host = nullptr;  // page-locked
  uint8_t* dev = nullptr;
  cudaEvent_t h2d_done = nullptr;      // the host buffer may be rewritten
  cudaEvent_t kernels_done = nullptr;  // the device buffer may be overwritten
  bool h2d_pending = false, kernels_pending = false;
};

struct IoSet {
  void* q = nullptr;
  void* k = nullptr;
  void* v = nullptr;
  void* out = nullptr;
  cudaEvent_t h2d_done = nullptr, compute_done = nullptr, d2h_done = nullptr;
  int64_t ticket = 0;  // the last host-fed step that used the set
};

}  // namespace

struct pa_decoder {
  pa_decoder_config_t cfg{};
  pa_alloc_t* alloc = nullptr;
  int device = 0;
  cudaStream_t copy_stream = nullptr, h2d_stream = nullptr, d2h_stream = nullptr;

  // bound batch
  std::vector<int64_t> ids, base_lens;
  int num_seqs = 0, members = 0, partition = 0;
  bool bound = false, rolling = false, stepped = false;
  // a CUDA call failed after the block manager had committed a step: the allocator
  // is ahead of the device cache, so every later step is refused
  bool broken = false;
  size_t off_slots = 0, off_pairs = 0, off_lens = 0, off_tables = 0, off_pparts = 0,
         off_cmembers = 0, off_cparts = 0, off_order = 0, stage_bytes = 0;
  StageSet sets[2];
  int cur = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;

  // host-fed steps
  IoSet io[2];
  int io_next = 0;
  bool io_fresh = true;  // the I/O sets' events are recorded at the first host-fed step
  int64_t tickets = 0;
  size_t q_bytes = 0, kv_bytes = 0;

  bool fp8() const { return cfg.cache_dtype == PA_FP8_E4M3; }
  template <typename T>
  T* h(const StageSet& s, size_t off) const {
    return reinterpret_cast<T*>(s.host + off);
  }
  template <typename T>
  T* d(const StageSet& s, size_t off) const {
    return reinterpret_cast<T*>(s.dev + off);
  }
};

namespace {

// Waits for everything the decoder has in flight (host waits, bounded by the GPU).
cudaError_t quiesce(pa_decoder* d) {
  cudaError_t e = cudaSuccess;
  for (StageSet& s : d->sets) {
    if (s.h2d_pending && s.h2d_done) e = cudaEventSynchronize(s.h2d_done);
    if (e == cudaSuccess && s.kernels_pending && s.kernels_done)
      e = cudaEventSynchronize(s.kernels_done);
    if (e != cudaSuccess) return e;
  }
  for (IoSet& s : d->io)
    for (cudaEvent_t ev : {s.h2d_done, s.compute_done, s.d2h_done})
      if (ev && (e = cudaEventSynchronize(ev)) != cudaSuccess) return e;
  return e;
}

// Drops the bound batch's buffers: frees the page-locked staging halves (the
// decoder's own) and forgets the caller's device buffer.
void free_stage(pa_decoder* d) {
  for (StageSet& s : d->sets) {
    if (s.host) cudaFreeHost(s.host);
    s.host = nullptr;
    s.dev = nullptr;
    s.h2d_pending = s.kernels_pending = false;
  }
  d->ws = nullptr;
  d->ws_bytes = 0;
  for (IoSet& s : d->io) s.q = s.k = s.v = s.out = nullptr;
  d->io_fresh = true;
}

// Byte layout of a bound batch.  Staging offsets are the same in the host and the
// device halves; device offsets are into the caller's buffer.  Every piece starts on
// a 256-byte boundary.
struct BatchLayout {
  size_t off_slots, off_pairs, off_lens, off_tables, off_pparts, off_cmembers, off_cparts,
      off_order, stage_bytes;
  int partition;
  size_t ws_bytes, q_bytes, kv_bytes;
  size_t dev_stage[2], dev_ws, dev_io[2][4], device_bytes;
};

int plan_batch(const pa_decoder* d, int num_seqs, BatchLayout* L) {
  const pa_decoder_config_t& c = d->cfg;
  const int64_t cap = static_cast<int64_t>(c.max_blocks_per_seq) * c.block_size;
  int partition = c.partition_size;
  if (partition == 0) {
    partition = pa_decode_partition_size(c.cache_dtype, num_seqs, c.num_heads, c.num_kv_heads,
                                         c.head_dim, c.block_size, static_cast<int>(cap), 0);
    if (partition <= 0) return PA_ERR_CUDA;
  }
  L->partition = partition;
  L->ws_bytes = pa_decode_workspace_bytes(num_seqs, c.num_heads, c.head_dim,
                                          static_cast<int>(cap), partition);
  const size_t S = static_cast<size_t>(num_seqs);
  const size_t MM = static_cast<size_t>(std::max(1, d->members));
  size_t off = 0;
  auto take = [&off](size_t n) {
    const size_t at = off;
    off += align256(n);
    return at;
  };
  L->off_slots = take(8 * S);
  L->off_pairs = take(8 * S);
  L->off_lens = take(4 * S);
  L->off_tables = take(4 * S * static_cast<size_t>(c.max_blocks_per_seq));
  L->off_pparts = take(4 * S);
  L->off_cmembers = take(4 * S * MM);
  L->off_cparts = take(4 * S);
  L->off_order = take(4 * S);
  L->stage_bytes = off;
  L->q_bytes = S * c.num_heads * c.head_dim * elem_size(c.dtype);
  L->kv_bytes = S * c.num_kv_heads * c.head_dim * elem_size(c.dtype);
  size_t dev = 0;
  auto place = [&dev](size_t n) {
    const size_t at = dev;
    dev += align256(n);
    return at;
  };
  L->dev_stage[0] = place(L->stage_bytes);
  L->dev_stage[1] = place(L->stage_bytes);
  L->dev_ws = place(L->ws_bytes);
  for (auto& io : L->dev_io) {
    io[0] = place(L->q_bytes);   // q
    io[1] = place(L->kv_bytes);  // new K
    io[2] = place(L->kv_bytes);  // new V
    io[3] = place(L->q_bytes);   // out
  }
  L->device_bytes = dev;
  return PA_OK;
}

cudaError_t make_event(cudaEvent_t* ev) {
  return *ev ? cudaSuccess : cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

// Prefix groups are used by the decode call only for these shapes (the grouped entry
// point ignores them otherwise); the kernel count of a step follows the same rule.
bool groups_used(const pa_decoder* d, int parts) {
  const pa_decoder_config_t& c = d->cfg;
  const int group = c.num_heads / c.num_kv_heads;
  return !d->fp8() && d->members > 0 && parts > 1 && c.dtype != PA_F32 &&
         (c.block_size == 16 || c.block_size == 32) && d->members * group <= 16 &&
         (c.head_dim == 64 || c.head_dim == 128 || c.head_dim == 256);
}

// Host side of a step: block manager, staging, one copy to the device; the compute
// stream waits for the copy.
int prepare(pa_decoder* d, cudaStream_t comp, pa_step_info_t* info) {
  const int i = d->stepped ? d->cur ^ 1 : 0;
  StageSet& st = d->sets[i];
  if (st.h2d_pending) {  // that set's host buffer is free again after its copy
    cudaError_t e = cudaEventSynchronize(st.h2d_done);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    st.h2d_pending = false;
  }
  const int S = d->num_seqs;
  const pa_decoder_config_t& c = d->cfg;
  int rc;
  if (d->rolling && d->stepped) {
    rc = pa_seq_truncate(d->alloc, d->ids.data(), d->base_lens.data(), S);
    if (rc != PA_OK) return rc;
  }
  int ncow = 0;
  int64_t* slots = d->h<int64_t>(st, d->off_slots);
  int32_t* pairs = d->h<int32_t>(st, d->off_pairs);
  int32_t* tables = d->h<int32_t>(st, d->off_tables);
  int32_t* lens = d->h<int32_t>(st, d->off_lens);
  // Everything that can refuse the step is checked before the block manager commits
  // it: a sequence already at the table's capacity (rolling batches stay at their
  // bind-time lengths, which bind checked).  After the append only CUDA calls can
  // fail, and such a failure marks the decoder broken.
  if (!d->rolling) {
    const int64_t cap = static_cast<int64_t>(c.max_blocks_per_seq) * c.block_size;
    for (int s = 0; s < S; ++s) {
      int64_t len = 0;
      rc = pa_seq_len(d->alloc, d->ids[static_cast<size_t>(s)], &len);
      if (rc != PA_OK) return rc;
      if (len >= cap) return PA_ERR_INVALID_ARG;
    }
  }
  rc = pa_seq_append_slots(d->alloc, d->ids.data(), S, slots, pairs, &ncow);
  if (rc != PA_OK) return rc;
  d->cur = i;
  d->stepped = true;
  rc = pa_build_block_tables(d->alloc, d->ids.data(), S, tables, c.max_blocks_per_seq, lens);
  if (rc != PA_OK) {  // excluded by the checks above
    d->broken = true;
    return rc;
  }
  int max_len = 0;
  for (int s = 0; s < S; ++s) max_len = std::max(max_len, lens[s]);
  // the partition grid takes the sequences longest first (ties in batch order)
  int32_t* order = d->h<int32_t>(st, d->off_order);
  for (int s = 0; s < S; ++s) order[s] = s;
  std::stable_sort(order, order + S, [lens](int32_t x, int32_t y) { return lens[x] > lens[y]; });
  const int parts = (max_len + d->partition - 1) / d->partition;
  int num_chunks = 0, max_chunk_parts = 0, first_part = 0;
  if (groups_used(d, parts)) {
    int32_t* pp = d->h<int32_t>(st, d->off_pparts);
    rc = pa_build_prefix_groups(d->alloc, d->ids.data(), S, d->partition, d->members, pp,
                                d->h<int32_t>(st, d->off_cmembers),
                                d->h<int32_t>(st, d->off_cparts), &num_chunks,
                                &max_chunk_parts);
    if (rc != PA_OK) {  // excluded by the checks above
      d->broken = true;
      return rc;
    }
    if (num_chunks > 0) {
      // the lowest partition any sequence computes itself
      first_part = INT32_MAX;
      for (int s = 0; s < S; ++s) {
        const int own = lens[s] > 0 ? (lens[s] - 1) / d->partition : 0;
        first_part = std::min(first_part, std::min(pp[s], own));
      }
    }
  }
  cudaError_t e = cudaSuccess;
  if (st.kernels_pending) e = cudaStreamWaitEvent(d->copy_stream, st.kernels_done, 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st.dev, st.host, d->stage_bytes, cudaMemcpyHostToDevice, d->copy_stream);
  if (e == cudaSuccess) e = cudaEventRecord(st.h2d_done, d->copy_stream);
  if (e == cudaSuccess) st.h2d_pending = true;
  if (e == cudaSuccess) e = cudaStreamWaitEvent(comp, st.h2d_done, 0);
  if (e != cudaSuccess) {
    d->broken = true;
    return PA_ERR_CUDA;
  }

  info->num_cow = ncow;
  info->max_seq_len = max_len;
  info->partition_size = d->partition;
  info->num_chunks = num_chunks;
  info->max_chunk_parts = max_chunk_parts;
  info->first_part = first_part;
  // copies, the new tokens' write, the partition grid, then the merge (a grouped
  // call launches its counters' clear before the grid instead)
  info->kernels = (ncow ? 1 : 0) + 1 + 1 + (parts > 1 ? 1 : 0);
  info->slots = slots;
  info->cow_pairs = pairs;
  info->block_tables = tables;
  info->seq_lens = lens;
  return PA_OK;
}

// Device side of a step on the compute stream: copies, the new tokens' K/V, attention.
int launch(pa_decoder* d, const pa_step_info_t* info, const void* q, const void* new_k,
           const void* new_v, void* out, cudaStream_t comp, cudaEvent_t ev_begin,
           cudaEvent_t ev_end) {
  StageSet& st = d->sets[d->cur];
  const pa_decoder_config_t& c = d->cfg;
  const int S = d->num_seqs;
  int rc = PA_OK;
  if (info->num_cow > 0)
    rc = pa_copy_blocks(c.k_cache, c.v_cache, d->d<int32_t>(st, d->off_pairs), info->cow_pairs,
                        info->num_cow, c.num_kv_heads, c.head_dim, c.block_size, c.num_blocks,
                        c.cache_dtype, comp);
  if (rc != PA_OK) return rc;
  const int64_t* slots = d->d<int64_t>(st, d->off_slots);
  rc = d->fp8() ? pa_reshape_and_cache_fp8(new_k, new_v, c.k_cache, c.v_cache, slots, S,
                                           c.num_kv_heads, c.head_dim, c.block_size,
                                           c.num_blocks, c.dtype, c.k_scale, c.v_scale, comp)
                : pa_reshape_and_cache(new_k, new_v, c.k_cache, c.v_cache, slots, S,
                                       c.num_kv_heads, c.head_dim, c.block_size, c.num_blocks,
                                       c.dtype, comp);
  if (rc != PA_OK) return rc;
  if (ev_begin && cudaEventRecord(ev_begin, comp) != cudaSuccess) return PA_ERR_CUDA;
  const int32_t* tables = d->d<int32_t>(st, d->off_tables);
  const int32_t* lens = d->d<int32_t>(st, d->off_lens);
  pa_decode_args_t a{};
  a.struct_size = sizeof(a);
  a.out = out;
  a.q = q;
  a.k_cache = c.k_cache;
  a.v_cache = c.v_cache;
  a.block_tables = tables;
  a.seq_lens = lens;
  a.scale = c.scale;
  a.block_size = c.block_size;
  a.num_kv_heads = c.num_kv_heads;
  a.num_seqs = S;
  a.num_heads = c.num_heads;
  a.head_dim = c.head_dim;
  a.max_blocks_per_seq = c.max_blocks_per_seq;
  a.num_blocks = c.num_blocks;
  a.max_seq_len = info->max_seq_len;
  a.partition_size = d->partition;
  a.dtype = c.dtype;
  a.cache_dtype = c.cache_dtype;
  a.k_scale = c.k_scale;
  a.v_scale = c.v_scale;
  // longest first, prefix groups included: in the grouped grid the sequences' own
  // partitions follow the groups' shared ones, and taking them longest first shortens
  // the end of the grid (173.1 against 174.9 us on the 256-sequence shared-prefix batch)
  a.seq_order = d->d<int32_t>(st, d->off_order);
  if (info->num_chunks > 0) {
    a.prefix_parts = d->d<int32_t>(st, d->off_pparts);
    a.chunk_members = d->d<int32_t>(st, d->off_cmembers);
    a.chunk_parts = d->d<int32_t>(st, d->off_cparts);
    a.num_chunks = info->num_chunks;
    a.max_members = d->members;
    a.max_chunk_parts = info->max_chunk_parts;
    a.first_part = info->first_part;
  }
  a.workspace = d->ws;
  a.workspace_bytes = d->ws_bytes;
  a.stream = comp;
  rc = pa_decode(&a);
  if (rc != PA_OK) return rc;
  if (ev_end && cudaEventRecord(ev_end, comp) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaEventRecord(st.kernels_done, comp) != cudaSuccess) return PA_ERR_CUDA;
  st.kernels_pending = true;
  return PA_OK;
}

bool valid_config(const pa_decoder_config_t* c) {
  if (!c || c->struct_size != sizeof(pa_decoder_config_t)) return false;
  if (!c->k_cache || !c->v_cache || c->num_blocks <= 0 || c->num_kv_heads <= 0 ||
      c->num_heads <= 0 || c->num_heads % c->num_kv_heads || c->head_dim <= 0 ||
      c->block_size <= 0 || c->max_blocks_per_seq <= 0 || c->partition_size < 0 ||
      c->group_members < 0 || c->group_members > 16)
    return false;
  if (c->dtype != PA_F32 && c->dtype != PA_BF16 && c->dtype != PA_F16) return false;
  if (c->cache_dtype != c->dtype &&
      !(c->cache_dtype == PA_FP8_E4M3 && c->dtype != PA_F32))
    return false;
  if (c->partition_size % c->block_size) return false;
  if (static_cast<int64_t>(c->max_blocks_per_seq) * c->block_size > INT32_MAX) return false;
  return ((reinterpret_cast<uintptr_t>(c->k_cache) | reinterpret_cast<uintptr_t>(c->v_cache)) &
          15u) == 0;
}

}  // namespace

extern "C" {

int pa_decoder_create(const pa_decoder_config_t* cfg, pa_alloc_t* alloc, pa_decoder_t** out) {
  if (!out) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!alloc || !valid_config(cfg)) return PA_ERR_INVALID_ARG;
  pa_stats_t stats;
  if (pa_alloc_stats(alloc, &stats) != PA_OK || stats.block_size != cfg->block_size ||
      stats.num_blocks > cfg->num_blocks)
    return PA_ERR_INVALID_ARG;
  pa_decoder* d = new (std::nothrow) pa_decoder();
  if (!d) return PA_ERR_INVALID_ARG;
  d->cfg = *cfg;
  d->alloc = alloc;
  d->members = d->fp8() ? 0 : cfg->group_members;
  cudaError_t e = cudaGetDevice(&d->device);
  for (cudaStream_t* s : {&d->copy_stream, &d->h2d_stream, &d->d2h_stream})
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
  for (StageSet& s : d->sets) {
    if (e == cudaSuccess) e = make_event(&s.h2d_done);
    if (e == cudaSuccess) e = make_event(&s.kernels_done);
  }
  for (IoSet& s : d->io)
    for (cudaEvent_t* ev : {&s.h2d_done, &s.compute_done, &s.d2h_done})
      if (e == cudaSuccess) e = make_event(ev);
  if (e != cudaSuccess) {
    pa_decoder_destroy(d);
    return PA_ERR_CUDA;
  }
  *out = d;
  return PA_OK;
}

int pa_decoder_destroy(pa_decoder_t* d) {
  if (!d) return PA_ERR_INVALID_ARG;
  DeviceGuard g(d->device);
  quiesce(d);
  free_stage(d);
  for (StageSet& s : d->sets)
    for (cudaEvent_t ev : {s.h2d_done, s.kernels_done})
      if (ev) cudaEventDestroy(ev);
  for (IoSet& s : d->io)
    for (cudaEvent_t ev : {s.h2d_done, s.compute_done, s.d2h_done})
      if (ev) cudaEventDestroy(ev);
  for (cudaStream_t s : {d->copy_stream, d->h2d_stream, d->d2h_stream})
    if (s) cudaStreamDestroy(s);
  delete d;
  return PA_OK;
}

int pa_decoder_device_bytes(const pa_decoder_t* d, int num_seqs, size_t* bytes) {
  if (!d || num_seqs <= 0 || num_seqs > 65535 || !bytes) return PA_ERR_INVALID_ARG;
  DeviceGuard g(d->device);  // the partition choice asks the decoder's device
  if (!g.ok()) return PA_ERR_CUDA;
  BatchLayout L{};
  const int rc = plan_batch(d, num_seqs, &L);
  if (rc != PA_OK) return rc;
  *bytes = L.device_bytes;
  return PA_OK;
}

int pa_decoder_bind(pa_decoder_t* d, const int64_t* seq_ids, int num_seqs, int rolling,
                    void* device_buffer, size_t device_bytes) {
  if (!d || num_seqs <= 0 || !seq_ids || num_seqs > 65535) return PA_ERR_INVALID_ARG;
  if (!device_buffer || (reinterpret_cast<uintptr_t>(device_buffer) & 255u))
    return PA_ERR_INVALID_ARG;
  DeviceGuard g(d->device);
  if (!g.ok()) return PA_ERR_CUDA;
  const pa_decoder_config_t& c = d->cfg;
  std::vector<int64_t> ids(seq_ids, seq_ids + num_seqs), lens(static_cast<size_t>(num_seqs));
  std::vector<int64_t> sorted = ids;
  std::sort(sorted.begin(), sorted.end());
  if (std::adjacent_find(sorted.begin(), sorted.end()) != sorted.end()) return PA_ERR_INVALID_ARG;
  const int64_t cap = static_cast<int64_t>(c.max_blocks_per_seq) * c.block_size;
  for (int s = 0; s < num_seqs; ++s) {
    const int rc = pa_seq_len(d->alloc, ids[s], &lens[s]);
    if (rc != PA_OK) return rc;
    if (lens[s] >= cap) return PA_ERR_INVALID_ARG;  // no room for the step's token
  }
  BatchLayout L{};
  int rc = plan_batch(d, num_seqs, &L);
  if (rc != PA_OK) return rc;
  if (device_bytes < L.device_bytes) return PA_ERR_INVALID_ARG;
  if (quiesce(d) != cudaSuccess) return PA_ERR_CUDA;
  free_stage(d);
  d->bound = false;

  d->off_slots = L.off_slots;
  d->off_pairs = L.off_pairs;
  d->off_lens = L.off_lens;
  d->off_tables = L.off_tables;
  d->off_pparts = L.off_pparts;
  d->off_cmembers = L.off_cmembers;
  d->off_cparts = L.off_cparts;
  d->off_order = L.off_order;
  d->stage_bytes = L.stage_bytes;
  uint8_t* base = static_cast<uint8_t*>(device_buffer);
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < 2; ++i) {
    StageSet& st = d->sets[i];
    st.dev = base + L.dev_stage[i];
    if (e == cudaSuccess)
      e = cudaHostAlloc(reinterpret_cast<void**>(&st.host), L.stage_bytes, cudaHostAllocDefault);
    if (e == cudaSuccess) std::memset(st.host, 0, L.stage_bytes);
  }
  if (e != cudaSuccess) {
    free_stage(d);
    return PA_ERR_CUDA;
  }
  d->ws = L.ws_bytes ? base + L.dev_ws : nullptr;
  d->ws_bytes = L.ws_bytes;
  for (int i = 0; i < 2; ++i) {
    IoSet& io = d->io[i];
    io.q = base + L.dev_io[i][0];
    io.k = base + L.dev_io[i][1];
    io.v = base + L.dev_io[i][2];
    io.out = base + L.dev_io[i][3];
  }
  d->q_bytes = L.q_bytes;
  d->kv_bytes = L.kv_bytes;
  d->io_fresh = true;
  d->ids = std::move(ids);
  d->base_lens = std::move(lens);
  d->num_seqs = num_seqs;
  d->partition = L.partition;
  d->rolling = rolling != 0;
  d->stepped = false;
  d->broken = false;
  d->cur = 0;
  d->bound = true;
  return PA_OK;
}

int pa_decoder_step(pa_decoder_t* d, const void* q, const void* new_k, const void* new_v,
                    void* out, pa_stream_t stream, void* ev_begin, void* ev_end,
                    pa_step_info_t* info) {
  if (!d || !d->bound || !q || !new_k || !new_v || !out) return PA_ERR_INVALID_ARG;
  if (info && info->struct_size != sizeof(pa_step_info_t)) return PA_ERR_INVALID_ARG;
  if (d->broken) return PA_ERR_CUDA;
  DeviceGuard g(d->device);
  if (!g.ok()) return PA_ERR_CUDA;
  pa_step_info_t local{};
  pa_step_info_t* inf = info ? info : &local;
  cudaStream_t comp = static_cast<cudaStream_t>(stream);
  int rc = prepare(d, comp, inf);
  if (rc != PA_OK) return rc;
  rc = launch(d, inf, q, new_k, new_v, out, comp, static_cast<cudaEvent_t>(ev_begin),
              static_cast<cudaEvent_t>(ev_end));
  if (rc != PA_OK) d->broken = true;
  return rc;
}

int pa_decoder_step_host(pa_decoder_t* d, const void* q, const void* new_k, const void* new_v,
                         void* out, pa_stream_t stream, int64_t* ticket, pa_step_info_t* info) {
  if (!d || !d->bound || !q || !new_k || !new_v || !out) return PA_ERR_INVALID_ARG;
  if (info && info->struct_size != sizeof(pa_step_info_t)) return PA_ERR_INVALID_ARG;
  if (d->broken) return PA_ERR_CUDA;
  DeviceGuard g(d->device);
  if (!g.ok()) return PA_ERR_CUDA;
  cudaStream_t comp = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (d->io_fresh) {  // events start out completed
    for (IoSet& s : d->io)
      for (cudaEvent_t ev : {s.h2d_done, s.compute_done, s.d2h_done})
        if (e == cudaSuccess) e = cudaEventRecord(ev, comp);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    d->io_fresh = false;
    d->io_next = 0;
  }
  IoSet& io = d->io[d->io_next];
  // inputs: the set's previous kernels must be done with the device copies
  e = cudaStreamWaitEvent(d->h2d_stream, io.compute_done, 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(io.q, q, d->q_bytes, cudaMemcpyHostToDevice, d->h2d_stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(io.k, new_k, d->kv_bytes, cudaMemcpyHostToDevice, d->h2d_stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(io.v, new_v, d->kv_bytes, cudaMemcpyHostToDevice, d->h2d_stream);
  if (e == cudaSuccess) e = cudaEventRecord(io.h2d_done, d->h2d_stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(comp, io.h2d_done, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(comp, io.d2h_done, 0);  // out read back
  if (e != cudaSuccess) return PA_ERR_CUDA;
  pa_step_info_t local{};
  pa_step_info_t* inf = info ? info : &local;
  int rc = prepare(d, comp, inf);
  if (rc != PA_OK) return rc;
  rc = launch(d, inf, io.q, io.k, io.v, io.out, comp, nullptr, nullptr);
  if (rc == PA_OK) {
    e = cudaEventRecord(io.compute_done, comp);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(d->d2h_stream, io.compute_done, 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(out, io.out, d->q_bytes, cudaMemcpyDeviceToHost, d->d2h_stream);
    if (e == cudaSuccess) e = cudaEventRecord(io.d2h_done, d->d2h_stream);
    if (e != cudaSuccess) rc = PA_ERR_CUDA;
  }
  if (rc != PA_OK) {
    d->broken = true;
    return rc;
  }
  d->io_next ^= 1;
  io.ticket = ++d->tickets;
  if (ticket) *ticket = io.ticket;
  return PA_OK;
}

int pa_decoder_wait(pa_decoder_t* d, int64_t ticket) {
  if (!d || ticket <= 0 || ticket > d->tickets) return PA_ERR_INVALID_ARG;
  // Read-backs run in order on one stream, so the set that holds this ticket, or
  // else the older of the two (both newer than the ticket), completes it.
  const IoSet& a = d->io[0];
  const IoSet& b = d->io[1];
  const IoSet& s = a.ticket == ticket ? a : b.ticket == ticket ? b : a.ticket < b.ticket ? a : b;
  if (!s.d2h_done) return PA_OK;
  return cuda_status(cudaEventSynchronize(s.d2h_done));
}

int pa_decoder_drain(pa_decoder_t* d, pa_stream_t stream) {
  if (!d) return PA_ERR_INVALID_ARG;
  if (!d->bound || d->io_fresh) return PA_OK;
  DeviceGuard g(d->device);
  cudaStream_t comp = static_cast<cudaStream_t>(stream);
  for (IoSet& s : d->io)
    if (cudaStreamWaitEvent(comp, s.d2h_done, 0) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

int pa_decoder_query(const pa_decoder_t* d, int* partition_size, size_t* workspace_bytes,
                     size_t* staging_bytes) {
  if (!d || !d->bound) return PA_ERR_INVALID_ARG;
  if (partition_size) *partition_size = d->partition;
  if (workspace_bytes) *workspace_bytes = d->ws_bytes;
  if (staging_bytes) *staging_bytes = d->stage_bytes;
  return PA_OK;
}

}  // extern "C"
