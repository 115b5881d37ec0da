// pa_decode_attention_static_ws: decode attention for callers that may not allocate
// device memory.  The partition scratch lives in one fixed array that the library
// itself owns; the caller still passes every input and output.
//
// The array is a file-scope device variable, so every GPU that loads the library
// holds PA_STATIC_WORKSPACE_BYTES of it until the process exits.  Host code must not
// hand the array's name to a kernel (on the host it is only a stand-in symbol): the
// device address is looked up with cudaGetSymbolAddress, once per device, by the
// first call made with that device current, and cached.
#include <atomic>

#include "common.cuh"

static __device__ __align__(256) unsigned char g_pa_static_workspace[PA_STATIC_WORKSPACE_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<void*> g_static_ws_addr[kMaxDevices];

// Device address of the array on the current device (set up on first use).
int static_workspace_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    pa::note_cuda_error(e);
    return PA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
  void* p = g_static_ws_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_pa_static_workspace);
    if (e != cudaSuccess || !p) {
      pa::note_cuda_error(e);
      return PA_ERR_CUDA;
    }
    g_static_ws_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return PA_OK;
}

}  // namespace

extern "C" int pa_decode_attention_static_ws(void* out, const void* q, const void* k_cache,
                                             const void* v_cache, const int32_t* block_tables,
                                             const int32_t* seq_lens, float scale,
                                             int block_size, int num_kv_heads, int num_seqs,
                                             int num_heads, int head_dim, int max_blocks_per_seq,
                                             int64_t num_blocks, int max_seq_len,
                                             int partition_size, int dtype, pa_stream_t stream) {
  const size_t need = pa_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_seq_len,
                                                partition_size);
  if (need > static_cast<size_t>(PA_STATIC_WORKSPACE_BYTES)) return PA_ERR_TOO_LARGE;
  void* ws = nullptr;
  const int rc = static_workspace_address(&ws);
  if (rc != PA_OK) return rc;
  return pa_decode_attention(out, q, k_cache, v_cache, block_tables, seq_lens, scale,
                             block_size, num_kv_heads, num_seqs, num_heads, head_dim,
                             max_blocks_per_seq, num_blocks, max_seq_len, partition_size, dtype,
                             ws, static_cast<size_t>(PA_STATIC_WORKSPACE_BYTES), stream);
}
