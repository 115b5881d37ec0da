// Cache maintenance kernels: pa_reshape_and_cache (write each new token's K/V into
// its slot) and pa_copy_blocks (the private copy of copy-on-write).
//
// "How PagedAttention Powers vLLM's KV Cache" (hassanahmed.net), "Quick recap: the
// KV cache is per token, and it grows" and "The bonus contiguous storage can't give
// you: sharing"; "PagedAttention" attention-lab explainer (divagr.pages.dev),
// "Share matching prefixes".
//
// Both are pure HBM copies: 16-byte vectors, one per thread per step, grid-stride
// loops sized to the SM count.  Cache layout [num_blocks, num_kv_heads, block_size,
// head_dim]; one block of one tensor is num_kv_heads*block_size*head_dim elements.
#include <algorithm>
#include <cmath>
#include <vector>

#include "common.cuh"

namespace pa {
namespace {

// One 16-byte vector of one token row per thread.  nvr = vectors per (token, head) row.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int64_t num_tokens,
    int num_kv_heads, int nvr, int block_size, int64_t num_slots, uint32_t* err) {
  allow_dependents();  // the decode kernel after this one may start its prologue
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * nvr;
  const int64_t total = num_tokens * per_token;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t r = i - t * per_token;
    const int h = static_cast<int>(r / nvr);
    const int v = static_cast<int>(r - static_cast<int64_t>(h) * nvr);
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      set_error(err, PA_DEVERR_SLOT);
      continue;
    }
    const int64_t blk = slot / block_size;
    const int64_t off = slot - blk * block_size;
    // cache row (blk, h, off): ((blk * Hkv + h) * bs + off) * nvr vectors
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * nvr + v;
    k_cache[dst] = __ldg(key + i);
    v_cache[dst] = __ldg(value + i);
  }
}

// fp8 write: each thread makes one 16-byte vector of e4m3 codes (16 elements of one
// token row) from the float32 value of each input element times the reciprocal of
// the tensor's scale, rounded to nearest even and saturated (CUDA's conversion).
template <typename TQ>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(
    const TQ* __restrict__ key, const TQ* __restrict__ value, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int64_t num_tokens,
    int num_kv_heads, int head_dim, int block_size, int64_t num_slots, float k_inv,
    float v_inv, uint32_t* err) {
  allow_dependents();  // the decode kernel after this one may start its prologue
  constexpr int VQ = ElemTraits<TQ>::kVec;
  const int nvr = head_dim / 16;  // output vectors per (token, head) row
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * nvr;
  const int64_t total = num_tokens * per_token;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int64_t r = i - t * per_token;
    const int h = static_cast<int>(r / nvr);
    const int v = static_cast<int>(r - static_cast<int64_t>(h) * nvr);
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      set_error(err, PA_DEVERR_SLOT);
      continue;
    }
    const int64_t src = (t * num_kv_heads + h) * head_dim + v * 16;
    const int64_t blk = slot / block_size;
    const int64_t off = slot - blk * block_size;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * nvr + v;
#pragma unroll
    for (int kv = 0; kv < 2; ++kv) {
      const TQ* in = (kv ? value : key) + src;
      const float inv = kv ? v_inv : k_inv;
      float f[16];
#pragma unroll
      for (int u = 0; u < 16 / VQ; ++u)
        vec_to_float(__ldg(reinterpret_cast<const uint4*>(in + u * VQ)), f + u * VQ, TQ());
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_fp8x2_storage_t lo =
            __nv_cvt_float2_to_fp8x2(make_float2(f[4 * j] * inv, f[4 * j + 1] * inv),
                                     __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi =
            __nv_cvt_float2_to_fp8x2(make_float2(f[4 * j + 2] * inv, f[4 * j + 3] * inv),
                                     __NV_SATFINITE, __NV_E4M3);
        w[j] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
      }
      (kv ? v_cache : k_cache)[dst] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// grid: x = chunk of the block, y = pair, z = 0 (K) / 1 (V).  Each CTA copies
// kCopyPerThread*256 vectors of one block of one tensor from the source cache to the
// destination cache (the same cache for copy-on-write; a device and a host-resident
// cache for swapping).
constexpr int kCopyPerThread = 4;
__global__ void __launch_bounds__(256) copy_blocks_kernel(
    uint4* __restrict__ dst_k, uint4* __restrict__ dst_v, const uint4* __restrict__ src_k,
    const uint4* __restrict__ src_v, const int32_t* __restrict__ mapping, int64_t vecs_per_block,
    int64_t src_blocks, int64_t dst_blocks, uint32_t* err) {
  const int32_t src = __ldg(mapping + 2 * blockIdx.y);
  const int32_t dst = __ldg(mapping + 2 * blockIdx.y + 1);
  if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) set_error(err, PA_DEVERR_COPY_BLOCK);
    return;
  }
  const uint4* s = (blockIdx.z ? src_v : src_k) + static_cast<int64_t>(src) * vecs_per_block;
  uint4* d = (blockIdx.z ? dst_v : dst_k) + static_cast<int64_t>(dst) * vecs_per_block;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * (256 * kCopyPerThread) + threadIdx.x;
  uint4 tmp[kCopyPerThread];
#pragma unroll
  for (int u = 0; u < kCopyPerThread; ++u) {
    const int64_t i = first + u * 256;
    if (i < vecs_per_block) tmp[u] = s[i];
  }
#pragma unroll
  for (int u = 0; u < kCopyPerThread; ++u) {
    const int64_t i = first + u * 256;
    if (i < vecs_per_block) d[i] = tmp[u];
  }
}

int elem_bytes(int dtype) {
  switch (dtype) {
    case PA_F32: return 4;
    case PA_BF16: return 2;
    case PA_F16: return 2;
    case PA_FP8_E4M3: return 1;
    default: return 0;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The address a kernel on the current device may use for p: device memory of this
// device, or page-locked host memory (reachable through unified addressing).  Returns
// nullptr for anything else (pageable host memory, another device's memory).
const void* device_view(const void* p) {
  if (!p) return nullptr;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();  // clear the non-sticky error
    return nullptr;
  }
  if ((at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) && at.device == dev)
    return at.devicePointer ? at.devicePointer : p;
  if (at.type == cudaMemoryTypeHost && at.devicePointer) return at.devicePointer;
  return nullptr;
}

// Host-side check of a (src, dst) pair list: ids in range, destinations distinct, and
// (same_cache) no destination that is also a source.
bool pairs_ok(const int32_t* pairs, int n, int64_t src_blocks, int64_t dst_blocks,
              bool same_cache) {
  std::vector<int32_t> dsts(n), srcs(n);
  for (int i = 0; i < n; ++i) {
    srcs[i] = pairs[2 * i];
    dsts[i] = pairs[2 * i + 1];
    if (srcs[i] < 0 || srcs[i] >= src_blocks || dsts[i] < 0 || dsts[i] >= dst_blocks) return false;
  }
  std::sort(dsts.begin(), dsts.end());
  if (std::adjacent_find(dsts.begin(), dsts.end()) != dsts.end()) return false;
  if (same_cache) {
    std::sort(srcs.begin(), srcs.end());
    for (int32_t d : dsts)
      if (std::binary_search(srcs.begin(), srcs.end(), d)) return false;
  }
  return true;
}

int launch_copy(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                const int32_t* mapping, int num_pairs, int64_t block_bytes, int64_t src_blocks,
                int64_t dst_blocks, cudaStream_t stream) {
  const int64_t vecs = block_bytes / 16;
  const int64_t chunks = (vecs + 256 * kCopyPerThread - 1) / (256 * kCopyPerThread);
  if (chunks > 0x7fffffff) return PA_ERR_INVALID_ARG;
  uint32_t* err = device_error_word();
  if (!err) {
    note_cuda_error(cudaGetLastError());
    return PA_ERR_CUDA;
  }
  dim3 grid(static_cast<unsigned>(chunks), static_cast<unsigned>(num_pairs), 2);
  copy_blocks_kernel<<<grid, 256, 0, stream>>>(
      static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), static_cast<const uint4*>(src_k),
      static_cast<const uint4*>(src_v), mapping, vecs, src_blocks, dst_blocks, err);
  const cudaError_t e = cudaGetLastError();
  note_cuda_error(e);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" int pa_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache,
                                        void* v_cache, const int64_t* slot_mapping,
                                        int64_t num_tokens, int num_kv_heads, int head_dim,
                                        int block_size, int64_t num_blocks, int input_dtype,
                                        float k_scale, float v_scale, pa_stream_t stream) {
  if ((input_dtype != PA_F32 && input_dtype != PA_BF16 && input_dtype != PA_F16) ||
      num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 16 != 0 ||
      block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  const float k_inv = 1.0f / k_scale, v_inv = 1.0f / v_scale;
  const int64_t total = num_tokens * num_kv_heads * (head_dim / 16);
  const int64_t want = (total + 255) / 256;
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sm_count()) * 8));
  uint32_t* err = device_error_word();
  if (!err) {
    note_cuda_error(cudaGetLastError());
    return PA_ERR_CUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t slots = num_blocks * block_size;
  auto* kc = static_cast<uint4*>(k_cache);
  auto* vc = static_cast<uint4*>(v_cache);
  if (input_dtype == PA_BF16)
    reshape_and_cache_fp8_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(key), static_cast<const __nv_bfloat16*>(value), kc, vc,
        slot_mapping, num_tokens, num_kv_heads, head_dim, block_size, slots, k_inv, v_inv, err);
  else if (input_dtype == PA_F16)
    reshape_and_cache_fp8_kernel<__half><<<grid, 256, 0, st>>>(
        static_cast<const __half*>(key), static_cast<const __half*>(value), kc, vc, slot_mapping,
        num_tokens, num_kv_heads, head_dim, block_size, slots, k_inv, v_inv, err);
  else
    reshape_and_cache_fp8_kernel<float><<<grid, 256, 0, st>>>(
        static_cast<const float*>(key), static_cast<const float*>(value), kc, vc, slot_mapping,
        num_tokens, num_kv_heads, head_dim, block_size, slots, k_inv, v_inv, err);
  const cudaError_t e = cudaGetLastError();
  note_cuda_error(e);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                    void* v_cache, const int64_t* slot_mapping,
                                    int64_t num_tokens, int num_kv_heads, int head_dim,
                                    int block_size, int64_t num_blocks, int dtype,
                                    pa_stream_t stream) {
  const int eb = elem_bytes(dtype);
  if (eb == 0 || num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if ((static_cast<int64_t>(head_dim) * eb) % 16 != 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;  // (an fp8 cache copies fp8 rows here, bit for bit)
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  const int nvr = head_dim * eb / 16;
  const int64_t total = num_tokens * num_kv_heads * nvr;
  const int64_t want = (total + 255) / 256;
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sm_count()) * 8));
  uint32_t* err = device_error_word();
  if (!err) {
    note_cuda_error(cudaGetLastError());
    return PA_ERR_CUDA;
  }
  reshape_and_cache_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value),
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slot_mapping, num_tokens,
      num_kv_heads, nvr, block_size, num_blocks * block_size, err);
  const cudaError_t e = cudaGetLastError();
  note_cuda_error(e);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* block_mapping_dev,
                              const int32_t* block_mapping_host, int num_pairs, int num_kv_heads,
                              int head_dim, int block_size, int64_t num_blocks, int dtype,
                              pa_stream_t stream) {
  const int eb = elem_bytes(dtype);
  if (eb == 0 || num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || num_pairs > 65535)
    return PA_ERR_INVALID_ARG;
  const int64_t block_bytes = static_cast<int64_t>(num_kv_heads) * block_size * head_dim * eb;
  if (block_bytes % 16 != 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !block_mapping_dev) return PA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
  if (block_mapping_host && !pairs_ok(block_mapping_host, num_pairs, num_blocks, num_blocks, true))
    return PA_ERR_INVALID_ARG;
  return launch_copy(k_cache, v_cache, k_cache, v_cache, block_mapping_dev, num_pairs, block_bytes,
                     num_blocks, num_blocks, static_cast<cudaStream_t>(stream));
}

extern "C" int pa_swap_blocks(void* dst_k, void* dst_v, int64_t dst_num_blocks,
                              const void* src_k, const void* src_v, int64_t src_num_blocks,
                              const int32_t* block_mapping, const int32_t* block_mapping_host,
                              int num_pairs, int num_kv_heads, int head_dim, int block_size,
                              int dtype, pa_stream_t stream) {
  const int eb = elem_bytes(dtype);
  if (eb == 0 || num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      dst_num_blocks <= 0 || src_num_blocks <= 0 || num_pairs > 65535)
    return PA_ERR_INVALID_ARG;
  const int64_t block_bytes = static_cast<int64_t>(num_kv_heads) * block_size * head_dim * eb;
  if (block_bytes % 16 != 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!aligned16(dst_k) || !aligned16(dst_v) || !aligned16(src_k) || !aligned16(src_v))
    return PA_ERR_INVALID_ARG;
  // every pointer the kernel dereferences must be reachable from this device
  const void* dk = device_view(dst_k);
  const void* dv = device_view(dst_v);
  const void* sk = device_view(src_k);
  const void* sv = device_view(src_v);
  const void* mp = device_view(block_mapping);
  if (!dk || !dv || !sk || !sv || !mp) return PA_ERR_INVALID_ARG;
  if (block_mapping_host &&
      !pairs_ok(block_mapping_host, num_pairs, src_num_blocks, dst_num_blocks, false))
    return PA_ERR_INVALID_ARG;
  return launch_copy(const_cast<void*>(dk), const_cast<void*>(dv), sk, sv,
                     static_cast<const int32_t*>(mp), num_pairs, block_bytes, src_num_blocks,
                     dst_num_blocks, static_cast<cudaStream_t>(stream));
}
