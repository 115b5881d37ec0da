// pa_decode_attention: argument checks, workspace layout, choice of partition
// kernel (tensor-core tile for grouped-query head groups, CUDA cores otherwise) and
// the log-sum-exp merge kernel that combines partitions.
//
// "How PagedAttention Powers vLLM's KV Cache" (hassanahmed.net), "The attention
// kernel has to read scattered blocks" and "Where it bites" (grouped-query
// attention); "PagedAttention" attention-lab explainer (divagr.pages.dev), "Keep
// pages in order" and "Measure memory use across requests" (the attention equation
// is unchanged by paging).
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "decode_simt.cuh"

namespace pa {

cudaError_t launch_decode_simt_f32(const DecodeParams& p, int gs, cudaStream_t st);
cudaError_t launch_decode_simt_bf16(const DecodeParams& p, int gs, cudaStream_t st);
cudaError_t launch_decode_simt_f16(const DecodeParams& p, int gs, cudaStream_t st);
cudaError_t launch_decode_simt_fp8(const DecodeParams& p, int q_dtype, int gs, cudaStream_t st);
cudaError_t launch_decode_mma_fp8(const DecodeParams& p, int q_dtype, cudaStream_t st);
cudaError_t launch_decode_tc_fp8(const DecodeParams& p, int q_dtype, cudaStream_t st);
bool tc_fp8_eligible(int group, int head_dim, int block_size, int num_seqs, int num_kv_heads);
cudaError_t launch_decode_mma_bf16(const DecodeParams& p, cudaStream_t st);
cudaError_t launch_decode_mma_f16(const DecodeParams& p, cudaStream_t st);
cudaError_t launch_decode_grouped_bf16(const DecodeParams& p, cudaStream_t st);
cudaError_t launch_decode_grouped_f16(const DecodeParams& p, cudaStream_t st);

namespace {

constexpr int kDefaultPartition = 512;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct WsLayout {
  int parts = 1;
  size_t o_off = 0, m_off = 0, l_off = 0, cnt_off = 0, bytes = 0;
};

WsLayout ws_layout(int64_t num_seqs, int64_t num_heads, int64_t head_dim, int64_t max_seq_len,
                   int64_t partition_size) {
  WsLayout w;
  w.parts = max_seq_len > 0 ? static_cast<int>((max_seq_len + partition_size - 1) / partition_size) : 1;
  if (w.parts <= 1) return w;
  const size_t rows = static_cast<size_t>(num_seqs) * num_heads * w.parts;
  w.o_off = 0;
  w.m_off = align256(rows * head_dim * sizeof(float));
  w.l_off = w.m_off + align256(rows * sizeof(float));
  w.cnt_off = w.l_off + align256(rows * sizeof(float));
  w.bytes = w.cnt_off + align256(static_cast<size_t>(num_seqs) * num_heads * sizeof(int));
  return w;
}

// Merge: combine the partitions of every (sequence, head) row that has more than one:
//   M = max_p m_p,  w_p = l_p 2^(m_p - M),  out = sum_p w_p o_p / sum_p w_p
// (m_p in base-2 logits, o_p normalised by its own l_p).  A CTA of 8 warps serves
// 8/WPR rows with WPR warps each (WPR grows with the partition count, so long rows
// are read by up to 8 warps at once); lanes own head_dim/32 consecutive elements.
// Each warp walks partitions wsub, wsub+WPR, ... eight at a time with a running
// maximum (earlier sums rescaled when it grows), so the partials are read in one pass
// with eight loads in flight per lane; the row's warps then combine their (max, sum,
// weighted output) in shared memory.  (Up to 16 warps per row, each reading about
// eight partitions, measured 4 µs slower on the long-context shape: 352.6 against
// 348.7 µs per call.)
template <int DPL>
__device__ __forceinline__ void load_lane(const float* src, float (&o)[DPL]) {
  if constexpr (DPL % 4 == 0) {
#pragma unroll
    for (int j = 0; j < DPL; j += 4) {
      const float4 v = *reinterpret_cast<const float4*>(src + j);
      o[j] = v.x;
      o[j + 1] = v.y;
      o[j + 2] = v.z;
      o[j + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < DPL; j += 2) {
      const float2 v = *reinterpret_cast<const float2*>(src + j);
      o[j] = v.x;
      o[j + 1] = v.y;
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) merge_kernel(const DecodeParams p, int wpr) {
  constexpr int DPL = D / 32;
  constexpr int U = 8;  // partitions in flight per warp
  __shared__ float sh_acc[8][D];
  __shared__ float sh_den[8], sh_max[8];
  grid_dependency_wait();  // the partials of the partition kernel before this one
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_per_cta = 8 / wpr;
  const int wsub = warp % wpr;
  const int row = blockIdx.x * rows_per_cta + warp / wpr;
  // slots: partitions 0, step, 2 step, ... (a partition kernel that ran `step`
  // consecutive partitions per CTA left one partial in the first one's slot)
  const int step = p.part_step > 1 ? p.part_step : 1;
  int nparts = 0;
  if (row < p.num_seqs * p.num_heads) {
    const int L = checked_len(p, row / p.num_heads, false);
    nparts = L > 0 ? (L + p.partition_size - 1) / p.partition_size : 1;
    nparts = (nparts + step - 1) / step;
  }
  float acc[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) acc[j] = 0.f;
  float den = 0.f, M = -INFINITY;
  if (nparts > 1) {
    const int64_t mstride = static_cast<int64_t>(p.num_seqs) * p.num_heads;
    const int64_t sstride = mstride * step;  // slot pi (partition pi * step): pi * sstride
    const float* mrow = p.ws_m + row;
    const float* lrow = p.ws_l + row;
    const float* orow = p.ws_o + static_cast<int64_t>(row) * D + lane * DPL;
    for (int i = wsub; i < nparts; i += U * wpr) {
      float mv[U], lv[U], o[U][DPL];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int pi = i + u * wpr;
        if (pi < nparts) {
          mv[u] = mrow[pi * sstride];
          lv[u] = lrow[pi * sstride];
          load_lane<DPL>(orow + pi * sstride * D, o[u]);
        } else {
          mv[u] = -INFINITY;
          lv[u] = 0.f;
#pragma unroll
          for (int j = 0; j < DPL; ++j) o[u][j] = 0.f;
        }
      }
      float mx = M;
#pragma unroll
      for (int u = 0; u < U; ++u) mx = fmaxf(mx, mv[u]);
      const float c = exp2_safe(M, mx);
      den *= c;
#pragma unroll
      for (int j = 0; j < DPL; ++j) acc[j] *= c;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float w = lv[u] * exp2_safe(mv[u], mx);
        den += w;
#pragma unroll
        for (int j = 0; j < DPL; ++j) acc[j] = fmaf(w, o[u][j], acc[j]);
      }
      M = mx;
    }
  }
  if (wpr > 1) {
#pragma unroll
    for (int j = 0; j < DPL; ++j) sh_acc[warp][lane * DPL + j] = acc[j];
    if (lane == 0) {
      sh_den[warp] = den;
      sh_max[warp] = M;
    }
    __syncthreads();
    if (wsub == 0) {
      float Mr = M;
      for (int w2 = 1; w2 < wpr; ++w2) Mr = fmaxf(Mr, sh_max[warp + w2]);
      const float c0 = exp2_safe(M, Mr);
      den *= c0;
#pragma unroll
      for (int j = 0; j < DPL; ++j) acc[j] *= c0;
      for (int w2 = 1; w2 < wpr; ++w2) {
        const float c = exp2_safe(sh_max[warp + w2], Mr);
#pragma unroll
        for (int j = 0; j < DPL; ++j) acc[j] = fmaf(c, sh_acc[warp + w2][lane * DPL + j], acc[j]);
        den = fmaf(c, sh_den[warp + w2], den);
      }
    }
  }
  if (nparts > 1 && wsub == 0) {
    T* out = static_cast<T*>(p.out) + static_cast<int64_t>(row) * D + lane * DPL;
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int j = 0; j < DPL; ++j) store_elem(out + j, acc[j] * inv);
  }
}

// The same merge for partials written sparsely: a partition kernel that runs several
// consecutive partitions of a row in one CTA combines them itself (by the same rule)
// and leaves one partial for the range, in its first slot; its other slots hold an
// empty partial (exp-sum 0).  One warp per row: the lanes read the row's maxima and
// exp-sums 256 slots at a time (eight per lane in flight), list the slots with a
// non-zero exp-sum in shared memory, and only those partial outputs are read, sixteen
// in flight (eight for head_dim 256).  Any mix of full and empty slots gives the dense
// merge's result.
template <typename T, int D>
__global__ void __launch_bounds__(128) merge_sparse_kernel(const DecodeParams p) {
  constexpr int DPL = D / 32;
  constexpr int kWin = 256;  // slots examined per window
  constexpr int U = D <= 128 ? 16 : 8;  // partial outputs in flight per warp
  __shared__ int sh_slot[4][kWin];
  __shared__ float sh_mv[4][kWin], sh_lv[4][kWin];
  grid_dependency_wait();  // the partials of the partition kernel before this one
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;
  if (row >= p.num_seqs * p.num_heads) return;  // (no block-wide barrier below)
  const int L = checked_len(p, row / p.num_heads, false);
  const int nparts = L > 0 ? (L + p.partition_size - 1) / p.partition_size : 1;
  if (nparts <= 1) return;
  const int64_t mstride = static_cast<int64_t>(p.num_seqs) * p.num_heads;
  float acc[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) acc[j] = 0.f;
  float den = 0.f, M = -INFINITY;
  for (int w0 = 0; w0 < nparts; w0 += kWin) {
    float mv[kWin / 32], lv[kWin / 32];
#pragma unroll
    for (int k = 0; k < kWin / 32; ++k) {
      const int pi = w0 + k * 32 + lane;
      mv[k] = pi < nparts ? p.ws_m[pi * mstride + row] : -INFINITY;
      lv[k] = pi < nparts ? p.ws_l[pi * mstride + row] : 0.f;
    }
    int n = 0;
    float mx = M;
#pragma unroll
    for (int k = 0; k < kWin / 32; ++k) {
      const bool keep = lv[k] > 0.f;
      const uint32_t b = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const int at = n + __popc(b & ((1u << lane) - 1u));
        sh_slot[warp][at] = w0 + k * 32 + lane;
        sh_mv[warp][at] = mv[k];
        sh_lv[warp][at] = lv[k];
        mx = fmaxf(mx, mv[k]);
      }
      n += __popc(b);
    }
    mx = warp_max(mx);
    const float c = exp2_safe(M, mx);
    den *= c;
#pragma unroll
    for (int j = 0; j < DPL; ++j) acc[j] *= c;
    M = mx;
    __syncwarp();
    for (int b0 = 0; b0 < n; b0 += U) {
      float o[U][DPL], w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int at = b0 + u;
        if (at < n) {
          w[u] = sh_lv[warp][at] * exp2_safe(sh_mv[warp][at], M);
          load_lane<DPL>(p.ws_o + (sh_slot[warp][at] * mstride + row) * D + lane * DPL, o[u]);
        } else {
          w[u] = 0.f;
#pragma unroll
          for (int j = 0; j < DPL; ++j) o[u][j] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        den += w[u];
#pragma unroll
        for (int j = 0; j < DPL; ++j) acc[j] = fmaf(w[u], o[u][j], acc[j]);
      }
    }
    __syncwarp();  // the list is read before the next window overwrites it
  }
  T* out = static_cast<T*>(p.out) + static_cast<int64_t>(row) * D + lane * DPL;
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int j = 0; j < DPL; ++j) store_elem(out + j, acc[j] * inv);
}

// dependent: launched to overlap the tail of the partition kernel just before it on
// the stream (not after an event wait, which must hold in full)
template <typename T, int D>
cudaError_t launch_merge_d(const DecodeParams& p, int grid, int wpr, bool dependent,
                           bool sparse, cudaStream_t st) {
  if (sparse) {
    const int g4 = (p.num_seqs * p.num_heads + 3) / 4;
    if (dependent) return launch_dependent(merge_sparse_kernel<T, D>, dim3(g4), dim3(128), 0, st, p);
    merge_sparse_kernel<T, D><<<g4, 128, 0, st>>>(p);
    return cudaGetLastError();
  }
  if (dependent) return launch_dependent(merge_kernel<T, D>, dim3(grid), dim3(256), 0, st, p, wpr);
  merge_kernel<T, D><<<grid, 256, 0, st>>>(p, wpr);
  return cudaGetLastError();
}

// sparse: the partials come from a kernel that combines consecutive partitions itself
template <typename T>
cudaError_t launch_merge(const DecodeParams& p, bool dependent, bool sparse, cudaStream_t st) {
  // warps per row: enough that each walks at most ~32 slots
  const int step = p.part_step > 1 ? p.part_step : 1;
  const int slots = (p.max_parts + step - 1) / step;
  int wpr = 1;
  while (wpr < 8 && slots > 32 * wpr) wpr *= 2;
  const int rows = p.num_seqs * p.num_heads;
  const int rows_per_cta = 8 / wpr;
  const int grid = (rows + rows_per_cta - 1) / rows_per_cta;
  switch (p.head_dim) {
    case 64: return launch_merge_d<T, 64>(p, grid, wpr, dependent, sparse, st);
    case 128: return launch_merge_d<T, 128>(p, grid, wpr, dependent, sparse, st);
    case 256: return launch_merge_d<T, 256>(p, grid, wpr, dependent, sparse, st);
    default: return cudaErrorInvalidValue;
  }
}

// The arrival counters of a grouped call set to zero, launched in the chain before its
// grid: lets that grid launch at once, then waits for the kernel before it on the
// stream (the previous call on this workspace may still be counting) and clears them.
__global__ void __launch_bounds__(256) zero_counters_kernel(int* cnt, int n) {
  allow_dependents();
  grid_dependency_wait();
  for (int i = blockIdx.x * 256 + threadIdx.x; i < n; i += gridDim.x * 256) cnt[i] = 0;
}

cudaError_t launch_zero_counters(int* cnt, int n, cudaStream_t st) {
  const int grid = std::max(1, std::min((n + 255) / 256, 1184));
  return launch_dependent(zero_counters_kernel, dim3(grid), dim3(256), 0, st, cnt, n);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Heads per CTA on the CUDA-core path: the largest of 4, 2, 1 dividing the group
// (4 only up to head_dim 128, to bound registers).
int simt_heads_per_cta(int group, int head_dim) {
  if (group % 4 == 0 && head_dim <= 128) return 4;
  if (group % 2 == 0) return 2;
  return 1;
}

bool mma_eligible(int dtype, int group, int head_dim, int block_size) {
  return (dtype == PA_BF16 || dtype == PA_F16) && group % 8 == 0 && group <= 16 &&
         (head_dim == 64 || head_dim == 128 || head_dim == 256) &&
         (block_size == 16 || block_size == 32);
}

// Partitions per CTA of the per-sequence tensor-core kernels: about 2048 tokens, the
// partitions folded in registers (each keeping its own max and exp-sum), where the
// tile leaves the registers for a second set of accumulators (head_dim / 16 k-steps
// times group / 8 column tiles at most 8: the kernel's own rule); 1 otherwise.
int mma_part_step(int head_dim, int group, int partition_size) {
  if ((head_dim / 16) * (group / 8) > 8 || partition_size >= 2048) return 1;
  return 2048 / partition_size;
}

bool mma_fp8_eligible(int group, int block_size) {
  return group % 8 == 0 && group <= 16 && (block_size == 16 || block_size == 32);
}

// CTAs along the head axis of one sequence's partition grid, for the kernel that
// serves the shape: one per kv head on the tensor-core paths (all of a group's query
// heads are the columns of one tile), one per heads_per_cta query heads otherwise.
int64_t head_ctas(int cache_dtype, int num_heads, int num_kv_heads, int head_dim,
                  int block_size) {
  const int group = num_heads / num_kv_heads;
  const bool tc = cache_dtype == PA_FP8_E4M3 ? mma_fp8_eligible(group, block_size)
                                             : mma_eligible(cache_dtype, group, head_dim,
                                                            block_size);
  return tc ? num_kv_heads : num_heads / simt_heads_per_cta(group, head_dim);
}

// The partition kernels are sized to about 64 KiB of shared memory per CTA, so three
// are resident per SM; the automatic partition size aims at four waves of those.
constexpr int kAutoCtasPerSm = 3 * 4;

// The grouped form is the tensor-core kernel with (member, head) columns.
bool group_eligible(int dtype, int group, int head_dim, int block_size, int max_members) {
  return (dtype == PA_BF16 || dtype == PA_F16) && max_members >= 1 &&
         max_members * group <= 16 && (head_dim == 64 || head_dim == 128 || head_dim == 256) &&
         (block_size == 16 || block_size == 32);
}

struct GroupArgs {
  const int32_t* prefix_parts;
  const int32_t* chunk_members;
  const int32_t* chunk_parts;
  int num_chunks, max_members, max_chunk_parts, first_part;
};

int decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                const int32_t* block_tables, const int32_t* seq_lens, float scale, int block_size,
                int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                int max_blocks_per_seq, int64_t num_blocks, int max_seq_len, int partition_size,
                int dtype, int cache_dtype, float k_scale, float v_scale,
                const GroupArgs* groups, const int32_t* seq_order, void* workspace,
                size_t workspace_bytes, pa_stream_t stream);

}  // namespace

}  // namespace pa

using namespace pa;

extern "C" int pa_decode_uses_tensor_cores(int dtype, int num_heads, int num_kv_heads,
                                           int head_dim, int block_size) {
  if (num_kv_heads <= 0 || num_heads <= 0 || num_heads % num_kv_heads) return 0;
  return mma_eligible(dtype, num_heads / num_kv_heads, head_dim, block_size) ? 1 : 0;
}

extern "C" int pa_decode_partition_size(int cache_dtype, int num_seqs, int num_heads,
                                        int num_kv_heads, int head_dim, int block_size,
                                        int max_seq_len, int num_sms) {
  if (cache_dtype != PA_F32 && cache_dtype != PA_BF16 && cache_dtype != PA_F16 &&
      cache_dtype != PA_FP8_E4M3)
    return 0;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads ||
      head_dim <= 0 || max_seq_len < 0 || num_sms < 0)
    return 0;
  if (block_size != 4 && block_size != 8 && block_size != 16 && block_size != 32) return 0;
  if (num_sms == 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess || num_sms <= 0) {
      note_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidDevice);
      return 0;
    }
  }
  const int64_t rows =
      static_cast<int64_t>(num_seqs) * head_ctas(cache_dtype, num_heads, num_kv_heads,
                                                 head_dim, block_size);
  const int64_t target = static_cast<int64_t>(kAutoCtasPerSm) * num_sms;
  // Double the partition from the default while the grid keeps enough working CTAs.
  // With P > 1 partitions a sequence of uniformly spread length works in (P + 1) / 2
  // of them on average; with one partition every CTA works.  The estimate only falls
  // as the partition grows, so the first size below the target ends the search.
  int64_t best = kDefaultPartition;
  for (int64_t ps = kDefaultPartition; ps <= (int64_t{1} << 30); ps *= 2) {
    const int64_t parts = (max_seq_len + ps - 1) / ps;
    const int64_t working = parts <= 1 ? rows : rows * (parts + 1) / 2;
    if (working < target) break;
    best = ps;
    if (parts <= 1) break;
  }
  return static_cast<int>(best);
}

extern "C" size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                            int max_seq_len, int partition_size) {
  if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_seq_len < 0 || partition_size < 0)
    return 0;
  if (partition_size == 0) partition_size = kDefaultPartition;
  return ws_layout(num_seqs, num_heads, head_dim, max_seq_len, partition_size).bytes;
}

extern "C" int pa_decode_attention(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables,
                                   const int32_t* seq_lens, float scale, int block_size,
                                   int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                                   int max_blocks_per_seq, int64_t num_blocks, int max_seq_len,
                                   int partition_size, int dtype, void* workspace,
                                   size_t workspace_bytes, pa_stream_t stream) {
  return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, scale, block_size,
                     num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks,
                     max_seq_len, partition_size, dtype, dtype, 1.f, 1.f, nullptr, nullptr, workspace,
                     workspace_bytes, stream);
}

extern "C" int pa_decode_attention_fp8(void* out, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* block_tables,
                                       const int32_t* seq_lens, float scale, int block_size,
                                       int num_kv_heads, int num_seqs, int num_heads,
                                       int head_dim, int max_blocks_per_seq, int64_t num_blocks,
                                       int max_seq_len, int partition_size, int dtype,
                                       float k_scale, float v_scale, void* workspace,
                                       size_t workspace_bytes, pa_stream_t stream) {
  return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, scale, block_size,
                     num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks,
                     max_seq_len, partition_size, dtype, PA_FP8_E4M3, k_scale, v_scale, nullptr,
                     nullptr, workspace, workspace_bytes, stream);
}

extern "C" int pa_decode(const pa_decode_args_t* a) {
  if (!a || a->struct_size != sizeof(pa_decode_args_t)) return PA_ERR_INVALID_ARG;
  const bool fp8 = a->cache_dtype == PA_FP8_E4M3;
  if (!fp8 && a->cache_dtype != a->dtype) return PA_ERR_INVALID_ARG;
  GroupArgs g{};
  const GroupArgs* gp = nullptr;
  if (a->num_chunks != 0) {
    if (fp8 || a->num_chunks < 0 || a->num_chunks > 65535 || a->max_chunk_parts < 0 ||
        a->max_members < 1 || a->max_members > 16 || a->first_part < 0 ||
        !a->prefix_parts || !a->chunk_members || !a->chunk_parts)
      return PA_ERR_INVALID_ARG;
    g = GroupArgs{a->prefix_parts, a->chunk_members, a->chunk_parts, a->num_chunks,
                  a->max_members, a->max_chunk_parts, a->first_part};
    gp = &g;
  }
  return decode_impl(a->out, a->q, a->k_cache, a->v_cache, a->block_tables, a->seq_lens,
                     a->scale, a->block_size, a->num_kv_heads, a->num_seqs, a->num_heads,
                     a->head_dim, a->max_blocks_per_seq, a->num_blocks, a->max_seq_len,
                     a->partition_size, a->dtype, a->cache_dtype,
                     fp8 ? a->k_scale : 1.f, fp8 ? a->v_scale : 1.f, gp, a->seq_order,
                     a->workspace, a->workspace_bytes, a->stream);
}

extern "C" int pa_decode_attention_grouped(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* seq_lens, float scale, int block_size,
    int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
    int64_t num_blocks, int max_seq_len, int partition_size, int dtype,
    const int32_t* prefix_parts, const int32_t* chunk_members, const int32_t* chunk_parts,
    int num_chunks, int max_members, int max_chunk_parts, int first_part, void* workspace,
    size_t workspace_bytes, pa_stream_t stream) {
  if (num_chunks < 0 || max_chunk_parts < 0 || max_members < 1 || max_members > 16 ||
      first_part < 0)
    return PA_ERR_INVALID_ARG;
  if (num_chunks > 65535) return PA_ERR_INVALID_ARG;
  if (num_chunks > 0 && (!prefix_parts || !chunk_members || !chunk_parts))
    return PA_ERR_INVALID_ARG;
  const GroupArgs g{prefix_parts, chunk_members, chunk_parts, num_chunks, max_members,
                    max_chunk_parts, first_part};
  return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, scale, block_size,
                     num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq, num_blocks,
                     max_seq_len, partition_size, dtype, dtype, 1.f, 1.f, &g, nullptr, workspace,
                     workspace_bytes, stream);
}

namespace pa {
namespace {

int decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                const int32_t* block_tables, const int32_t* seq_lens, float scale, int block_size,
                int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                int max_blocks_per_seq, int64_t num_blocks, int max_seq_len, int partition_size,
                int dtype, int cache_dtype, float k_scale, float v_scale,
                const GroupArgs* groups, const int32_t* seq_order, void* workspace,
                size_t workspace_bytes, pa_stream_t stream) {
  if (dtype != PA_F32 && dtype != PA_BF16 && dtype != PA_F16) return PA_ERR_INVALID_ARG;
  const bool fp8 = cache_dtype == PA_FP8_E4M3;
  if (cache_dtype != dtype && !fp8) return PA_ERR_INVALID_ARG;
  if (fp8) {
    if (dtype == PA_F32) return PA_ERR_UNSUPPORTED;
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
      return PA_ERR_INVALID_ARG;
    if (head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  }
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads ||
      head_dim <= 0 || block_size <= 0 || max_blocks_per_seq < 0 || num_blocks <= 0 ||
      max_seq_len < 0 || partition_size < 0)
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  if (block_size != 4 && block_size != 8 && block_size != 16 && block_size != 32)
    return PA_ERR_UNSUPPORTED;
  if (partition_size == 0) partition_size = kDefaultPartition;
  if (partition_size % block_size) return PA_ERR_INVALID_ARG;
  if (num_seqs > 65535) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  const WsLayout ws = ws_layout(num_seqs, num_heads, head_dim, max_seq_len, partition_size);
  if (ws.parts > 65535) return PA_ERR_INVALID_ARG;
  if (ws.bytes > 0 && (!workspace || workspace_bytes < ws.bytes || !aligned16(workspace)))
    return PA_ERR_INVALID_ARG;

  DecodeParams p{};
  p.out = out;
  p.q = q;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.scale_log2 = scale * k_scale * 1.4426950408889634f;
  p.v_scale = v_scale;
  p.seq_order = seq_order;
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.head_dim = head_dim;
  p.block_size = block_size;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.max_seq_len = max_seq_len;
  p.partition_size = partition_size;
  p.max_parts = ws.parts;
  if (ws.bytes > 0) {
    uint8_t* base = static_cast<uint8_t*>(workspace);
    p.ws_o = reinterpret_cast<float*>(base + ws.o_off);
    p.ws_m = reinterpret_cast<float*>(base + ws.m_off);
    p.ws_l = reinterpret_cast<float*>(base + ws.l_off);
    p.ws_cnt = reinterpret_cast<int*>(base + ws.cnt_off);
  }
  p.err = device_error_word();
  if (!p.err) {
    note_cuda_error(cudaGetLastError());
    return PA_ERR_CUDA;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int group = num_heads / num_kv_heads;
  cudaError_t e;
  const bool tc = fp8 && tc_fp8_eligible(group, head_dim, block_size, num_seqs, num_kv_heads);
  bool merged = false;  // the partition grid also combines the partitions
  if (!fp8 && groups && groups->num_chunks > 0 && groups->max_chunk_parts > 0 && ws.parts > 1 &&
      group_eligible(dtype, group, head_dim, block_size, groups->max_members)) {
    // Prefix groups (only useful when sequences span several partitions): one grid of
    // the groups' shared partitions, then every sequence's own partitions
    p.prefix_parts = groups->prefix_parts;
    p.chunk_members = groups->chunk_members;
    p.chunk_parts = groups->chunk_parts;
    p.max_members = groups->max_members;
    p.num_chunks = groups->num_chunks;
    p.group_zparts = groups->max_chunk_parts < ws.parts ? groups->max_chunk_parts : ws.parts;
    // partitions below first_part belong to the groups for every sequence
    p.part_base = groups->first_part < ws.parts - 1 ? groups->first_part : ws.parts - 1;
    // the grid combines every row itself (the CTA that writes a row's last partial):
    // its counters start at zero, and no merge launch follows
    e = launch_zero_counters(p.ws_cnt, num_seqs * num_heads, st);
    if (e == cudaSuccess)
      e = dtype == PA_BF16 ? launch_decode_grouped_bf16(p, st) : launch_decode_grouped_f16(p, st);
    merged = true;
  } else if (tc) {
    e = launch_decode_tc_fp8(p, dtype, st);
  } else if (fp8 && mma_fp8_eligible(group, block_size)) {
    p.part_step = mma_part_step(head_dim, group, partition_size);
    e = launch_decode_mma_fp8(p, dtype, st);
  } else if (fp8) {
    e = launch_decode_simt_fp8(p, dtype, simt_heads_per_cta(group, head_dim), st);
  } else if (mma_eligible(dtype, group, head_dim, block_size)) {
    p.part_step = mma_part_step(head_dim, group, partition_size);
    e = dtype == PA_BF16 ? launch_decode_mma_bf16(p, st) : launch_decode_mma_f16(p, st);
  } else {
    const int gs = simt_heads_per_cta(group, head_dim);
    e = dtype == PA_F32    ? launch_decode_simt_f32(p, gs, st)
        : dtype == PA_BF16 ? launch_decode_simt_bf16(p, gs, st)
                           : launch_decode_simt_f16(p, gs, st);
  }
  if (e != cudaSuccess) {
    note_cuda_error(e);
    return PA_ERR_CUDA;
  }
  if (ws.parts > 1 && !merged) {
    e = dtype == PA_F32    ? launch_merge<float>(p, true, tc, st)
        : dtype == PA_BF16 ? launch_merge<__nv_bfloat16>(p, true, tc, st)
                           : launch_merge<__half>(p, true, tc, st);
    if (e != cudaSuccess) {
      note_cuda_error(e);
      return PA_ERR_CUDA;
    }
  }
  return PA_OK;
}

}  // namespace
}  // namespace pa
