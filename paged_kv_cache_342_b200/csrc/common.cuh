// Shared device helpers for the sm_100a kernels: element types, 16-byte vector
// conversions, mbarrier and bulk-copy (TMA) wrappers, bounded waits, error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>
#include <utility>

#include "../../include/pa.h"

namespace pa {

// ---------------------------------------------------------------------------
// host-side launch parameters (plain data, passed by value to the kernels)
// ---------------------------------------------------------------------------
struct DecodeParams {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  float scale_log2;  // scale * log2(e): logits live in the base-2 domain
  int num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq;
  int64_t num_blocks;
  int max_seq_len, partition_size, max_parts;
  float* ws_o;  // [P, S, Hq, D]  normalised partial outputs, see o_index
  float* ws_m;  // [P, S, Hq]     partition max (base-2 logits), see ml_index
  float* ws_l;  // [P, S, Hq]     partition exp-sum
  // [S, Hq] arrival counters of the grouped form, zeroed before its grid: the CTA
  // that writes the last partial of a (sequence, kv head) combines that row
  // group's partials itself (entry s * Hq + kv head * group)
  int* ws_cnt;
  uint32_t* err;
  // prefix groups (all null / 0 for the plain call): whole partitions that a group of
  // sequences shares are computed once per group, by the tensor-core kernel's grouped
  // form
  const int32_t* prefix_parts;   // [S] shared partitions of each sequence (0 = none)
  const int32_t* chunk_members;  // [num_chunks, max_members] batch positions, -1 padded
  const int32_t* chunk_parts;    // [num_chunks] shared partitions of each chunk
  int max_members;
  // the one-grid form of a grouped call: chunks, and shared partitions per chunk, in
  // the grid before the sequences' own partitions
  int num_chunks, group_zparts;
  float v_scale;  // output multiplier (the fp8 cache's V scale; 1 otherwise)
  int part_base;  // partition index of grid z = 0 in the per-sequence kernels
  // partitions per CTA of the per-sequence tensor-core kernel (0 or 1: one): a CTA
  // folds its consecutive partitions into one partial, in the slot of the first; the
  // merge reads every part_step-th slot
  int part_step;
  // [S] or null: grid row y of the per-sequence kernels serves sequence seq_order[y]
  // (longest first, so that the long rows start early and the short ones fill the end)
  const int32_t* seq_order;
};

// Index of (query row, partition) in the partition maxima / exp-sums ws_m, ws_l:
// partition-major [P, S * Hq], so that one partition's values for a run of query
// heads are contiguous (and can be written with one bulk copy).
__device__ __forceinline__ int64_t ml_index(const DecodeParams& p, int64_t row, int part) {
  return static_cast<int64_t>(part) * p.num_seqs * p.num_heads + row;
}
// Offset of the partial output row (query row, partition) in ws_o, partition-major
// [P, S * Hq, D] like ws_m / ws_l.
__device__ __forceinline__ int64_t o_index(const DecodeParams& p, int64_t row, int part) {
  return ml_index(p, row, part) * p.head_dim;
}

// The sequence grid row y serves; -1 (reported) for an order entry out of range.
__device__ __forceinline__ int row_sequence(const DecodeParams& p, int y, bool report) {
  if (!p.seq_order) return y;
  const int s = __ldg(p.seq_order + y);
  if (s < 0 || s >= p.num_seqs) {
    if (report && p.err) atomicOr(p.err, PA_DEVERR_ORDER);
    return -1;
  }
  return s;
}

// Device address of the library's error word on the current device.
uint32_t* device_error_word();

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------
template <typename T> struct ElemTraits;
template <> struct ElemTraits<float> { static constexpr int kVec = 4; };
template <> struct ElemTraits<__nv_bfloat16> { static constexpr int kVec = 8; };
template <> struct ElemTraits<__half> { static constexpr int kVec = 8; };
template <> struct ElemTraits<__nv_fp8_e4m3> { static constexpr int kVec = 16; };

// 16 bytes of T -> floats (kVec of them)
__device__ __forceinline__ void vec_to_float(const uint4& v, float* f, float) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}
__device__ __forceinline__ void bf16x2_to_float(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}
__device__ __forceinline__ void vec_to_float(const uint4& v, float* f, __nv_bfloat16) {
  bf16x2_to_float(v.x, f[0], f[1]);
  bf16x2_to_float(v.y, f[2], f[3]);
  bf16x2_to_float(v.z, f[4], f[5]);
  bf16x2_to_float(v.w, f[6], f[7]);
}
__device__ __forceinline__ void h2_to_float(uint32_t w, float& lo, float& hi) {
  __half2 h = *reinterpret_cast<const __half2*>(&w);
  float2 f = __half22float2(h);
  lo = f.x;
  hi = f.y;
}
__device__ __forceinline__ void vec_to_float(const uint4& v, float* f, __half) {
  h2_to_float(v.x, f[0], f[1]);
  h2_to_float(v.y, f[2], f[3]);
  h2_to_float(v.z, f[4], f[5]);
  h2_to_float(v.w, f[6], f[7]);
}

// 16 e4m3 codes -> floats (CUDA's fp8 conversion; exact)
__device__ __forceinline__ void vec_to_float(const uint4& v, float* f, __nv_fp8_e4m3) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>(w[i] >> (16 * j));
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float2 ff = __half22float2(*reinterpret_cast<const __half2*>(&h));
      f[4 * i + 2 * j] = ff.x;
      f[4 * i + 2 * j + 1] = ff.y;
    }
  }
}

// e4m3 -> f16 by bit placement: with x = [c1 * c0 *] (two codes in the high bytes of
// the halves; the low bytes are ignored), a code s|eeee|mmm becomes the f16 s|0eeee|mmm0000000: exponent bias 15
// instead of 7, so the f16 is the code's value times 2^-8, exactly, for every finite
// code (subnormal codes become f16 subnormals the same way).  Integer ALU only.
__device__ __forceinline__ uint32_t e4m3_place(uint32_t x) {
  return (x & 0x80008000u) | ((x >> 1) & 0x3f803f80u);
}

// ---- mixed-precision arithmetic for fp8 caches on CUDA cores -------------------
// 16 e4m3 codes -> 8 f16x2 words (codes 2i, 2i+1 in word i, low half first), exact.
__device__ __forceinline__ void e4m3x16_to_f16x2(const uint4& v, uint32_t* h) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>(w[i] >> (16 * j)), __NV_E4M3);
      h[2 * i + j] = *reinterpret_cast<const uint32_t*>(&r);
    }
  }
}
// c + a.lo * b.lo + a.hi * b.hi with f16 multiplicands and float32 sums (each step one
// fused multiply-add of exact f16 products: fma.rn.f32.f16).
__device__ __forceinline__ float fma_f16x2_f32(uint32_t a2, uint32_t b2, float c) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
      : "+f"(c)
      : "r"(a2), "r"(b2));
  return c;
}
// c0 += p * v.lo, c1 += p * v.hi (f16 p and v, float32 sums).
__device__ __forceinline__ void fma_f16_f16x2_f32(uint16_t p, uint32_t v2, float& c0,
                                                  float& c1) {
  asm("{\n\t.reg .b16 vl, vh;\n\t"
      "mov.b32 {vl, vh}, %3;\n\t"
      "fma.rn.f32.f16 %0, %2, vl, %0;\n\t"
      "fma.rn.f32.f16 %1, %2, vh, %1;\n\t}"
      : "+f"(c0), "+f"(c1)
      : "h"(p), "r"(v2));
}

__device__ __forceinline__ void store_elem(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store_elem(__half* p, float x) { *p = __float2half_rn(x); }

// ---------------------------------------------------------------------------
// shared-memory barriers and bulk asynchronous copies (TMA engine)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
// Wait for the phase with the given parity to complete; give up after about one
// second (or 2^26 polls) and return false so the caller can record the timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; it < (1u << 26); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && global_timer_ns() - t0 > 1000000000ull) return false;
  }
  return false;
}
// Order this thread's earlier generic-proxy shared-memory accesses before later
// async-proxy (TMA) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// 1-D bulk copy global -> shared, completion counted on an mbarrier.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 2-D tiled TMA load of one box into shared memory, completion on an mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// bulk_g2s with an L2 cache policy
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// L2 eviction policies (createpolicy): streamed K/V go first, small results last
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// tma_load_2d with an L2 cache policy
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, int x,
                                                 int y, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

// a float store with an L2 cache policy
__device__ __forceinline__ void st_hint(float* dst, float v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(dst), "f"(v), "l"(policy)
               : "memory");
}

__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Online softmax with a lazy running max: the max m that the weights are taken against
// moves only when a new logit passes it by more than this (base 2), so weights stay
// below 2^kLazyMax and most blocks skip the rescale of the accumulators.
constexpr float kLazyMax = 8.f;

// exp2 of a base-2 logit difference, a - m <= kLazyMax in every use, by the hardware's
// approximate base-2 exponential (PTX ex2.approx.ftz.f32, relative error about 2^-22).
// Results below 2^-126 flush to zero: such a weight next to the largest weight (at
// least 1) changes no float sum.  -inf - -inf (an empty state) gives 0.
__device__ __forceinline__ float exp2_safe(float a, float m) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(a - m));
  return (m == -INFINITY) ? 0.f : y;
}

// Record a failing CUDA call for pa_last_cuda_error (thread-local text).
void note_cuda_error(cudaError_t e);

// Raise a kernel's dynamic shared-memory limit once per device.  The kernel is a
// template argument so every instantiation keeps its own per-device flags.
// Programmatic dependent launch (sm_90+): a kernel launched with launch_dependent()
// may be scheduled while the kernel before it on the stream is finishing, once that
// kernel's CTAs have called allow_dependents() (or exited); its CTAs then block in
// grid_dependency_wait(), their first statement, until that kernel has completed and
// its writes are visible, so nothing is ever read early, whatever kernel precedes.
// What overlaps is the launch and CTA start-up.  Both are no-ops for kernels launched
// the ordinary way.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <auto Kern>
cudaError_t ensure_smem_limit(int bytes) {
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
  return e;
}

}  // namespace pa
