// Tensor-core paged decode attention for grouped-query head groups (partition
// kernel).  Same result as the CUDA-core kernel; used when 8 or 16 query heads
// share one kv head, so that scores and p.V form dense tiles ("How PagedAttention
// Powers vLLM's KV Cache", hassanahmed.net, "Where it bites": grouped-query
// attention stacks with paging; "The attention kernel has to read scattered
// blocks": the kernel walks the block table and gathers K/V block by block).
//
// Per block of BS tokens of one kv head (BS = 16 or 32):
//   S^T [tokens x heads] = K [tokens x D] . Q^T [D x heads]    mma m16n8k16, A = K
//   online softmax per head (column) in float32, base-2 logits
//   O^T [D x heads]     += V^T [D x tokens] . P^T [tokens x heads]   A = V^T
// K/V blocks arrive by tensor-map TMA (cp.async.bulk.tensor.2d, 64-element x BS-row
// boxes with the 128-byte swizzle, so the 8-row ldmatrix reads hit 8 different bank
// groups) into NST stages per warp, completing on the stage mbarrier.  A and B
// operands are bf16 (or f16), accumulators float32.  The score fragment (C layout)
// becomes the B operand of p.V through one movmatrix.trans per 8x8 quarter.
// Tokens past the sequence end get -inf scores, and their V rows are zeroed in
// shared memory first (0 * NaN would otherwise poison the tile).
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "decode_simt.cuh"  // checked_len

namespace pa {

template <typename T> struct MmaOps;

template <> struct MmaOps<__nv_bfloat16> {
  static __device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4],
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};

template <> struct MmaOps<__half> {
  static __device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4],
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// Four e4m3 codes (bytes 0..3 of w) -> f16x2 (codes 0,1) and f16x2 (codes 2,3), exact,
// by the hardware convert.
__device__ __forceinline__ void e4m3x4_to_f16x2x2_cvt(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const __half2_raw l = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xffffu),
                                                   __NV_E4M3);
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16),
                                                   __NV_E4M3);
  lo = *reinterpret_cast<const uint32_t*>(&l);
  hi = *reinterpret_cast<const uint32_t*>(&h);
}
// Codes (byte0, byte2) -> f16x2 `even`, (byte1, byte3) -> f16x2 `odd`, each value the
// code's times 2^-8 (e4m3_place).
// e4m3_place reads codes from the high byte of each 16-bit half: bytes 1 and 3 already
// sit there, bytes 0 and 2 get there by one shift.
__device__ __forceinline__ void e4m3_pairs_to_f16x2_bits(uint32_t w, uint32_t& even,
                                                         uint32_t& odd) {
  even = e4m3_place(w << 8);
  odd = e4m3_place(w);
}

// FP8: the cache holds e4m3 codes; TMA lands them as 128-element x BS-row slabs and
// the MMA operands are loaded straight from them with ldmatrix (a pair of codes is
// one 16-bit ldmatrix element) and converted to f16 in registers, exactly:
//   - K (A of S^T = K.Q^T): a thread holds 4 consecutive dims of one token; the
//     k-order of each 16-dim step is permuted (dims 4t..4t+1 and 4t+2..4t+3 play
//     k = 2t..2t+1 and 2t+8..2t+9), and Q^T's B fragments use the same permutation;
//   - V (A of O^T += V^T.P^T): the transposing ldmatrix gives a thread 2 tokens x 2
//     dims; even dims form rows 0-7 of the m16 tile, odd dims rows 8-15, and the
//     epilogue puts the dims back in order.
// Conversions: K codes through the hardware e4m3x2 -> f16x2 convert; V codes by
// bit placement (sign to bit 15, the 7 magnitude bits to bits 13..7 of the f16),
// which is the code's value times 2^-8 for every finite code (normal and subnormal
// alike), the 2^8 going into v_scale.  The split keeps both the conversion unit and
// the integer ALU busy: converting K by bit placement as well made the kernel ALU
// bound (294 us against 254 us on the long-context GQA shape).  Codes 0x7F / 0xFF (NaN) are not special-cased
// on that path; a cache holds them only for NaN inputs.
template <typename T, int D, int BS, int NT, int NW, int NST, bool FP8 = false, bool PAD = true>
struct MmaCfg {
  static constexpr int kHalves = D / 64;         // 128-byte column slabs per 16-bit row
  static constexpr int kSlabBytes = BS * 128;    // one slab of one tile
  static constexpr int kTileBytes = kHalves * kSlabBytes;  // 16-bit tile = BS * D * 2
  static constexpr int kF8Slabs = D / 128;       // 128-byte slabs per fp8 row
  static constexpr int kF8Tile = BS * D;         // fp8 tile bytes
  static constexpr int kStageBytes = FP8 ? 2 * kF8Tile : 2 * kTileBytes;  // K + V as stored
  static constexpr int kTT = BS / 16;            // 16-token row tiles per block
  static constexpr int kKS = D / 16;             // k-steps of q.K / m-tiles of V^T
  static constexpr int kHeads = 8 * NT;
  static constexpr int kStageArea = NW * NST * kStageBytes;
  static constexpr int kRedBytes = NW * kHeads * (D + 2) * 4;
  // dynamic shared memory from its 1024-aligned base: the stages (the warps' partial
  // results reuse them at the end), the copy barriers, then the CTA's small per-column
  // arrays (8 + NW arrays of kHeads 4-byte words and one flag word); PAD reserves 1024
  // bytes in front for aligning a base that may not be aligned
  static constexpr int kAreaBytes = kStageArea > kRedBytes ? kStageArea : kRedBytes;
  static constexpr int kBarOff = kAreaBytes;
  static constexpr int kSmallOff = kBarOff + NW * NST * 8;
  static constexpr int kSmallBytes = ((8 + NW) * kHeads + 1) * 4;
  static constexpr int kSmemBytes = (PAD ? 1024 : 0) + kSmallOff + kSmallBytes;
  static_assert(sizeof(T) == 2, "tensor-core path computes in 16-bit types");
  static_assert(BS % 16 == 0 && kSlabBytes % 1024 == 0, "slabs must stay 1024-byte aligned");
  static_assert(!FP8 || D % 128 == 0, "fp8 tiles are whole 128-byte slabs");
};

// q (TQ pair) -> MMA operand pair (T): exact when the types agree
template <typename T, typename TQ>
__device__ __forceinline__ uint32_t q_pair(const TQ* qp) {
  const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(qp));
  if constexpr (std::is_same<T, TQ>::value) {
    return w;
  } else {
    float lo, hi;
    if constexpr (std::is_same<TQ, __nv_bfloat16>::value) bf16x2_to_float(w, lo, hi);
    else h2_to_float(w, lo, hi);
    return MmaOps<T>::pack(lo, hi);
  }
}

// byte offset of (row r, 16-byte chunk c of the full row) inside a tile stored as
// D/64 slabs of [BS rows][128 bytes] with the 128-byte swizzle (chunk ^= row % 8)
template <int BS>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * (BS * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// One warp combines the partials of query row `row` (sequence s, one head) into its
// output by the merge rule: M = max m_j, w_j = l_j 2^(m_j - M), out = sum w_j o_j /
// sum w_j, over the slots j in [0, a) and [b, n) (eight in flight, in increasing j,
// the same arithmetic as the merge kernel).  Slot own_part (-1: none) is this CTA's
// own partial, taken from shared memory (own_o, own_m, own_l); the others come from
// other CTAs of the grid: read from L2 (ld.global.cg) unless L1 holds lines fetched
// after an acquire of the row's counter (L1 = true).
template <typename TQ, int D, bool L1>
__device__ __forceinline__ void combine_row(const DecodeParams& p, int row, int a, int b, int n,
                                            int lane, int own_part, const float* own_o,
                                            float own_m, float own_l) {
  constexpr int DPL = D / 32, U = 8;
  const int ns = a + (n > b ? n - b : 0);
  float acc[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) acc[j] = 0.f;
  float den = 0.f, M = -INFINITY;
  for (int i = 0; i < ns; i += U) {
    float mv[U], lv[U], o[U][DPL];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = i + u;
      const int part = k < a ? k : b + (k - a);
      if (k < ns && part == own_part) {
        mv[u] = own_m;
        lv[u] = own_l;
#pragma unroll
        for (int j = 0; j < DPL; ++j) o[u][j] = own_o[lane * DPL + j];
      } else if (k < ns) {
        const float* src = p.ws_o + o_index(p, row, part) + lane * DPL;
        if constexpr (L1) {
          mv[u] = __ldca(p.ws_m + ml_index(p, row, part));
          lv[u] = __ldca(p.ws_l + ml_index(p, row, part));
        } else {
          mv[u] = __ldcg(p.ws_m + ml_index(p, row, part));
          lv[u] = __ldcg(p.ws_l + ml_index(p, row, part));
        }
        if constexpr (DPL % 4 == 0) {
#pragma unroll
          for (int j = 0; j < DPL; j += 4) {
            const float4* q4 = reinterpret_cast<const float4*>(src + j);
            const float4 v = L1 ? __ldca(q4) : __ldcg(q4);
            o[u][j] = v.x;
            o[u][j + 1] = v.y;
            o[u][j + 2] = v.z;
            o[u][j + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < DPL; j += 2) {
            const float2* q2 = reinterpret_cast<const float2*>(src + j);
            const float2 v = L1 ? __ldca(q2) : __ldcg(q2);
            o[u][j] = v.x;
            o[u][j + 1] = v.y;
          }
        }
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
  TQ* out = static_cast<TQ*>(p.out) + static_cast<int64_t>(row) * D + lane * DPL;
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int j = 0; j < DPL; ++j) store_elem(out + j, acc[j] * inv);
}

// Arrival counters and the partials they guard (device scope).
__device__ __forceinline__ int atomic_add_acq_rel_gpu(int* addr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;"
               : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* addr) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void prefetch_l1(const void* addr) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(addr));
}

// Grouped form, after a CTA has stored its partials: it counts them on the arrival
// counter of each (sequence, kv head) it wrote (entry s * Hq + kv head * G), and the
// CTA whose count completes a counter combines that sequence's G heads itself, so
// no merge launch follows the grid.  A (sequence, kv head) expects one partial per
// partition the call writes for it: the group's below a = group_parts(s), then its
// own from b = max(a, part_base) to its last, n - 1.  col_n / col_a / col_b hold n, a
// and b for a column that counts (its first head), col_n 0 for the others.  The count
// is one acquire-release atomic by the counting thread after a block barrier: it
// publishes every thread's partial stores before it, and the CTA that completes the
// count sees the other CTAs' partials after it (read from L2 after a second barrier).
// Called by every thread of the CTA.
template <typename TQ, int D, int NW, int H>
__device__ __forceinline__ void finish_rows(const DecodeParams& p, const int* col_row,
                                            const int* col_n, const int* col_a,
                                            const int* col_b, int* fin, int G) {
  __syncthreads();  // the CTA's partial stores are issued
  const int c = static_cast<int>(threadIdx.x);
  if (c < H) {
    const int n = col_n[c], b = col_b[c];
    const int expect = col_a[c] + (n > b ? n - b : 0);
    fin[c] = n > 0 && atomic_add_acq_rel_gpu(p.ws_cnt + col_row[c], 1) == expect - 1;
  }
  __syncthreads();
  const int warp = c >> 5, lane = c & 31;
  int k = 0;  // finished rows, dealt to the warps in turn
  for (int c2 = 0; c2 < H; ++c2) {
    if (!fin[c2]) continue;
    for (int j = 0; j < G; ++j, ++k)
      if (k % NW == warp)
        combine_row<TQ, D, false>(p, col_row[c2] + j, col_a[c2], col_b[c2], col_n[c2], lane,
                                  -1, nullptr, 0.f, 0.f);
  }
}

// GROUP = false: one CTA per (sequence, 8*NT query heads of one kv head, partition).
// GROUP = true : a grouped call in one flat grid of two kinds of work.  First the
//   prefix groups' shared partitions, one CTA per (kv head, chunk of a group, shared
//   partition) with kv head fastest: the tile's columns are (member, head) pairs,
//   member = column / group, and the partition's blocks - identical for every member -
//   are read once for all of them.  Then every sequence's own partitions, one CTA per
//   (kv head, grid row - longest first when an order is given -, partition from
//   part_base on), the columns the group's query heads of that kv head.  So the long
//   shared partitions start first, the short own ones fill the end, and neither kind
//   has a last wave of its own.
// T = MMA operand type, TQ = query / output type, FP8 = e4m3 cache converted to T,
// CHUNK = several partitions per CTA (per-sequence form, p.part_step of them).
template <typename T, typename TQ, int D, int BS, int NT, int NW, int NST, bool GROUP,
          bool FP8, bool CHUNK = false>
__global__ void __launch_bounds__(NW * 32)
    decode_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
  // launched to overlap the end of the kernel before it on the stream (typically the
  // write of the new tokens' K/V): nothing is read before that kernel is done
  grid_dependency_wait();
  // the grouped form's one-warp CTAs keep no padding (one more CTA fits on an SM)
  using C = MmaCfg<T, D, BS, NT, NW, NST, FP8, !GROUP>;
  using Ops = MmaOps<T>;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int TT = C::kTT, KS = C::kKS;
  // Several partitions per CTA (per-sequence form): each keeps its own running max and
  // exp-sum per warp; a finished partition is folded into the warp's running result by
  // the log-sum-exp rule, which takes a second set of accumulators - registers the
  // small tiles have to spare
  constexpr bool kChunked = CHUNK && !GROUP && KS * NT <= 8;
  static_assert(!CHUNK || kChunked, "several partitions per CTA need a small tile");

  // All of the CTA's shared memory is dynamic (no static arrays): with nothing in
  // front of it, the window's dynamic part starts 1024-byte aligned, as the 128-byte
  // swizzle atoms need, and the grouped form relies on that (checked: a CTA that
  // finds it otherwise reports PA_DEVERR_SMEM and does nothing)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  if constexpr (!GROUP) {
  } else if (base != raw) {
    if (threadIdx.x == 0) set_error(p.err, PA_DEVERR_SMEM);
    return;
  }
  uint8_t* smem = smem_raw + (base - raw);
  constexpr int H = C::kHeads;
  int* const small = reinterpret_cast<int*>(smem + C::kSmallOff);
  int* const col_row = small;       // q / out row (sequence * Hq + head) of each column
  int* const col_ok = small + H;    // the column's result is written by this CTA
  // grouped form: partitions of the column's sequence (n), the group's (a) and where
  // its own start (b), set on the column that counts the sequence's partials
  int* const col_n = small + 2 * H;
  int* const col_a = small + 3 * H;
  int* const col_b = small + 4 * H;
  float* const col_m = reinterpret_cast<float*>(small + 5 * H);  // epilogue: max,
  float* const col_l = reinterpret_cast<float*>(small + 6 * H);  // exp-sum per column
  int* const fin = small + 7 * H;   // grouped form: this CTA merges the column's rows
  float* const col_w = reinterpret_cast<float*>(small + 8 * H);  // [NW][H] warp weights
  int* const sh_pre = small + (8 + NW) * H;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3;  // fragment row group / thread in group
  const int G = p.num_heads / p.num_kv_heads;
  const int ps = p.partition_size;
  int kvh, part, nparts, tok_begin, tok_end, table_seq;
  bool own_row = false;  // grouped form: a sequence's own partition, one of several
  if constexpr (!GROUP) {
    const int s =
        row_sequence(p, blockIdx.y, threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0);
    if (s < 0) return;
    const int h0 = blockIdx.x * C::kHeads;
    // a CTA runs `step` consecutive partitions (one chunk) of the sequence
    const int step = kChunked && p.part_step > 1 ? p.part_step : 1;
    part = p.part_base + blockIdx.z * step;
    kvh = h0 / G;
    const int L = checked_len(p, s, threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0);
    nparts = L > 0 ? (L + ps - 1) / ps : 1;
    const int own = group_parts(p, s, L);
    if (blockIdx.z == 0 && own < p.part_base && threadIdx.x == 0 && blockIdx.x == 0)
      set_error(p.err, PA_DEVERR_GROUP);
    if (part >= nparts || part < own) return;
    tok_begin = part * ps;
    tok_end = min(L, min(nparts, part + step) * ps);
    // one chunk covering the whole sequence writes the output rows themselves
    if (part == 0 && nparts <= step) nparts = 1;
    table_seq = s;
    if (threadIdx.x < C::kHeads) {
      col_row[threadIdx.x] = s * p.num_heads + h0 + threadIdx.x;
      col_ok[threadIdx.x] = 1;
    }
  } else {
    int chunk = 0;
    int b = blockIdx.x;
    const int n_group = p.num_kv_heads * p.num_chunks * p.group_zparts;
    kvh = b % p.num_kv_heads;
    const bool own_item = b >= n_group;
    if (!own_item) {
      b /= p.num_kv_heads;
      chunk = b % p.num_chunks;
      part = b / p.num_chunks;
    } else {
      // a sequence's own partition: as the per-sequence kernel, heads of kv head kvh
      b = (b - n_group) / p.num_kv_heads;
      const int y = b % p.num_seqs, z = b / p.num_seqs;
      const bool report = threadIdx.x == 0 && kvh == 0 && z == 0;
      const int s = row_sequence(p, y, report);
      if (s < 0) return;
      part = p.part_base + z;
      const int L = checked_len(p, s, report);
      nparts = L > 0 ? (L + ps - 1) / ps : 1;
      const int own = group_parts(p, s, L);
      if (report && own < p.part_base) set_error(p.err, PA_DEVERR_GROUP);
      if (part >= nparts || part < own) return;
      own_row = nparts > 1;
      tok_begin = part * ps;
      tok_end = min(L, tok_begin + ps);
      table_seq = s;
      const int c = static_cast<int>(threadIdx.x);
      if (c < C::kHeads) {
        col_row[c] = c < G ? s * p.num_heads + kvh * G + c : -1;
        col_ok[c] = c < G ? 1 : 0;
        col_n[c] = c == 0 ? nparts : 0;
        col_a[c] = own;
        col_b[c] = own > p.part_base ? own : p.part_base;
      }
    }
    if (!own_item) {
      if (part >= __ldg(p.chunk_parts + chunk)) return;
      nparts = 2;  // a grouped partition is always one of several: write partials
      tok_begin = part * ps;
      tok_end = tok_begin + ps;
      if (threadIdx.x < C::kHeads) {
        const int c = threadIdx.x, mi = c / G;
        const int m = mi < p.max_members ? __ldg(p.chunk_members + chunk * p.max_members + mi) : -1;
        const bool member = m >= 0 && m < p.num_seqs;
        col_row[c] = member ? m * p.num_heads + kvh * G + (c - mi * G) : -1;
        const int Lm = member ? checked_len(p, m, false) : 0;
        const int gm = member ? group_parts(p, m, Lm) : 0;
        col_ok[c] = member && part < gm;
        col_n[c] = col_ok[c] && c == mi * G ? (Lm + ps - 1) / ps : 0;
        col_a[c] = gm;
        col_b[c] = gm > p.part_base ? gm : p.part_base;
      }
      __syncthreads();
      // blocks come from the table of the first member that owns this partition
      table_seq = -1;
      for (int c = 0; c < C::kHeads; ++c)
        if (col_ok[c]) {
          table_seq = col_row[c] / p.num_heads;
          break;
        }
      if (table_seq < 0) return;  // no member needs this partition
    }
  }
  __syncthreads();
  const int nblk = tok_end > tok_begin ? (tok_end - tok_begin + BS - 1) / BS : 0;
  const int32_t* table =
      p.block_tables + static_cast<int64_t>(table_seq) * p.max_blocks_per_seq + tok_begin / BS;

  const uint32_t stage0 = base + warp * NST * C::kStageBytes;
  const uint32_t bar0 = base + C::kBarOff + warp * NST * 8;
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NST; ++i) mbar_init(bar0 + 8 * i, 1);
    mbar_init_fence();
  }
  __syncwarp();

  // Q^T as B fragments: qb[nt][ks][0] = q[column nt*8+g8][16ks + 2t4 .. +1], [1] = +8
  // dims (FP8: dims 16ks + 4t4 .. +1 and +2 .. +3, the K operand's permutation); a
  // column with no member gets zeros (its result is never written)
  uint32_t qb[NT][KS][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int row = col_row[nt * 8 + g8];
    const TQ* qp0 = static_cast<const TQ*>(p.q) + static_cast<int64_t>(row < 0 ? 0 : row) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const TQ* qp = qp0 + ks * 16 + (FP8 ? 4 * t4 : 2 * t4);
      qb[nt][ks][0] = row < 0 ? 0u : q_pair<T, TQ>(qp);
      qb[nt][ks][1] = row < 0 ? 0u : q_pair<T, TQ>(qp + (FP8 ? 2 : 8));
    }
  }

  // per thread: heads nt*8 + 2t4 + {0,1}
  float m[NT][2], l[NT][2];
  float oacc[KS][NT][4];
  auto reset = [&]() {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) oacc[mt][nt][i] = 0.f;
    }
  };
  reset();
  // chunked form: the warp's finished partitions, combined (max, exp-sum, output)
  constexpr int RN = kChunked ? NT : 1, RK = kChunked ? KS : 1;
  float mr[RN][2], lr[RN][2], ar[RK][RN][4];
#pragma unroll
  for (int nt = 0; nt < RN; ++nt) {
    mr[nt][0] = mr[nt][1] = -INFINITY;
    lr[nt][0] = lr[nt][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < RK; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) ar[mt][nt][i] = 0.f;
  }
  int cur_part = -1;  // the partition the warp's (m, l, oacc) belong to
  int cur_end = 0;    // ... and its end, in tokens from tok_begin
  // M = max(mr, m), result = result * 2^(mr - M) + partition * 2^(m - M), per column
  auto fold = [&]() {
    if constexpr (kChunked) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float mn = fmaxf(mr[nt][j], m[nt][j]);
          const float co = exp2_safe(mr[nt][j], mn), cn = exp2_safe(m[nt][j], mn);
          lr[nt][j] = fmaf(lr[nt][j], co, l[nt][j] * cn);
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            ar[mt][nt][j] = fmaf(ar[mt][nt][j], co, oacc[mt][nt][j] * cn);
            ar[mt][nt][2 + j] = fmaf(ar[mt][nt][2 + j], co, oacc[mt][nt][2 + j] * cn);
          }
          mr[nt][j] = mn;
        }
      reset();
    }
  };

  const int nb_w = nblk > warp ? (nblk - warp + NW - 1) / NW : 0;
  int tab_base = 0;
  int32_t tab = (lane < nb_w) ? __ldg(table + warp + lane * NW) : -1;
  uint32_t bad = 0;

  const uint64_t stream_policy = l2_evict_first_policy();  // K/V are read once
  auto issue = [&](int k) {
    if (k - tab_base >= 32) {
      tab_base += 32;
      const int kk = tab_base + lane;
      tab = (kk < nb_w) ? __ldg(table + warp + kk * NW) : -1;
    }
    const int32_t blk = __shfl_sync(FULL, tab, k - tab_base);
    const bool ok = blk >= 0 && blk < p.num_blocks;
    const int st = k % NST;
    bad = ok ? (bad & ~(1u << st)) : (bad | (1u << st));
    if (lane == 0) {
      const uint32_t bar = bar0 + 8 * st;
      if (ok) {
        const int row0 = (blk * p.num_kv_heads + kvh) * BS;
        const uint32_t dst = stage0 + st * C::kStageBytes;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, C::kStageBytes);
        if constexpr (FP8) {
#pragma unroll
          for (int h = 0; h < C::kF8Slabs; ++h) {
            tma_load_2d_hint(dst + h * C::kSlabBytes, &tmk, 128 * h, row0, bar, stream_policy);
            tma_load_2d_hint(dst + C::kF8Tile + h * C::kSlabBytes, &tmv, 128 * h, row0, bar,
                             stream_policy);
          }
        } else {
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) {
            tma_load_2d_hint(dst + h * C::kSlabBytes, &tmk, 64 * h, row0, bar, stream_policy);
            tma_load_2d_hint(dst + C::kTileBytes + h * C::kSlabBytes, &tmv, 64 * h, row0, bar,
                             stream_policy);
          }
        }
      } else {
        set_error(p.err, PA_DEVERR_TABLE);
        mbar_arrive(bar);
      }
    }
  };

  const int npre = nb_w < NST ? nb_w : NST;
  for (int k = 0; k < npre; ++k) issue(k);
  // Grouped form, a sequence's own partition: when every other partial of its
  // (sequence, kv head) is stored already (the counter, read with acquire, is one
  // short of complete), this CTA combines the rows at its end without counting; the
  // other partials' lines are fetched into L1 while the blocks stream.  Otherwise it
  // counts at its end like every other CTA.
  bool pre = false;
  if constexpr (GROUP) {
    if (own_row) {  // the same for the whole CTA
      if (threadIdx.x == 0) {
        const int n = col_n[0], b = col_b[0];
        const int expect = col_a[0] + (n > b ? n - b : 0);
        *sh_pre = ld_acquire_gpu(p.ws_cnt + col_row[0]) == expect - 1;
      }
      __syncthreads();
      pre = *sh_pre;
      if (pre && warp == 0) {
        // 128-byte lines: D / 32 of each partial output row, one each for m and l
        const int a = col_a[0], b = col_b[0], n = col_n[0];
        const int others = a + (n > b ? n - b : 0) - 1;
        const int per = D / 32 + 2, total = G * others * per;
        if (total <= 8 * 32) {
          for (int i = lane; i < total; i += 32) {
            // slot list [0, a) then [b, n); this CTA's own partition (list index
            // a + part - b) is skipped
            const int line = i % per, t = i / per, r = t % G, k2 = t / G;
            const int k = k2 < a + (part - b) ? k2 : k2 + 1;
            const int j = k < a ? k : b + (k - a);
            const int row = col_row[0] + r;
            const float* addr = line < D / 32 ? p.ws_o + o_index(p, row, j) + line * 32
                                : line == D / 32 ? p.ws_m + ml_index(p, row, j)
                                                 : p.ws_l + ml_index(p, row, j);
            prefetch_l1(addr);
          }
        }
      }
    }
  }
  int issued = npre;
  int k = 0;
  bool aborted = false;
  for (; k < nb_w; ++k) {
    const int st = k % NST;
    if constexpr (kChunked) {
      // a block of the next partition: fold the finished one into the running result
      const int off = (warp + k * NW) * BS;
      if (off >= cur_end) {
        if (cur_part >= 0) fold();
        cur_part = part + off / ps;
        cur_end = (cur_part - part + 1) * ps;
      }
    }
    const bool ok = mbar_wait_bounded(bar0 + 8 * st, (k / NST) & 1);
    if (!__all_sync(FULL, ok)) {
      aborted = true;
      break;
    }
    if (!((bad >> st) & 1u)) {
      const uint32_t kt = stage0 + st * C::kStageBytes;
      const uint32_t vt = kt + (FP8 ? C::kF8Tile : C::kTileBytes);
      const int valid = min(BS, tok_end - (tok_begin + (warp + k * NW) * BS));
      if (!FP8 && valid < BS) {
        // zero the V rows past the end (0 * NaN would poison the tile; the FP8 path's
        // V conversion never makes a NaN): 16 bytes per lane per step
        uint8_t* vg = smem + (vt - base);
        const int nchunks = (BS - valid) * (D / 8);
        for (int i = lane; i < nchunks; i += 32) {
          const int r = valid + i / (D / 8), c = i % (D / 8);
          *reinterpret_cast<uint4*>(vg + swz<BS>(r, c)) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      // ---- S^T = K Q^T --------------------------------------------------
      float sacc[TT][NT][4];
#pragma unroll
      for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) sacc[tt][nt][i] = 0.f;
      {
        const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
          const int r = tt * 16 + (mi & 1) * 8 + ri;
          if constexpr (FP8) {
            // one ldmatrix.x4 = 16 tokens x 32 dims of codes = two k-steps
#pragma unroll
            for (int kp = 0; kp < KS / 2; ++kp) {
              uint32_t w[4];
              ldsm_x4(kt + swz<BS>(r, 2 * kp + (mi >> 1)), w);
              uint32_t a0[4], a1[4];
              e4m3x4_to_f16x2x2_cvt(w[0], a0[0], a0[2]);
              e4m3x4_to_f16x2x2_cvt(w[1], a0[1], a0[3]);
              e4m3x4_to_f16x2x2_cvt(w[2], a1[0], a1[2]);
              e4m3x4_to_f16x2x2_cvt(w[3], a1[1], a1[3]);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                Ops::mma(sacc[tt][nt], a0, qb[nt][2 * kp][0], qb[nt][2 * kp][1]);
                Ops::mma(sacc[tt][nt], a1, qb[nt][2 * kp + 1][0], qb[nt][2 * kp + 1][1]);
              }
            }
          } else {
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              uint32_t a[4];
              ldsm_x4(kt + swz<BS>(r, 2 * ks + (mi >> 1)), a);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                Ops::mma(sacc[tt][nt], a, qb[nt][ks][0], qb[nt][ks][1]);
            }
          }
        }
      }
      // ---- online softmax per head column ----------------------------------
      // The running max moves only when some column's block max passes it by more
      // than kLazyMax (base 2): until then the weights exp2(s - m) stay below
      // 2^kLazyMax, which P's 16-bit type holds with its full precision, and the
      // accumulators and sums need no rescale for this block.
      float bmax[NT][2];
      bool grow = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float mx = -INFINITY;
#pragma unroll
          for (int tt = 0; tt < TT; ++tt)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const int tok = tt * 16 + g8 + 8 * r;
              const float sv = tok < valid ? sacc[tt][nt][2 * r + j] * p.scale_log2 : -INFINITY;
              sacc[tt][nt][2 * r + j] = sv;
              mx = fmaxf(mx, sv);
            }
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16));
          bmax[nt][j] = mx;
          grow |= mx > m[nt][j] + kLazyMax;
        }
      }
      if (__any_sync(FULL, grow)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float mn = fmaxf(m[nt][j], bmax[nt][j]);
            const float corr = exp2_safe(m[nt][j], mn);
            m[nt][j] = mn;
            l[nt][j] *= corr;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
              oacc[mt][nt][j] *= corr;
              oacc[mt][nt][2 + j] *= corr;
            }
          }
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float ls = 0.f;
#pragma unroll
          for (int tt = 0; tt < TT; ++tt)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const float pv = exp2_safe(sacc[tt][nt][2 * r + j], m[nt][j]);
              sacc[tt][nt][2 * r + j] = pv;
              ls += pv;
            }
          l[nt][j] += ls;
        }
      }
      // ---- P^T as B fragments (movmatrix.trans of each 8x8 quarter) ----------
      uint32_t pb[TT][NT][2];
#pragma unroll
      for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          pb[tt][nt][0] = movmatrix_trans(Ops::pack(sacc[tt][nt][0], sacc[tt][nt][1]));
          pb[tt][nt][1] = movmatrix_trans(Ops::pack(sacc[tt][nt][2], sacc[tt][nt][3]));
        }
      // ---- O^T += V^T P^T -------------------------------------------------
      {
        const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
          if constexpr (FP8) {
            // one transposing ldmatrix.x4 = 16 tokens x 32 dims of codes = two m-tiles
            const int r = tt * 16 + (mi & 1) * 8 + ri;
#pragma unroll
            for (int mp = 0; mp < KS / 2; ++mp) {
              uint32_t w[4];
              ldsm_x4_trans(vt + swz<BS>(r, 2 * mp + (mi >> 1)), w);
              uint32_t a0[4], a1[4];
              e4m3_pairs_to_f16x2_bits(w[0], a0[0], a0[1]);
              e4m3_pairs_to_f16x2_bits(w[1], a0[2], a0[3]);
              e4m3_pairs_to_f16x2_bits(w[2], a1[0], a1[1]);
              e4m3_pairs_to_f16x2_bits(w[3], a1[2], a1[3]);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                Ops::mma(oacc[2 * mp][nt], a0, pb[tt][nt][0], pb[tt][nt][1]);
                Ops::mma(oacc[2 * mp + 1][nt], a1, pb[tt][nt][0], pb[tt][nt][1]);
              }
            }
          } else {
            const int r = tt * 16 + (mi >> 1) * 8 + ri;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
              uint32_t a[4];
              ldsm_x4_trans(vt + swz<BS>(r, 2 * mt + (mi & 1)), a);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                Ops::mma(oacc[mt][nt], a, pb[tt][nt][0], pb[tt][nt][1]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (issued < nb_w) {
      issue(issued);
      ++issued;
    }
  }
  allow_dependents();  // the merge may launch now; it waits for this grid's writes
  if constexpr (kChunked) {
    if (cur_part >= 0) fold();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        m[nt][j] = mr[nt][j];
        l[nt][j] = lr[nt][j];
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          oacc[mt][nt][j] = ar[mt][nt][j];
          oacc[mt][nt][2 + j] = ar[mt][nt][2 + j];
        }
      }
  }
  if (aborted) {
    if (lane == 0) set_error(p.err, PA_DEVERR_TIMEOUT);
    for (; k < issued; ++k) mbar_wait_bounded(bar0 + 8 * (k % NST), (k / NST) & 1);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = -INFINITY;
  }

  // exp-sums: add the partial sums of the 8 lanes that share a head column
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float x = l[nt][j];
      x += __shfl_xor_sync(FULL, x, 4);
      x += __shfl_xor_sync(FULL, x, 8);
      x += __shfl_xor_sync(FULL, x, 16);
      l[nt][j] = aborted ? 0.f : x;
    }

  // merge warps through shared memory
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float* r = red + (warp * C::kHeads + nt * 8 + 2 * t4 + j) * (D + 2);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        // FP8: rows g8 / g8 + 8 of an m-tile hold dims 2g8 / 2g8 + 1
        r[mt * 16 + (FP8 ? 2 * g8 : g8)] = oacc[mt][nt][j];
        r[mt * 16 + (FP8 ? 2 * g8 + 1 : g8 + 8)] = oacc[mt][nt][2 + j];
      }
      if (g8 == 0) {
        r[D] = m[nt][j];
        r[D + 1] = l[nt][j];
      }
    }
  __syncthreads();
  // per head column, once: the max M, the exp-sum and each warp's weight
  // exp2(m_w - M) * v_scale / sum, so that an output element is NW fused multiply-adds
  if (threadIdx.x < C::kHeads) {
    const int hh = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red[(w * C::kHeads + hh) * (D + 2) + D]);
    float f[NW], den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* r = red + (w * C::kHeads + hh) * (D + 2);
      f[w] = exp2_safe(r[D], M);
      den = fmaf(r[D + 1], f[w], den);
    }
    // FP8: the V operands carry the code values times 2^-8
    const float sc = den > 0.f ? (FP8 ? p.v_scale * 256.f : p.v_scale) / den : 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) col_w[w * H + hh] = f[w] * sc;
    col_m[hh] = M;
    col_l[hh] = den;
  }
  __syncthreads();
  const uint64_t keep_policy = l2_evict_last_policy();
  for (int idx = threadIdx.x; idx < C::kHeads * D; idx += NW * 32) {
    const int hh = idx / D, d = idx - hh * D;
    if (!col_ok[hh]) continue;
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w)
      o = fmaf(red[(w * C::kHeads + hh) * (D + 2) + d], col_w[w * H + hh], o);
    const float den = col_l[hh];
    if (!(den > 0.f)) o = 0.f;
    const int64_t row = col_row[hh];
    if (nparts == 1) {
      store_elem(static_cast<TQ*>(p.out) + row * D + d, o);
    } else if (pre) {
      red[hh * (D + 2) + d] = o;  // this CTA's own partial, combined below (read in place)
    } else {
      st_hint(p.ws_o + o_index(p, row, part) + d, o, keep_policy);  // L2, for the merge
      if (d == 0) {
        st_hint(p.ws_m + ml_index(p, row, part), col_m[hh], keep_policy);
        st_hint(p.ws_l + ml_index(p, row, part), den, keep_policy);
      }
    }
  }
  if constexpr (GROUP) {
    if (pre) {
      __syncthreads();  // the own partial is in shared memory
      for (int r = warp; r < G; r += NW)
        combine_row<TQ, D, true>(p, col_row[0] + r, col_a[0], col_b[0], col_n[0], lane, part,
                                 red + r * (D + 2), col_m[r], col_l[r]);
    } else if (nparts > 1) {
      finish_rows<TQ, D, NW, C::kHeads>(p, col_row, col_n, col_a, col_b, fin, G);
    }
  }
}

}  // namespace pa
