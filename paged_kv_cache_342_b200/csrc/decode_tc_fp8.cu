// Decode partition kernel for fp8 (e4m3) caches with grouped-query heads on the 5th-
// generation tensor cores (tcgen05.mma kind::f8f6f4, accumulators in tensor memory).
// Same result as the other partition kernels: softmax(scale * q.K) V over the tokens
// of each partition, as a normalised partial (max, exp-sum, output) or the final row
// ("How PagedAttention Powers vLLM's KV Cache", hassanahmed.net, "The attention kernel
// has to read scattered blocks"; "Where it bites": grouped-query attention and a
// quantized cache stack with paging).
//
// Persistent CTAs (two per SM) each take an equal contiguous range of the flat list of
// all partitions (few (sequence, kv head) rows: the shapes where this kernel is the
// faster one), as work items (sequence, kv head, run of consecutive partitions);
// 8 warps:
//   warps 0, 3  walk the block table and bring each block's K (warp 0) and V (warp 3)
//               rows in by TMA (128-byte rows, 128-byte swizzle) into stages of 128
//               tokens; a K stage is refilled as soon as its S is computed, a V stage
//               once its p.V is, so K runs ahead and items follow each other without
//               a pipeline ramp;
//   warp 1      issues S [128 tokens x NS] = K [128 x 128 dims] . Qt^T   (K-major A, B)
//   warp 2      issues O [128 dims x 2G] += V^T [128 x 128 tokens] . Pt  (MN-major A, B)
//   warps 4-7   one thread per token row: read S from tensor memory, online softmax per
//               head, write P; a partition's output (one thread per dim row) is read
//               from tensor memory after the next partition's first tile, from the
//               other of two O accumulators, so it never stalls the pipeline, and is
//               combined with the item's earlier partitions (log-sum-exp rule); one
//               partial per item leaves by bulk copy.
// The codes are never converted: K and V tiles are the MMA operands as TMA lands
// them.  q (bf16: 2 terms, f16: 3 terms) is carried as exact e4m3 terms t_j of
// q * 2^qe (qe per head puts the largest |q| in [128, 256)), the terms as separate
// columns of S, summed per head; the next item's q is prefetched into registers and
// written to the Q operand once the current item's last S has been computed.  P is
// split into hi = e4m3(p) and lo = e4m3((p - hi) * 32), again as separate columns of O:
// o = O_hi + O_lo / 32.  Weights stay in (0, 2^8] under the lazy running max, so both
// fit e4m3 (|p - hi| <= 8).  Tokens past the end (or in blocks whose table entry is
// out of range) get -inf scores, and their V rows are zeroed in shared memory
// (0 * NaN would poison O).  Every wait is bounded; a CTA that gives up sets
// PA_DEVERR_TIMEOUT, drains its copies and MMAs (bounded), frees its tensor memory
// and writes nothing more.
#include <type_traits>

#include "common.cuh"
#include "decode_simt.cuh"  // checked_len, group_parts
#include "tcgen05.cuh"
#include "tensor_map.cuh"

namespace pa {
namespace {

constexpr int kTcThreads = 256;
constexpr int kTcCtasPerSm = 2;
constexpr int kTcMaxItems = 96;  // work items of one CTA (at most one per row)
constexpr int kTcMaxSeqs = 256;  // the split's per-row scratch (16 bytes each) in the P buffers

template <typename TQ, int G, int BS, int NST>
struct TcCfg {
  static constexpr int D = 128, TM = 128, BPT = TM / BS;
  static constexpr int NQT = std::is_same<TQ, __half>::value ? 3 : 2;  // q terms
  static constexpr int NS = (G * NQT + 15) / 16 * 16;                   // S columns
  static constexpr int NO = 2 * G;                                      // O columns
  // tensor memory: O[0], O[1] (NO columns each), then S[0], S[1] (NS each)
  static constexpr int kTmemNeed = 2 * NO + 2 * NS;
  static constexpr int kTmemCols = kTmemNeed <= 32    ? 32
                                   : kTmemNeed <= 64  ? 64
                                   : kTmemNeed <= 128 ? 128
                                                      : 256;
  static constexpr int TILE = TM * D;        // one K or V tile, bytes
  static constexpr int STAGE = 2 * TILE;     // K then V
  static constexpr int QOFF = NST * STAGE;
  static constexpr int QBYTES = (NS * 128 + 1023) / 1024 * 1024;  // the Q operand
  static constexpr int POFF = QOFF + QBYTES;
  static constexpr int PBYTES = TM * NO;     // one P buffer
  // P as the MN-major (no swizzle) B operand: core matrices of 8 tokens x 16 bytes;
  // the NO / 16 core matrices of one 8-token group side by side (stride 128 bytes),
  // 8-token groups PK_STRIDE apart.  Byte (t, n) = (t/8) PK_STRIDE + (n/16) 128 +
  // (t%8) 16 + n%16.  Every stride is small, so the operand stays inside its buffer.
  static constexpr int PK_STRIDE = 128 * (NO / 16);
  // one partition's output on its way out by bulk copy: G rows of 128 floats (or of
  // 128 output elements), then the partition's G maxima and G exp-sums
  static constexpr int SOFF = POFF + 2 * PBYTES;
  static constexpr int STBYTES = G * 512 + 2 * G * 4;
  static constexpr int SMEM = 1024 + SOFF + STBYTES;
  static_assert(2 * PBYTES >= kTcMaxSeqs * 16, "the P buffers hold the split's scratch");
  static constexpr uint32_t IDESC_S = idesc_e4m3(128, NS, false, false);
  static constexpr uint32_t IDESC_O = idesc_e4m3(128, NO, true, true);
  static_assert(G == 8 || G == 16, "head groups of 8 or 16");
  static_assert(BS == 16 || BS == 32, "block size 16 or 32");
  static_assert(kTmemNeed <= 256, "tensor memory budget");
  static_assert(NS <= 48 && NS % 16 == 0 && NO % 16 == 0, "tile widths");
};

__device__ __forceinline__ float e4m3_pair_back(uint16_t pair, float& hi) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pair),
                                                   __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  hi = f.y;
  return f.x;
}
// Two floats -> e4m3 codes (a in the low byte), round to nearest even, saturating.
__device__ __forceinline__ uint16_t e4m3_pair(float a, float b) {
  return static_cast<uint16_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// Bounded wait of one thread, then the softmax warpgroup agrees (all or none go on).
__device__ __forceinline__ bool wg_wait(uint32_t bar, uint32_t parity) {
  const bool ok = mbar_wait_bounded(bar, parity);
  return bar_red_and(1, 128, ok);
}
// Bounded wait by lane 0 of a warp, the result shared with the whole warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int lane) {
  const bool ok = lane == 0 ? mbar_wait_bounded(bar, parity) : true;
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Tokens of partition j of a sequence of length L (partition size ps).
__device__ __forceinline__ int part_tokens(int j, int ps, int L) {
  const int b = j * ps;
  return max(0, min(L, b + ps) - b);
}

// A work item: partitions [pbeg, pend) of sequence s for the query heads of kv head kvh;
// kind 1 is an empty sequence (its output is zeros), kind 2 has tiles.
struct TcItem {
  int s, kvh, L, pbeg, pend, kind;
};
// Groups of 8 fit two CTAs per SM (shared memory), so registers are held to 128 per
// thread; groups of 16 need more shared memory and run one CTA per SM.
template <typename TQ, int G, int BS, int NST>
__global__ void __launch_bounds__(kTcThreads, G == 8 ? 2 : 1)
    decode_tc_fp8_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv) {
  using C = TcCfg<TQ, G, BS, NST>;
  constexpr int TM = C::TM, NS = C::NS, NO = C::NO, BPT = C::BPT, D = C::D;
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full_k[NST], bar_full_v[NST];
  __shared__ __align__(8) uint64_t bar_k_empty[NST], bar_v_empty[NST];
  __shared__ __align__(8) uint64_t bar_s_full[2], bar_s_empty[2], bar_p_full[2], bar_p_empty[2];
  __shared__ __align__(8) uint64_t bar_q_full, bar_drain[2];
  __shared__ uint32_t tmem_base_sm;
  __shared__ float sh_c[G];          // per-head logit factor (base 2, times 2^-qe)
  __shared__ float sh_red[4][G];     // per-warp maxima of the softmax warpgroup
  __shared__ float sh_sum[4][G];     // per-warp exp-sums of the softmax warpgroup
  __shared__ float sh_den[2][G], sh_m[2][G];  // per O buffer: exp-sums and maxima
  // an item's partitions combined so far (per head): maximum and exp-sum; the factors
  // that bring the running output and the newest partition to the common maximum; at
  // the item's end, v_scale / exp-sum (0 if none)
  __shared__ float sh_run_m[G], sh_run_l[G], sh_c_old[G], sh_c_new[G], sh_fin[G];
  __shared__ TcItem sh_items[kTcMaxItems];    // this CTA's work, in order
  __shared__ int sh_nitems;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ps = p.partition_size;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto b32 = [](const uint64_t& b) { return smem_u32(&b); };

  if (threadIdx.x == 64) {  // the p.V warp has nothing else to do at the start
    for (int i = 0; i < NST; ++i) {
      mbar_init(b32(bar_full_k[i]), 1);
      mbar_init(b32(bar_full_v[i]), 1);
      mbar_init(b32(bar_k_empty[i]), 1);
      mbar_init(b32(bar_v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b32(bar_s_full[i]), 1);
      mbar_init(b32(bar_s_empty[i]), 128);
      mbar_init(b32(bar_p_full[i]), 128);
      mbar_init(b32(bar_p_empty[i]), 1);
      mbar_init(b32(bar_drain[i]), 1);
    }
    mbar_init(b32(bar_q_full), 128);
    mbar_init_fence();
  }
  if (warp == 3) {
    tmem_alloc(smem_u32(&tmem_base_sm), C::kTmemCols);
    tmem_relinquish();
  }
  // launched to overlap the end of the kernel before it on the stream: the set-up above
  // touches no global memory; from here on everything may depend on that kernel
  grid_dependency_wait();
  if (warp == 2) {
    // Balanced split: every (sequence row, kv head) contributes its partitions; the
    // flat list of all partitions (row-major) is cut into gridDim.x equal ranges and
    // this CTA takes its range as runs of consecutive partitions.  Per sequence row:
    // its sequence, length and first / count of partitions, in the P buffers (free
    // until the first tile).
    int* rs = reinterpret_cast<int*>(smem + C::POFF);
    const int S = p.num_seqs, Hkv = p.num_kv_heads;
    for (int y = lane; y < S; y += 32) {
      const bool report = blockIdx.x == 0;
      const int sq = row_sequence(p, y, report);
      int L = 0, first = 0, cnt = 0;
      if (sq >= 0) {
        L = checked_len(p, sq, report);
        const int nparts = L > 0 ? (L + ps - 1) / ps : 1;
        first = max(group_parts(p, sq, L), p.part_base);
        cnt = max(0, nparts - first);
      }
      rs[4 * y] = sq;
      rs[4 * y + 1] = L;
      rs[4 * y + 2] = first;
      rs[4 * y + 3] = cnt;
    }
    __syncwarp();
    if (lane == 0) {
      int64_t total = 0;
      for (int y = 0; y < S; ++y) total += static_cast<int64_t>(rs[4 * y + 3]) * Hkv;
      const int64_t lo = total * blockIdx.x / gridDim.x;
      const int64_t hi = total * (blockIdx.x + 1) / gridDim.x;
      int n = 0;
      int64_t at = 0;  // flat index of row y's first partition
      for (int y = 0; y < S && at < hi && n < kTcMaxItems; ++y) {
        const int cnt = rs[4 * y + 3];
        const int64_t span = static_cast<int64_t>(cnt) * Hkv;
        if (at + span > lo) {
          for (int kv = 0; kv < Hkv && n < kTcMaxItems; ++kv) {
            const int64_t b = at + static_cast<int64_t>(kv) * cnt;  // this row's first
            const int64_t from = max(b, lo), to = min(b + cnt, hi);
            if (from >= to) continue;
            TcItem it;
            it.s = rs[4 * y];
            it.kvh = kv;
            it.L = rs[4 * y + 1];
            it.pbeg = rs[4 * y + 2] + static_cast<int>(from - b);
            it.pend = rs[4 * y + 2] + static_cast<int>(to - b);
            it.kind = it.L > 0 ? 2 : 1;
            sh_items[n++] = it;
          }
        }
        at += span;
      }
      sh_nitems = n;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_sm;
  const int nitems = sh_nitems;
  bool aborted = false;
  // The merge after this kernel may be scheduled once every CTA has got here: its
  // CTAs then take only what this grid leaves free, and wait for its writes.
  allow_dependents();

  if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------------ producers
    const bool is_k = warp == 0;
    uint64_t* full = is_k ? bar_full_k : bar_full_v;
    uint64_t* empty = is_k ? bar_k_empty : bar_v_empty;
    const CUtensorMap* map = is_k ? &tmk : &tmv;
    const uint32_t half = is_k ? 0u : static_cast<uint32_t>(C::TILE);
    const uint64_t stream_policy = l2_evict_first_policy();  // K/V are read once
    int g = 0;
    for (int k = 0; k < nitems && !aborted; ++k) {
      const TcItem it = sh_items[k];
      if (it.kind != 2) continue;
      const int32_t* seq_table =
          p.block_tables + static_cast<int64_t>(it.s) * p.max_blocks_per_seq;
      for (int j = it.pbeg; j < it.pend && !aborted; ++j) {
        const int nblk = (part_tokens(j, ps, it.L) + BS - 1) / BS;
        const int32_t* table = seq_table + j * ps / BS;
        int tab_base = 0;
        int32_t tab = lane < nblk ? __ldg(table + lane) : -1;
        for (int b0 = 0; b0 < nblk; b0 += BPT, ++g) {
          const int st = g % NST;
          if (g >= NST && !warp_wait(b32(empty[st]), ((g / NST) - 1) & 1, lane)) {
            aborted = true;
            break;
          }
          if (b0 - tab_base >= 32) {
            tab_base += 32;
            tab = tab_base + lane < nblk ? __ldg(table + tab_base + lane) : -1;
          }
          const int32_t blk = __shfl_sync(FULL, tab, (b0 - tab_base + lane) & 31);
          const bool in_part = lane < BPT && b0 + lane < nblk;
          const bool ok = in_part && blk >= 0 && blk < p.num_blocks;
          if (is_k && in_part && !ok) set_error(p.err, PA_DEVERR_TABLE);
          const uint32_t nok = __popc(__ballot_sync(FULL, ok));
          if (lane == 0) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(b32(full[st]), nok * BS * 128);
          }
          __syncwarp();
          if (ok)
            tma_load_2d_hint(base + st * C::STAGE + half + lane * BS * 128, map, 0,
                             (blk * p.num_kv_heads + it.kvh) * BS, b32(full[st]), stream_policy);
        }
      }
    }
    if (aborted && lane == 0) {
      // the last NST issued tiles may still be landing: wait for them (bounded)
      for (int k = (g > NST ? g - NST : 0); k < g; ++k)
        mbar_wait_bounded(b32(full[k % NST]), (k / NST) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ S = K . Qt^T
    const uint32_t tS0 = tbase + 2 * NO;
    int g = 0, kq = 0;
    for (int k = 0; k < nitems && !aborted; ++k) {
      const TcItem it = sh_items[k];
      if (it.kind != 2) continue;
      if (!warp_wait(b32(bar_q_full), kq & 1, lane)) {  // this item's q terms
        aborted = true;
        break;
      }
      const uint32_t qaddr = base + C::QOFF;
      ++kq;
      for (int j = it.pbeg; j < it.pend && !aborted; ++j) {
        const int nt = (part_tokens(j, ps, it.L) + TM - 1) / TM;
        for (int i = 0; i < nt; ++i, ++g) {
          const int st = g % NST;
          if (!warp_wait(b32(bar_full_k[st]), (g / NST) & 1, lane) ||
              (g >= 2 && !warp_wait(b32(bar_s_empty[g & 1]), ((g >> 1) - 1) & 1, lane))) {
            aborted = true;
            break;
          }
          if (lane == 0) {
            tc_fence_after();
            const uint32_t ka = base + st * C::STAGE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_e4m3(tS0 + (g & 1) * NS, smem_desc(ka + kk * 32, 16, 1024, kSwizzle128),
                        smem_desc(qaddr + kk * 32, 16, 1024, kSwizzle128), C::IDESC_S, kk > 0);
            umma_commit(b32(bar_s_full[g & 1]));
            umma_commit(b32(bar_k_empty[st]));  // the K stage may be refilled
          }
          __syncwarp();
        }
      }
    }
    if (aborted && lane == 0 && g > 0) {
      umma_commit(b32(bar_drain[0]));  // every MMA this thread issued has completed
      mbar_wait_bounded(b32(bar_drain[0]), 0);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------------ O += V^T . Pt
    const uint32_t paddr = base + C::POFF;
    int g = 0, pc = 0;
    for (int k = 0; k < nitems && !aborted; ++k) {
      const TcItem it = sh_items[k];
      if (it.kind != 2) continue;
      for (int j = it.pbeg; j < it.pend && !aborted; ++j, ++pc) {
        const int nt = (part_tokens(j, ps, it.L) + TM - 1) / TM;
        const uint32_t tO = tbase + (pc & 1) * NO;
        for (int i = 0; i < nt; ++i, ++g) {
          const int st = g % NST;
          if (!warp_wait(b32(bar_p_full[g & 1]), (g >> 1) & 1, lane) ||
              !warp_wait(b32(bar_full_v[st]), (g / NST) & 1, lane)) {
            aborted = true;
            break;
          }
          if (lane == 0) {
            tc_fence_after();
            const uint32_t va = base + st * C::STAGE + C::TILE;
            const uint32_t pa_ = paddr + (g & 1) * C::PBYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_e4m3(tO, smem_desc(va + kk * 4096, 1024, 1024, kSwizzle128),
                        smem_desc(pa_ + kk * 4 * C::PK_STRIDE, C::PK_STRIDE, 128, kSwizzleNone),
                        C::IDESC_O, i > 0 || kk > 0);
            umma_commit(b32(bar_v_empty[st]));  // the V stage may be refilled
            umma_commit(b32(bar_p_empty[g & 1]));
          }
          __syncwarp();
        }
      }
    }
    if (aborted && lane == 0 && g > 0) {
      umma_commit(b32(bar_drain[1]));
      mbar_wait_bounded(b32(bar_drain[1]), 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ softmax warps
    const int wt = threadIdx.x - 128;  // 0..127
    const int wq = warp & 3;           // tensor-memory lane quarter of this warp
    const int trow = wq * 32 + lane;   // token row of a tile, dim row of O
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS0 = tbase + 2 * NO + lane_off;

    // q of an item: this thread's 8 dims of heads wt/16 (+ 8) as raw TQ bits
    struct QRaw {
      uint4 v[G / 8];
    };
    auto load_q = [&](const TcItem& it) {
      QRaw r;
#pragma unroll
      for (int k = 0; k < G / 8; ++k) {
        const int h = wt / 16 + 8 * k, c = wt % 16;
        r.v[k] = __ldg(reinterpret_cast<const uint4*>(
            static_cast<const TQ*>(p.q) +
            (static_cast<int64_t>(it.s) * p.num_heads + it.kvh * G + h) * D + c * 8));
      }
      return r;
    };
    // ... written into the Q operand as exact e4m3 terms: K-major rows (term * G +
    // head) of 128 bytes with the 128-byte swizzle; then released to the S warp (the
    // previous item's S MMAs have all completed by then)
    auto store_q = [&](const QRaw raw_q) {
      uint8_t* qb = smem + C::QOFF;
#pragma unroll
      for (int k = 0; k < G / 8; ++k) {
        const int h = wt / 16 + 8 * k, c = wt % 16;
        float y[8];
        vec_to_float(raw_q.v[k], y, TQ{});
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(y[e]));
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
        // 2^qe puts the largest magnitude in [128, 256)
        int qe = mx > 0.f ? 7 - (static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127) : 0;
        qe = qe < -126 ? -126 : (qe > 126 ? 126 : qe);
        const float sc = __uint_as_float(static_cast<uint32_t>(qe + 127) << 23);
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] *= sc;
#pragma unroll
        for (int t = 0; t < C::NQT; ++t) {
          uint32_t word[2];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint16_t pr = e4m3_pair(y[2 * e], y[2 * e + 1]);
            float bhi;
            const float blo = e4m3_pair_back(pr, bhi);
            y[2 * e] -= blo;  // the remainder, exact in float32
            y[2 * e + 1] -= bhi;
            if (e & 1) word[e >> 1] |= static_cast<uint32_t>(pr) << 16;
            else word[e >> 1] = pr;
          }
          const int r = t * G + h;
          *reinterpret_cast<uint2*>(qb + (r >> 3) * 1024 + (r & 7) * 128 +
                                    ((((c >> 1) ^ (r & 7)) << 4) | ((c & 1) << 3))) =
              make_uint2(word[0], word[1]);
        }
        if (c == 0) sh_c[h] = p.scale_log2 * __uint_as_float(static_cast<uint32_t>(127 - qe) << 23);
      }
      for (int k = (G * C::NQT) * 128 / 16 + wt; k < NS * 128 / 16; k += 128)  // padding rows
        *reinterpret_cast<uint4*>(qb + k * 16) = make_uint4(0, 0, 0, 0);
      fence_proxy_async_smem();
      mbar_arrive(b32(bar_q_full));
    };
    // the first item with tiles at list position >= k (nitems if none)
    auto tile_item_from = [&](int k) {
      while (k < nitems && sh_items[k].kind != 2) ++k;
      return k;
    };
    // block-table entry of this thread's token in tile i of partition j of item k
    // (-1 past the partition's end); fetched one tile ahead of its use
    auto entry = [&](int k, int j, int i) -> int32_t {
      const TcItem& it = sh_items[k];
      const int t = i * TM + trow;
      return t < part_tokens(j, ps, it.L)
                 ? __ldg(p.block_tables + static_cast<int64_t>(it.s) * p.max_blocks_per_seq +
                         (j * ps + t) / BS)
                 : -1;
    };
    // A partition's output, read from O buffer ob once its last p.V (tile g_last)
    // has landed (the partition's exp-sums and maxima are in sh_den / sh_m [ob]), is
    // combined with the item's earlier partitions by the log-sum-exp rule: per head,
    // M = max(m_run, m_j), o_run = o_run 2^(m_run - M) + o_j 2^(m_j - M), and the same
    // for the exp-sums (thread = dim row; o_run is kept, as float rows, in the staging
    // buffer the partial leaves from).  After the item's last partition the combined
    // partial goes out by bulk copies issued by one thread: into the slot of the item's
    // first partition (the item's other slots get an empty partial: exp-sum 0, maximum
    // -inf), or, for a sequence of one partition, as the output rows.
    // bits: 1 = O buffer, 2 = the item's last partition, 4 = a sequence of one partition
    struct Pending {
      int s, h0, j, pbeg, g_last, bits;
    };
    auto epilogue = [&](const Pending& e) -> bool {
      if (!wg_wait(b32(bar_p_empty[e.g_last & 1]), (e.g_last >> 1) & 1)) return false;
      tc_fence_after();
      const int ob = e.bits & 1;
      const bool first = e.j == e.pbeg, last = (e.bits & 2) != 0, single = (e.bits & 4) != 0;
      float ov[NO];
#pragma unroll
      for (int c16 = 0; c16 < NO / 16; ++c16) {
        float o16[16];
        tmem_ld16(tbase + lane_off + ob * NO + c16 * 16, o16);
#pragma unroll
        for (int k = 0; k < 16; ++k) ov[c16 * 16 + k] = o16[k];
      }
      tc_fence_before();  // O read before a later p.V overwrites it
      if (trow < G) {
        const float mj = sh_m[ob][trow], lj = sh_den[ob][trow];
        const float mo = first ? -INFINITY : sh_run_m[trow];
        const float lo = first ? 0.f : sh_run_l[trow];
        const float mn = fmaxf(mo, mj);
        const float co = exp2_safe(mo, mn), cn = exp2_safe(mj, mn);
        const float ln = lo * co + lj * cn;
        sh_c_old[trow] = co;
        sh_c_new[trow] = cn;
        sh_run_m[trow] = mn;
        sh_run_l[trow] = ln;
        if (last) sh_fin[trow] = ln > 0.f ? p.v_scale / ln : 0.f;
      }
      const int64_t row0 = static_cast<int64_t>(e.s) * p.num_heads + e.h0;
      if (!first && wt < 2 * G)  // this partition's slot holds no partial of its own
        (wt < G ? p.ws_m : p.ws_l)[ml_index(p, row0 + (wt % G), e.j)] = wt < G ? -INFINITY : 0.f;
      if (first && wt == 0) bulk_wait_read_all();  // the previous output has left staging
      named_sync(1, 128);
      uint8_t* stg = smem + C::SOFF;
      float* o_run = reinterpret_cast<float*>(stg) + trow;  // head h at o_run[h * D]
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float oj = (ov[h] + ov[G + h] * (1.f / 32.f)) * sh_c_new[h];
        const float on = first ? oj : fmaf(o_run[h * D], sh_c_old[h], oj);
        if (!last) o_run[h * D] = on;
        else if (single) store_elem(reinterpret_cast<TQ*>(stg) + h * D + trow, on * sh_fin[h]);
        else o_run[h * D] = on * sh_fin[h];
      }
      if (!last) return true;
      if (!single && trow < G) {
        float* ml = reinterpret_cast<float*>(stg + G * 512);
        ml[trow] = sh_run_m[trow];
        ml[G + trow] = sh_run_l[trow];
      }
      fence_proxy_async_smem();
      named_sync(1, 128);
      if (wt == 0) {
        const uint32_t sa = base + C::SOFF;
        if (single) {
          bulk_s2g(static_cast<TQ*>(p.out) + row0 * D, sa, G * D * sizeof(TQ));
        } else {
          // partials stay in L2 for the merge
          const uint64_t keep = l2_evict_last_policy();
          bulk_s2g_hint(p.ws_o + o_index(p, row0, e.pbeg), sa, G * 512, keep);  // G rows
          bulk_s2g_hint(p.ws_m + ml_index(p, row0, e.pbeg), sa + G * 512, G * 4, keep);
          bulk_s2g_hint(p.ws_l + ml_index(p, row0, e.pbeg), sa + G * 512 + G * 4, G * 4, keep);
        }
        bulk_commit();
      }
      return true;
    };

    Pending pend{};
    bool pending = false;
    int g = 0, pc = 0;
    QRaw raw_q{};
    int kcur = tile_item_from(0);
    int32_t ent = -1;
    if (kcur < nitems) {
      raw_q = load_q(sh_items[kcur]);
      store_q(raw_q);
      ent = entry(kcur, sh_items[kcur].pbeg, 0);
    }
    for (int k = 0; k < nitems && !aborted; ++k) {
      const TcItem cur = sh_items[k];
      if (cur.kind == 1) {  // an empty sequence: zeros
        for (int e = wt; e < G * D; e += 128)
          store_elem(static_cast<TQ*>(p.out) +
                         (static_cast<int64_t>(cur.s) * p.num_heads + cur.kvh * G) * D + e,
                     0.f);
        continue;
      }
      if (cur.kind != 2) continue;
      // this item's q terms are in the Q operand; prefetch the next item's q, which
      // replaces them once this item's last S has been computed
      const int knext = tile_item_from(k + 1);
      if (knext < nitems) raw_q = load_q(sh_items[knext]);
      named_sync(1, 128);  // sh_c of this item is complete
      float cf[G];
#pragma unroll
      for (int h = 0; h < G; ++h) cf[h] = sh_c[h];
      const int h0 = cur.kvh * G;
      const int nparts = (cur.L + ps - 1) / ps;

      for (int j = cur.pbeg; j < cur.pend && !aborted; ++j, ++pc) {
        const int ntok = part_tokens(j, ps, cur.L);
        const int nt = (ntok + TM - 1) / TM;
        const int ob = pc & 1;
        const uint32_t tO = tbase + lane_off + ob * NO;
        float m[G], l[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m[h] = -INFINITY;
          l[h] = 0.f;
        }
        for (int i = 0; i < nt; ++i, ++g) {
          const int st = g % NST;
          // the next tile: in this partition, the next one, or the next item's first
          const int32_t ent_next =
              i + 1 < nt ? entry(k, j, i + 1)
                         : (j + 1 < cur.pend ? entry(k, j + 1, 0)
                                             : (knext < nitems
                                                    ? entry(knext, sh_items[knext].pbeg, 0)
                                                    : -1));
          const bool valid = ent >= 0 && ent < p.num_blocks;
          ent = ent_next;
          if (!wg_wait(b32(bar_s_full[g & 1]), (g >> 1) & 1)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          float sv[NS];
#pragma unroll
          for (int c16 = 0; c16 < NS / 16; ++c16) {
            float v16[16];
            tmem_ld16(tS0 + (g & 1) * NS + c16 * 16, v16);
#pragma unroll
            for (int k = 0; k < 16; ++k) sv[c16 * 16 + k] = v16[k];
          }
          tc_fence_before();
          mbar_arrive(b32(bar_s_empty[g & 1]));
          float sc[G];
          bool grow = false;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float a = sv[h];
#pragma unroll
            for (int t = 1; t < C::NQT; ++t) a += sv[t * G + h];
            sc[h] = valid ? a * cf[h] : -INFINITY;
            grow |= sc[h] > m[h] + kLazyMax;
          }
          if (i == nt - 1 && j == cur.pend - 1 && knext < nitems) {
            named_sync(1, 128);  // every thread has read this item's sh_c
            store_q(raw_q);      // the last S of this item is done: the next item's q
          }
          // the running max moves only when a head's tile max passes it by more than
          // kLazyMax (base 2); until then the weights stay below 2^kLazyMax
          if (bar_red_or(1, 128, grow)) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float w = warp_max(sc[h]);
              if (lane == 0) sh_red[wq][h] = w;
            }
            named_sync(1, 128);
            bool moved = false;
            float corr[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float tmax =
                  fmaxf(fmaxf(sh_red[0][h], sh_red[1][h]), fmaxf(sh_red[2][h], sh_red[3][h]));
              const float mn = tmax > m[h] + kLazyMax ? tmax : m[h];
              corr[h] = exp2_safe(m[h], mn);
              moved |= mn != m[h];
              l[h] *= corr[h];
              m[h] = mn;
            }
            if (moved && i > 0) {
              // rescale O (thread = dim row) once the previous tile's p.V has landed
              if (!wg_wait(b32(bar_p_empty[(g - 1) & 1]), ((g - 1) >> 1) & 1)) {
                aborted = true;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int c16 = 0; c16 < NO / 16; ++c16) {
                float o16[16];
                tmem_ld16(tO + c16 * 16, o16);
#pragma unroll
                for (int k = 0; k < 16; ++k) o16[k] *= corr[(c16 * 16 + k) % G];
                tmem_st16(tO + c16 * 16, o16);
              }
            }
          }
          // weights, split into two e4m3 terms (hi, (p - hi) * 32)
          uint32_t hiw[G / 4], low[G / 4];
#pragma unroll
          for (int h = 0; h < G; h += 2) {
            const float p0 = exp2_safe(sc[h], m[h]), p1 = exp2_safe(sc[h + 1], m[h + 1]);
            l[h] += p0;
            l[h + 1] += p1;
            const uint16_t hp = e4m3_pair(p0, p1);
            float b1;
            const float b0 = e4m3_pair_back(hp, b1);
            const uint16_t lp = e4m3_pair((p0 - b0) * 32.f, (p1 - b1) * 32.f);
            const int wi = h >> 2;
            if (h & 2) {
              hiw[wi] |= static_cast<uint32_t>(hp) << 16;
              low[wi] |= static_cast<uint32_t>(lp) << 16;
            } else {
              hiw[wi] = hp;
              low[wi] = lp;
            }
          }
          if (g >= 2 && !wg_wait(b32(bar_p_empty[g & 1]), ((g >> 1) - 1) & 1)) {
            aborted = true;
            break;
          }
          uint8_t* pb = smem + C::POFF + (g & 1) * C::PBYTES + (trow >> 3) * C::PK_STRIDE +
                        (trow & 7) * 16;
          if constexpr (G == 8) {
            *reinterpret_cast<uint4*>(pb) = make_uint4(hiw[0], hiw[1], low[0], low[1]);
          } else {
            *reinterpret_cast<uint4*>(pb) = make_uint4(hiw[0], hiw[1], hiw[2], hiw[3]);
            *reinterpret_cast<uint4*>(pb + 128) = make_uint4(low[0], low[1], low[2], low[3]);
          }
          // rows that carry no token: V zeroed (rows of the last block past the end are
          // landed by TMA, so wait for it first)
          if ((i + 1) * TM > ntok && !wg_wait(b32(bar_full_v[st]), (g / NST) & 1)) {
            aborted = true;
            break;
          }
          if (!valid) {
            uint4* vrow = reinterpret_cast<uint4*>(smem + st * C::STAGE + C::TILE + trow * 128);
#pragma unroll
            for (int k = 0; k < 8; ++k) vrow[k] = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(b32(bar_p_full[g & 1]));

          if (i == 0 && pending) {
            // the previous partition's output, once this partition's first tile is
            // under way
            if (!epilogue(pend)) {
              aborted = true;
              break;
            }
            pending = false;
          }
        }
        if (aborted) break;
        // this partition's exp-sums over the 128 token rows; its output is read after
        // the next partition's first tile
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float w = warp_sum(l[h]);
          if (lane == 0) sh_sum[wq][h] = w;
        }
        named_sync(1, 128);
        if (trow < G) {
          sh_den[ob][trow] = sh_sum[0][trow] + sh_sum[1][trow] + sh_sum[2][trow] + sh_sum[3][trow];
          sh_m[ob][trow] = m[trow];
        }
        pend = Pending{cur.s, h0, j, cur.pbeg, g - 1,
                       ob | (j + 1 == cur.pend ? 2 : 0) | (nparts == 1 ? 4 : 0)};
        pending = true;
      }
    }
    if (pending && !aborted) {
      named_sync(1, 128);  // sh_den / sh_m of the last partition are visible
      if (!epilogue(pend)) aborted = true;
    }
    if (wt == 0) bulk_wait_all();  // the outputs are written before the CTA ends
  }
  if (aborted) set_error(p.err, PA_DEVERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

template <typename TQ, int G, int BS, int NST>
cudaError_t launch_tc(const DecodeParams& p, cudaStream_t st) {
  using C = TcCfg<TQ, G, BS, NST>;
  const uint64_t cache_rows = static_cast<uint64_t>(p.num_blocks) * p.num_kv_heads * BS;
  if (cache_rows > 0x7fffffffull) return cudaErrorInvalidValue;  // int32 row coordinates
  CUtensorMap tmk, tmv;
  if (!make_cache_tensor_map(&tmk, p.k_cache, cache_rows, C::D, BS,
                             CU_TENSOR_MAP_DATA_TYPE_UINT8, 1) ||
      !make_cache_tensor_map(&tmv, p.v_cache, cache_rows, C::D, BS,
                             CU_TENSOR_MAP_DATA_TYPE_UINT8, 1))
    return cudaErrorInvalidValue;
  constexpr auto kern = decode_tc_fp8_kernel<TQ, G, BS, NST>;
  cudaError_t e = ensure_smem_limit<kern>(C::SMEM);
  if (e != cudaSuccess) return e;
  // Persistent CTAs, kTcCtasPerSm per SM; the partitions are split into equal
  // contiguous ranges, one per CTA (callers check tc_fp8_eligible: few rows).
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    sms = 148;
  // CTAs resident per SM: two are planned for (one if the kernel's registers or shared
  // memory did not allow two), from the kernel's attributes and the SM's budgets
  static const int per_sm = [] {
    cudaFuncAttributes fa{};
    int d = 0, smem_sm = 0, reserved = 0, regs_sm = 0;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || cudaGetDevice(&d) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, d) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, d) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, d) != cudaSuccess)
      return 1;
    const size_t smem_cta = fa.sharedSizeBytes + C::SMEM + static_cast<size_t>(reserved);
    const int regs_cta = (fa.numRegs * 32 + 255) / 256 * 256 * (kTcThreads / 32);
    int n = static_cast<int>(static_cast<size_t>(smem_sm) / smem_cta);
    if (regs_cta > 0 && regs_sm / regs_cta < n) n = regs_sm / regs_cta;
    return n < 1 ? 1 : (n > kTcCtasPerSm ? kTcCtasPerSm : n);
  }();
  const int parts = p.max_parts - p.part_base;
  const int64_t rows = static_cast<int64_t>(p.num_seqs) * p.num_kv_heads;
  if (p.num_seqs > kTcMaxSeqs || rows > kTcMaxItems - 1 || parts < 1) return cudaErrorInvalidValue;
  const int64_t slots = static_cast<int64_t>(per_sm) * sms;
  const int64_t work = rows * parts;  // an upper bound of the partitions to split
  const int64_t ctas = work < slots ? work : slots;
  return launch_dependent(kern, dim3(static_cast<unsigned>(ctas)), dim3(kTcThreads), C::SMEM,
                          st, p, tmk, tmv);
}

constexpr int kTcStages = 3;

template <typename TQ, int G>
cudaError_t by_bs(const DecodeParams& p, cudaStream_t st) {
  switch (p.block_size) {
    case 16: return launch_tc<TQ, G, 16, kTcStages>(p, st);
    case 32: return launch_tc<TQ, G, 32, kTcStages>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename TQ>
cudaError_t by_group(const DecodeParams& p, cudaStream_t st) {
  switch (p.num_heads / p.num_kv_heads) {
    case 8: return by_bs<TQ, 8>(p, st);
    case 16: return by_bs<TQ, 16>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// Shapes the kernel serves, and where it is the faster one: few (sequence, kv head)
// rows, split evenly over every SM.  With many short rows the per-item set-up (q, the
// pipeline's first tiles, the epilogue) outweighs what the tensor cores save, and the
// mma.sync kernel, one CTA per (row, partition), was faster (GQA-8 with 512 sequences
// of 128-2048 tokens: 110 against 118 us; 1024 log-normal sequences: 186 against 218 us).
bool tc_fp8_eligible(int group, int head_dim, int block_size, int num_seqs, int num_kv_heads) {
  return head_dim == 128 && (group == 8 || group == 16) && (block_size == 16 || block_size == 32) &&
         num_seqs <= kTcMaxSeqs && static_cast<int64_t>(num_seqs) * num_kv_heads <= kTcMaxItems - 1;
}

cudaError_t launch_decode_tc_fp8(const DecodeParams& p, int q_dtype, cudaStream_t st) {
  return q_dtype == PA_BF16 ? by_group<__nv_bfloat16>(p, st) : by_group<__half>(p, st);
}

}  // namespace pa
