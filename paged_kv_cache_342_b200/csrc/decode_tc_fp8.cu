// Decode partition kernel for fp8 (e4m3) caches with grouped-query heads on the 5th-
// generation tensor cores (tcgen05.mma kind::f8f6f4, accumulators in tensor memory).
// Same result as the other partition kernels: softmax(scale * q.K) V over the tokens
// of one partition, as a normalised partial (max, exp-sum, output) or the final row
// ("How PagedAttention Powers vLLM's KV Cache", hassanahmed.net, "The attention kernel
// has to read scattered blocks"; "Where it bites": grouped-query attention and a
// quantized cache stack with paging).
//
// One CTA per (sequence, kv head, partition); 6 warps:
//   warp 0     walks the block table and brings each block's K and V rows in by TMA
//              (128-byte rows, 128-byte swizzle) into stages of 128 tokens;
//   warp 1     issues the MMAs (one thread) as soon as their operands are ready:
//                S [128 tokens x NS] = K [128 x 128 dims] . Qt^T         (K-major A, B)
//                O [128 dims x 2G]  += V^T [128 dims x 128 tokens] . Pt  (MN-major A, B)
//   warps 2-5  one thread per token row: read S from tensor memory, online softmax
//              per head, write P; at the end one thread per dim row reads O.
// The codes are never converted: K and V tiles are the MMA operands as TMA lands
// them.  q (bf16: 2 terms, f16: 3 terms) is carried as exact e4m3 terms t_j of
// q * 2^qe (qe per head puts the largest |q| in [128, 256)), the terms as separate
// columns of S, summed per head.  P is split into hi = e4m3(p) and lo =
// e4m3((p - hi) * 32), again as separate columns of O: o = O_hi + O_lo / 32.  Weights
// stay in (0, 2^8] under the lazy running max, so both fit e4m3 (|p - hi| <= 8).
// Tokens past the end (or in blocks whose table entry is out of range) get -inf
// scores, and their V rows are zeroed in shared memory (0 * NaN would poison O).
// Every wait is bounded; a CTA that gives up sets PA_DEVERR_TIMEOUT, drains its
// copies and MMAs (bounded), frees its tensor memory and writes nothing.
#include <type_traits>

#include "common.cuh"
#include "decode_simt.cuh"  // checked_len, group_parts
#include "tcgen05.cuh"
#include "tensor_map.cuh"

namespace pa {
namespace {

constexpr int kTcThreads = 192;

template <typename TQ, int G, int BS, int NST>
struct TcCfg {
  static constexpr int D = 128, TM = 128, BPT = TM / BS;
  static constexpr int NQT = std::is_same<TQ, __half>::value ? 3 : 2;  // q terms
  static constexpr int NS = (G * NQT + 15) / 16 * 16;                   // S columns
  static constexpr int NO = 2 * G;                                      // O columns
  static constexpr int kTmemNeed = NO + 2 * NS;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : 128;
  static constexpr int TILE = TM * D;        // one K or V tile, bytes
  static constexpr int STAGE = 2 * TILE;     // K then V
  static constexpr int QOFF = NST * STAGE;
  static constexpr int QBYTES = (NS * 128 + 1023) / 1024 * 1024;
  static constexpr int POFF = QOFF + QBYTES;
  static constexpr int PBYTES = TM * NO;     // one P buffer
  // P as the MN-major (no swizzle) B operand: core matrices of 8 tokens x 16 bytes;
  // the NO / 16 core matrices of one 8-token group side by side (stride 128 bytes),
  // 8-token groups PK_STRIDE apart.  Byte (t, n) = (t/8) PK_STRIDE + (n/16) 128 +
  // (t%8) 16 + n%16.  Every stride is small, so the operand stays inside its buffer.
  static constexpr int PK_STRIDE = 128 * (NO / 16);
  static constexpr int SMEM = 1024 + POFF + 2 * PBYTES;
  static constexpr uint32_t IDESC_S = idesc_e4m3(128, NS, false, false);
  static constexpr uint32_t IDESC_O = idesc_e4m3(128, NO, true, true);
  static_assert(G == 8 || G == 16, "head groups of 8 or 16");
  static_assert(BS == 16 || BS == 32, "block size 16 or 32");
  static_assert(kTmemNeed <= 128, "tensor memory budget");
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

template <typename TQ, int G, int BS, int NST>
__global__ void __launch_bounds__(kTcThreads)
    decode_tc_fp8_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv) {
  grid_dependency_wait();
  using C = TcCfg<TQ, G, BS, NST>;
  constexpr int TM = C::TM, NS = C::NS, NO = C::NO, BPT = C::BPT;
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full_k[NST], bar_full_v[NST], bar_empty[NST];
  __shared__ __align__(8) uint64_t bar_s_full[2], bar_s_empty[2], bar_p_full[2], bar_p_empty[2];
  __shared__ __align__(8) uint64_t bar_drain;
  __shared__ uint32_t tmem_base_sm;
  __shared__ float sh_c[G];          // per-head logit factor (base 2, times 2^-qe)
  __shared__ float sh_red[4][G];     // per-warp maxima / sums of the softmax warpgroup

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool report = threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0;
  const int s = row_sequence(p, blockIdx.y, report);
  if (s < 0) return;
  const int kvh = blockIdx.x, h0 = kvh * G;
  const int part = p.part_base + blockIdx.z;
  const int L = checked_len(p, s, report);
  const int ps = p.partition_size;
  const int nparts = L > 0 ? (L + ps - 1) / ps : 1;
  const int own = group_parts(p, s, L);
  if (part >= nparts || part < own) return;
  const int tok_begin = part * ps;
  const int tok_end = min(L, tok_begin + ps);
  const int ntok = tok_end > tok_begin ? tok_end - tok_begin : 0;
  if (ntok == 0) {  // an empty sequence: zeros (a single partition)
    for (int i = threadIdx.x; i < G * C::D; i += kTcThreads)
      store_elem(static_cast<TQ*>(p.out) + (static_cast<int64_t>(s) * p.num_heads + h0) * C::D + i,
                 0.f);
    return;
  }
  const int ntiles = (ntok + TM - 1) / TM;
  const int nblk = (ntok + BS - 1) / BS;
  const int32_t* table =
      p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq + tok_begin / BS;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto b32 = [](const uint64_t& b) { return smem_u32(&b); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(b32(bar_full_k[i]), 1);
      mbar_init(b32(bar_full_v[i]), 1);
      mbar_init(b32(bar_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b32(bar_s_full[i]), 1);
      mbar_init(b32(bar_s_empty[i]), 128);
      mbar_init(b32(bar_p_full[i]), 128);
      mbar_init(b32(bar_p_empty[i]), 1);
    }
    mbar_init(b32(bar_drain), 1);
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sm), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_sm;
  bool aborted = false;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    int tab_base = 0;
    int32_t tab = lane < nblk ? __ldg(table + lane) : -1;
    int i = 0;
    for (; i < ntiles; ++i) {
      const int st = i % NST;
      if (i >= NST) {
        bool ok = lane == 0 ? mbar_wait_bounded(b32(bar_empty[st]), ((i / NST) - 1) & 1) : true;
        if (!__shfl_sync(FULL, ok, 0)) {
          aborted = true;
          break;
        }
      }
      const int b0 = i * BPT;
      if (b0 - tab_base >= 32) {
        tab_base += 32;
        tab = tab_base + lane < nblk ? __ldg(table + tab_base + lane) : -1;
      }
      const int b = b0 + lane;
      const int32_t blk = __shfl_sync(FULL, tab, (b0 - tab_base + lane) & 31);
      const bool in_part = lane < BPT && b < nblk;
      const bool ok = in_part && blk >= 0 && blk < p.num_blocks;
      if (in_part && !ok) set_error(p.err, PA_DEVERR_TABLE);
      const uint32_t nok = __popc(__ballot_sync(FULL, ok));
      const uint32_t kst = base + st * C::STAGE;
      if (lane == 0) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(b32(bar_full_k[st]), nok * BS * 128);
        mbar_arrive_expect_tx(b32(bar_full_v[st]), nok * BS * 128);
      }
      __syncwarp();
      if (ok) {
        const int row0 = (blk * p.num_kv_heads + kvh) * BS;
        tma_load_2d(kst + lane * BS * 128, &tmk, 0, row0, b32(bar_full_k[st]));
        tma_load_2d(kst + C::TILE + lane * BS * 128, &tmv, 0, row0, b32(bar_full_v[st]));
      }
    }
    if (aborted && lane == 0) {
      // the last NST issued tiles may still be landing: wait for them (bounded)
      for (int j = (i > NST ? i - NST : 0); j < i; ++j) {
        mbar_wait_bounded(b32(bar_full_k[j % NST]), (j / NST) & 1);
        mbar_wait_bounded(b32(bar_full_v[j % NST]), (j / NST) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issue
    named_sync(2, 160);  // q terms are in shared memory
    tc_fence_after();
    const uint32_t tO = tbase, tS0 = tbase + NO;
    const uint32_t qaddr = base + C::QOFF;
    const uint32_t paddr = base + C::POFF;
    int ns = 0, npv = 0;
    uint64_t t0 = global_timer_ns();
    uint32_t idle = 0;
    while (npv < ntiles) {
      bool prog = false;
      if (ns < ntiles) {
        const int st = ns % NST;
        bool ready = lane == 0 && mbar_test(b32(bar_full_k[st]), (ns / NST) & 1) &&
                     (ns < 2 || mbar_test(b32(bar_s_empty[ns & 1]), ((ns >> 1) - 1) & 1));
        if (__shfl_sync(FULL, ready, 0)) {
          if (lane == 0) {
            tc_fence_after();
            const uint32_t ka = base + st * C::STAGE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_e4m3(tS0 + (ns & 1) * NS, smem_desc(ka + kk * 32, 16, 1024, kSwizzle128),
                        smem_desc(qaddr + kk * 32, 16, 1024, kSwizzle128), C::IDESC_S, kk > 0);
            umma_commit(b32(bar_s_full[ns & 1]));
          }
          __syncwarp();
          ++ns;
          prog = true;
        }
      }
      if (npv < ns) {
        const int st = npv % NST;
        bool ready = lane == 0 && mbar_test(b32(bar_p_full[npv & 1]), (npv >> 1) & 1) &&
                     mbar_test(b32(bar_full_v[st]), (npv / NST) & 1);
        if (__shfl_sync(FULL, ready, 0)) {
          if (lane == 0) {
            tc_fence_after();
            const uint32_t va = base + st * C::STAGE + C::TILE;
            const uint32_t pa_ = paddr + (npv & 1) * C::PBYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_e4m3(tO, smem_desc(va + kk * 4096, 1024, 1024, kSwizzle128),
                        smem_desc(pa_ + kk * 4 * C::PK_STRIDE, C::PK_STRIDE, 128, kSwizzleNone),
                        C::IDESC_O, npv > 0 || kk > 0);
            umma_commit(b32(bar_empty[st]));
            umma_commit(b32(bar_p_empty[npv & 1]));
          }
          __syncwarp();
          ++npv;
          prog = true;
        }
      }
      // no progress for about a second: give up (decided by lane 0 for the warp)
      bool give_up = false;
      if (prog) {
        idle = 0;
        t0 = global_timer_ns();
      } else {
        __nanosleep(32);  // leave issue slots to the softmax warp on this scheduler
        if ((++idle & 255u) == 0) give_up = lane == 0 && global_timer_ns() - t0 > 1000000000ull;
      }
      if (__shfl_sync(FULL, give_up, 0)) {
        aborted = true;
        break;
      }
    }
    if (aborted && lane == 0 && ns + npv > 0) {
      umma_commit(b32(bar_drain));  // every MMA issued so far has completed
      mbar_wait_bounded(b32(bar_drain), 0);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int wt = threadIdx.x - 64;  // 0..127
    // q of the G heads as exact e4m3 terms, K-major rows (term * G + head) of 128
    // bytes with the 128-byte swizzle; each item is 8 dims of one head
#pragma unroll
    for (int it = 0; it < G / 8; ++it) {
      const int h = wt / 16 + 8 * it, c = wt % 16;
      const TQ* qp = static_cast<const TQ*>(p.q) +
                     (static_cast<int64_t>(s) * p.num_heads + h0 + h) * C::D + c * 8;
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(qp));
      float y[8];
      vec_to_float(w, y, TQ{});
      float mx = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(y[j]));
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
      // 2^qe puts the largest magnitude in [128, 256)
      int qe = mx > 0.f ? 7 - (static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127) : 0;
      qe = qe < -126 ? -126 : (qe > 126 ? 126 : qe);
      const float sc = __uint_as_float(static_cast<uint32_t>(qe + 127) << 23);
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] *= sc;
#pragma unroll
      for (int t = 0; t < C::NQT; ++t) {
        uint32_t word[2];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint16_t pr = e4m3_pair(y[2 * j], y[2 * j + 1]);
          float bhi;
          const float blo = e4m3_pair_back(pr, bhi);
          y[2 * j] -= blo;  // the remainder, exact in float32
          y[2 * j + 1] -= bhi;
          if (j & 1) word[j >> 1] |= static_cast<uint32_t>(pr) << 16;
          else word[j >> 1] = pr;
        }
        const int r = t * G + h;
        uint8_t* dst = smem + C::QOFF + (r >> 3) * 1024 + (r & 7) * 128 +
                       ((((c >> 1) ^ (r & 7)) << 4) | ((c & 1) << 3));
        *reinterpret_cast<uint2*>(dst) = make_uint2(word[0], word[1]);
      }
      if (c == 0) sh_c[h] = p.scale_log2 * __uint_as_float(static_cast<uint32_t>(127 - qe) << 23);
    }
    for (int i = (G * C::NQT) * 128 / 16 + wt; i < NS * 128 / 16; i += 128)  // padding rows
      *reinterpret_cast<uint4*>(smem + C::QOFF + i * 16) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    named_sync(2, 160);

    const int wq = warp & 3;       // tensor-memory lane quarter of this warp
    const int trow = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tO = tbase + lane_off, tS0 = tbase + NO + lane_off;
    float cf[G], m[G], l[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      cf[h] = sh_c[h];
      m[h] = -INFINITY;
      l[h] = 0.f;
    }
    int i = 0;
    for (; i < ntiles; ++i) {
      const int st = i % NST;
      const int tok = i * TM + trow;  // token within the partition
      bool valid = tok < ntok;
      if (valid) {
        const int32_t e = __ldg(table + tok / BS);
        valid = e >= 0 && e < p.num_blocks;
      }
      if (!wg_wait(b32(bar_s_full[i & 1]), (i >> 1) & 1)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      float sv[NS];
#pragma unroll
      for (int c16 = 0; c16 < NS / 16; ++c16) {
        float v16[16];
        tmem_ld16(tS0 + (i & 1) * NS + c16 * 16, v16);
#pragma unroll
        for (int j = 0; j < 16; ++j) sv[c16 * 16 + j] = v16[j];
      }
      tc_fence_before();
      mbar_arrive(b32(bar_s_empty[i & 1]));
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
          if (!wg_wait(b32(bar_p_empty[(i - 1) & 1]), ((i - 1) >> 1) & 1)) {
            aborted = true;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c16 = 0; c16 < NO / 16; ++c16) {
            float o16[16];
            tmem_ld16(tO + c16 * 16, o16);
#pragma unroll
            for (int j = 0; j < 16; ++j) o16[j] *= corr[(c16 * 16 + j) % G];
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
        const int wi = h >> 2, sh = (h & 2) ? 16 : 0;
        if (sh == 0) {
          hiw[wi] = hp;
          low[wi] = lp;
        } else {
          hiw[wi] |= static_cast<uint32_t>(hp) << 16;
          low[wi] |= static_cast<uint32_t>(lp) << 16;
        }
      }
      if (i >= 2 && !wg_wait(b32(bar_p_empty[i & 1]), ((i >> 1) - 1) & 1)) {
        aborted = true;
        break;
      }
      uint8_t* pb = smem + C::POFF + (i & 1) * C::PBYTES + (trow >> 3) * C::PK_STRIDE +
                    (trow & 7) * 16;
      if constexpr (G == 8) {
        *reinterpret_cast<uint4*>(pb) = make_uint4(hiw[0], hiw[1], low[0], low[1]);
      } else {
        *reinterpret_cast<uint4*>(pb) = make_uint4(hiw[0], hiw[1], hiw[2], hiw[3]);
        *reinterpret_cast<uint4*>(pb + 128) = make_uint4(low[0], low[1], low[2], low[3]);
      }
      // rows that carry no token: V zeroed (rows of the last block past the end are
      // landed by TMA, so wait for it first)
      if ((i + 1) * TM > ntok && !wg_wait(b32(bar_full_v[st]), (i / NST) & 1)) {
        aborted = true;
        break;
      }
      if (!valid) {
        uint4* vrow = reinterpret_cast<uint4*>(smem + st * C::STAGE + C::TILE + trow * 128);
#pragma unroll
        for (int j = 0; j < 8; ++j) vrow[j] = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(b32(bar_p_full[i & 1]));
    }

    if (!aborted) {
      const int last = ntiles - 1;
      aborted = !wg_wait(b32(bar_p_empty[last & 1]), (last >> 1) & 1);
    }
    if (!aborted) {
      tc_fence_after();
      // exp-sums over the 128 token rows
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float w = warp_sum(l[h]);
        if (lane == 0) sh_red[wq][h] = w;
      }
      named_sync(1, 128);
      float den[G];
#pragma unroll
      for (int h = 0; h < G; ++h) den[h] = sh_red[0][h] + sh_red[1][h] + sh_red[2][h] + sh_red[3][h];
      float ov[NO];
#pragma unroll
      for (int c16 = 0; c16 < NO / 16; ++c16) {
        float o16[16];
        tmem_ld16(tO + c16 * 16, o16);
#pragma unroll
        for (int j = 0; j < 16; ++j) ov[c16 * 16 + j] = o16[j];
      }
      const int d = trow;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float o = ov[h] + ov[G + h] * (1.f / 32.f);
        const float val = den[h] > 0.f ? o * (p.v_scale / den[h]) : 0.f;
        const int64_t row = static_cast<int64_t>(s) * p.num_heads + h0 + h;
        if (nparts == 1) {
          store_elem(static_cast<TQ*>(p.out) + row * C::D + d, val);
        } else {
          const int64_t prow = row * p.max_parts + part;
          p.ws_o[prow * C::D + d] = val;
          if (d == h) {
            p.ws_m[prow] = m[h];
            p.ws_l[prow] = den[h];
          }
        }
      }
    }
  }
  allow_dependents();
  if (aborted) set_error(p.err, PA_DEVERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

template <typename TQ, int G, int BS, int NST>
cudaError_t launch_tc(const DecodeParams& p, cudaStream_t st) {
  using C = TcCfg<TQ, G, BS, NST>;
  const uint64_t rows = static_cast<uint64_t>(p.num_blocks) * p.num_kv_heads * BS;
  if (rows > 0x7fffffffull) return cudaErrorInvalidValue;  // int32 row coordinates
  CUtensorMap tmk, tmv;
  if (!make_cache_tensor_map(&tmk, p.k_cache, rows, C::D, BS, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1) ||
      !make_cache_tensor_map(&tmv, p.v_cache, rows, C::D, BS, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1))
    return cudaErrorInvalidValue;
  constexpr auto kern = decode_tc_fp8_kernel<TQ, G, BS, NST>;
  cudaError_t e = ensure_smem_limit<kern>(C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_kv_heads, p.num_seqs, p.max_parts - p.part_base);
  return launch_dependent(kern, grid, dim3(kTcThreads), C::SMEM, st, p, tmk, tmv);
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

bool tc_fp8_eligible(int group, int head_dim, int block_size) {
  return head_dim == 128 && (group == 8 || group == 16) && (block_size == 16 || block_size == 32);
}

cudaError_t launch_decode_tc_fp8(const DecodeParams& p, int q_dtype, cudaStream_t st) {
  return q_dtype == PA_BF16 ? by_group<__nv_bfloat16>(p, st) : by_group<__half>(p, st);
}

}  // namespace pa
