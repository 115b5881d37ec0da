// CUDA-core paged decode attention (one query per sequence), partition kernel.
//
// What it computes ("How PagedAttention Powers vLLM's KV Cache", hassanahmed.net,
// "The attention kernel has to read scattered blocks"; "PagedAttention"
// attention-lab explainer, divagr.pages.dev, "Keep pages in order"): for sequence
// s, query heads h0..h0+GS-1 sharing kv head g, and the tokens of one partition,
// the running max m, exp-sum l and sum_t p_t V_t of softmax(scale * q . K_t), with
// K_t/V_t found through the block table.  One partition -> final output; several
// -> float32 partials that the merge kernel combines with log-sum-exp weights.
//
// How (B200):
//  * grid (num_heads/GS, num_seqs, max_partitions); a CTA of NW warps owns one
//    (sequence, head group, partition); partitions past the sequence exit at once.
//  * each warp streams its own blocks (local block w, w+NW, ...) through NST
//    shared-memory stages; lane 0 fetches a block's K and V runs (block_size *
//    head_dim contiguous elements each in the [blocks, kv_heads, bs, D] layout)
//    with two 1-D bulk copies (cp.async.bulk, the TMA engine) completing on the
//    stage's mbarrier, NST blocks ahead of the math.  No CTA-wide barrier in the
//    loop.  Table entries come from one coalesced load per 32 blocks held in
//    registers and handed to lane 0 with a shuffle.
//  * 8 lanes share a token row; each lane owns head_dim/8 elements (16-byte
//    vectors sub, sub+8, ...: every quarter warp reads 128 consecutive bytes of one
//    row, so shared loads are conflict-free).  A warp covers 4 rows per pass; the
//    q.k partial sums meet in 3 xor-shuffles.
//  * each 8-lane group keeps its own online-softmax state (m, l, acc) over the rows
//    it sees, per block: scores, block max, one rescale (fp8 caches: only when the
//    max moves by more than kLazyMax), then p*V.  Groups merge with shuffles at the
//    end, warps through shared memory.
//  * logits are kept in base 2 (q pre-scaled by scale*log2 e; hardware exp2).
#pragma once

#include "common.cuh"

namespace pa {

constexpr int kLanesPerRow = 8;
constexpr int kRowsPerPass = 4;

template <typename T, int D, int BS, int GS, int NW, int NST>
struct SimtCfg {
  static constexpr int kVec = ElemTraits<T>::kVec;  // cache elements per 16-byte vector
  static constexpr int kVecPerRow = D / kVec;
  static constexpr int kVecPerLane = kVecPerRow / kLanesPerRow;
  static constexpr int kEPL = kVecPerLane * kVec;  // = D / 8
  static constexpr int kPasses = BS / kRowsPerPass;
  static constexpr int kChunkBytes = BS * D * static_cast<int>(sizeof(T));
  static constexpr int kStageBytes = 2 * kChunkBytes;
  static constexpr int kStageArea = NW * NST * kStageBytes;
  static constexpr int kRedBytes = NW * GS * (D + 2) * 4;
  static constexpr int kSmemBytes =
      (kStageArea > kRedBytes ? kStageArea : kRedBytes) + NW * NST * 8;
  static_assert(kVecPerRow % kLanesPerRow == 0, "head_dim too small for 8 lanes per row");
  static_assert(BS % kRowsPerPass == 0, "block_size must be a multiple of 4");
  static_assert(kChunkBytes % 16 == 0 && (D * sizeof(T)) % 16 == 0,
                "bulk copies move multiples of 16 bytes (whole rows)");
};

// Sequence length as the kernels use it: an out-of-range value counts as 0 and is
// recorded in the error word by the (head group 0, partition 0) CTA.
__device__ __forceinline__ int checked_len(const DecodeParams& p, int s, bool report) {
  int L = __ldg(p.seq_lens + s);
  const int64_t cap = static_cast<int64_t>(p.max_blocks_per_seq) * p.block_size;
  if (L < 0 || L > p.max_seq_len || L > cap) {
    if (report) set_error(p.err, PA_DEVERR_SEQ_LEN);
    L = 0;
  }
  return L;
}

// Leading partitions of sequence s that its prefix group's kernel computes (0 when
// the call has no groups).  Never the partition holding the last token, so every
// sequence keeps at least one partition of its own and a grouped sequence always
// goes through the merge.  The per-sequence kernels and the grouped form evaluate this
// same expression, so every partition is written exactly once.
__device__ __forceinline__ int group_parts(const DecodeParams& p, int s, int L) {
  if (!p.prefix_parts || L <= 0) return 0;
  const int g = __ldg(p.prefix_parts + s);
  const int last = (L - 1) / p.partition_size;
  return g < 0 ? 0 : (g < last ? g : last);
}

// fp8 caches: the query heads h0..h0+GS-1 of sequence s as f16 pairs for this lane's
// elements (the same elements as the float path: vectors sub, sub+8, ... of VEC),
// times 2^qe per head (a bf16 q scaled so that its largest magnitude lies in
// [2^14, 2^15): every bf16 value of the row is then an f16, apart from parts below
// 2^-24 of that maximum; an f16 q as it is), and sl2 = scale * log2(e) * 2^-qe.
template <typename TQ, int D, int GS, int EPL, int NVL, int VEC>
__device__ __forceinline__ void load_q_f16(const DecodeParams& p, int s, int h0, int sub,
                                           uint32_t (&qh)[GS][EPL / 2], float (&sl2)[GS]) {
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int VQ = ElemTraits<TQ>::kVec;
  const TQ* qb = static_cast<const TQ*>(p.q) + (static_cast<int64_t>(s) * p.num_heads + h0) * D;
#pragma unroll
  for (int g = 0; g < GS; ++g) {
    float f[EPL];
#pragma unroll
    for (int k = 0; k < NVL; ++k)
#pragma unroll
      for (int u = 0; u < VEC / VQ; ++u) {
        const uint4 v =
            __ldg(reinterpret_cast<const uint4*>(qb + g * D + (sub + 8 * k) * VEC + u * VQ));
        vec_to_float(v, &f[k * VEC + u * VQ], TQ());
      }
    int qe = 0;
    if constexpr (std::is_same<TQ, __nv_bfloat16>::value) {
      float mx = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) mx = fmaxf(mx, fabsf(f[e]));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
      int ex = 0;
      if (mx > 0.f) frexpf(mx, &ex);  // mx in [2^(ex-1), 2^ex)
      qe = max(-126, min(126, 15 - ex));
    }
    const float sc = ldexpf(1.f, qe);
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e) {
      const __half2 h2 = __floats2half2_rn(f[2 * e] * sc, f[2 * e + 1] * sc);
      qh[g][e] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    sl2[g] = p.scale_log2 * ldexpf(1.f, -qe);
  }
}

// T = cache element type, TQ = query / output type (equal except for fp8 caches).
template <typename T, typename TQ, int D, int BS, int GS, int NW, int NST>
__global__ void __launch_bounds__(NW * 32) decode_simt_kernel(const DecodeParams p) {
  // launched to overlap the end of the kernel before it on the stream (typically the
  // write of the new tokens' K/V): nothing is read before that kernel is done
  grid_dependency_wait();
  using C = SimtCfg<T, D, BS, GS, NW, NST>;
  constexpr int VQ = ElemTraits<TQ>::kVec;  // query elements per 16-byte vector
  static_assert(C::kVec % VQ == 0, "a cache vector spans whole query vectors");
  constexpr int EPL = C::kEPL;
  constexpr int NVL = C::kVecPerLane;
  constexpr int VEC = C::kVec;
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 3, sub = lane & 7;
  const int s = row_sequence(p, blockIdx.y, threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0);
  const int part = p.part_base + blockIdx.z;
  if (s < 0) return;
  const int h0 = blockIdx.x * GS;
  const int kvh = h0 / (p.num_heads / p.num_kv_heads);

  const int L = checked_len(p, s, threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0);
  const int ps = p.partition_size;
  const int nparts = L > 0 ? (L + ps - 1) / ps : 1;
  const int own = group_parts(p, s, L);
  if (blockIdx.z == 0 && own < p.part_base && threadIdx.x == 0 && blockIdx.x == 0)
    set_error(p.err, PA_DEVERR_GROUP);
  if (part >= nparts || part < own) return;
  const int tok_begin = part * ps;
  const int tok_end = min(L, tok_begin + ps);
  const int nblk = tok_end > tok_begin ? (tok_end - tok_begin + BS - 1) / BS : 0;
  const int32_t* table =
      p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq + tok_begin / BS;

  uint8_t* my_stages = smem + warp * NST * C::kStageBytes;
  const uint32_t bar0 = smem_u32(smem + (C::kSmemBytes - NW * NST * 8)) + warp * NST * 8;
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NST; ++i) mbar_init(bar0 + 8 * i, 1);
    mbar_init_fence();
  }
  __syncwarp();

  // q for this lane's elements, pre-scaled into the base-2 logit domain (fp8 caches:
  // q as f16 pairs times 2^qe, the scale applied to each score instead)
  constexpr bool F8 = std::is_same<T, __nv_fp8_e4m3>::value;
  float qf[F8 ? 1 : GS][F8 ? 1 : EPL];
  uint32_t qh[F8 ? GS : 1][F8 ? EPL / 2 : 1];
  float sl2[GS];
  if constexpr (F8) {
    load_q_f16<TQ, D, GS, EPL, NVL, VEC>(p, s, h0, sub, qh, sl2);
  } else {
    const TQ* qb = static_cast<const TQ*>(p.q) + (static_cast<int64_t>(s) * p.num_heads + h0) * D;
#pragma unroll
    for (int g = 0; g < GS; ++g) {
#pragma unroll
      for (int k = 0; k < NVL; ++k) {
#pragma unroll
        for (int u = 0; u < VEC / VQ; ++u) {
          const uint4 v = __ldg(
              reinterpret_cast<const uint4*>(qb + g * D + (sub + 8 * k) * VEC + u * VQ));
          vec_to_float(v, &qf[g][k * VEC + u * VQ], TQ());
        }
      }
#pragma unroll
      for (int e = 0; e < EPL; ++e) qf[g][e] *= p.scale_log2;
      sl2[g] = 1.f;
    }
  }

  float m[GS], l[GS], acc[GS][EPL];
#pragma unroll
  for (int g = 0; g < GS; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
  }

  const int nb_w = nblk > warp ? (nblk - warp + NW - 1) / NW : 0;
  int tab_base = 0;
  int32_t tab = (lane < nb_w) ? __ldg(table + warp + lane * NW) : -1;
  uint32_t bad = 0;
  const T* kc = static_cast<const T*>(p.k_cache);
  const T* vc = static_cast<const T*>(p.v_cache);

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
        const int64_t off = (static_cast<int64_t>(blk) * p.num_kv_heads + kvh) * (BS * D);
        const uint32_t dst = smem_u32(my_stages + st * C::kStageBytes);
        // only the rows that hold tokens (the sequence's last block may be part-filled;
        // the rows past it are never read: their scores are -inf and their V is skipped)
        const int rows = min(BS, tok_end - (tok_begin + (warp + k * NW) * BS));
        const uint32_t bytes = static_cast<uint32_t>(rows) * D * sizeof(T);  // 16-byte multiple
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, 2 * bytes);
        bulk_g2s_hint(dst, kc + off, bytes, bar, stream_policy);
        bulk_g2s_hint(dst + C::kChunkBytes, vc + off, bytes, bar, stream_policy);
      } else {
        set_error(p.err, PA_DEVERR_TABLE);
        mbar_arrive(bar);
      }
    }
  };

  const int npre = nb_w < NST ? nb_w : NST;
  for (int k = 0; k < npre; ++k) issue(k);
  int issued = npre;
  int k = 0;
  bool aborted = false;
  for (; k < nb_w; ++k) {
    const int st = k % NST;
    const bool ok = mbar_wait_bounded(bar0 + 8 * st, (k / NST) & 1);
    if (!__all_sync(FULL, ok)) {
      aborted = true;
      break;
    }
    if (!((bad >> st) & 1u)) {
      const T* Ks = reinterpret_cast<const T*>(my_stages + st * C::kStageBytes);
      const T* Vs = Ks + BS * D;
      const int valid = min(BS, tok_end - (tok_begin + (warp + k * NW) * BS));
      float sc[GS][C::kPasses];
#pragma unroll
      for (int pp = 0; pp < C::kPasses; ++pp) {
        const int t = pp * kRowsPerPass + grp;
        float kf[F8 ? 1 : EPL];
        uint32_t kh[F8 ? EPL / 2 : 1];
#pragma unroll
        for (int kk = 0; kk < NVL; ++kk) {
          const uint4 v = *reinterpret_cast<const uint4*>(Ks + t * D + (sub + 8 * kk) * VEC);
          if constexpr (F8) e4m3x16_to_f16x2(v, &kh[kk * VEC / 2]);
          else vec_to_float(v, &kf[kk * VEC], T());
        }
#pragma unroll
        for (int g = 0; g < GS; ++g) {
          float d = 0.f;
          if constexpr (F8) {
#pragma unroll
            for (int e = 0; e < EPL / 2; ++e) d = fma_f16x2_f32(qh[g][e], kh[e], d);
          } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) d = fmaf(qf[g][e], kf[e], d);
          }
          d += __shfl_xor_sync(FULL, d, 1);
          d += __shfl_xor_sync(FULL, d, 2);
          d += __shfl_xor_sync(FULL, d, 4);
          sc[g][pp] = (t < valid) ? d * sl2[g] : -INFINITY;
        }
      }
      // fp8 caches keep a lazy running max (kLazyMax): the rescale runs only when some
      // group's block max passes its m by more than kLazyMax.  The others rescale on
      // every block (their kernels are bound by memory, not by instruction issue).
      bool grow = !F8;
      if constexpr (F8) {
#pragma unroll
        for (int g = 0; g < GS; ++g)
#pragma unroll
          for (int pp = 0; pp < C::kPasses; ++pp) grow |= sc[g][pp] > m[g] + kLazyMax;
        grow = __any_sync(FULL, grow);
      }
      if (grow) {
#pragma unroll
        for (int g = 0; g < GS; ++g) {
          float mn = m[g];
#pragma unroll
          for (int pp = 0; pp < C::kPasses; ++pp) mn = fmaxf(mn, sc[g][pp]);
          const float corr = exp2_safe(m[g], mn);
          l[g] *= corr;
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[g][e] *= corr;
          m[g] = mn;
        }
      }
#pragma unroll
      for (int g = 0; g < GS; ++g) {
#pragma unroll
        for (int pp = 0; pp < C::kPasses; ++pp) {
          float pw = exp2_safe(sc[g][pp], m[g]);
          if constexpr (F8) pw = __half2float(__float2half_rn(pw));  // the f16 weight of p.V
          sc[g][pp] = pw;
          l[g] += pw;
        }
      }
#pragma unroll
      for (int pp = 0; pp < C::kPasses; ++pp) {
        const int t = pp * kRowsPerPass + grp;
        if (t < valid) {
          if constexpr (F8) {
            uint32_t vh[EPL / 2];
#pragma unroll
            for (int kk = 0; kk < NVL; ++kk) {
              const uint4 v = *reinterpret_cast<const uint4*>(Vs + t * D + (sub + 8 * kk) * VEC);
              e4m3x16_to_f16x2(v, &vh[kk * VEC / 2]);
            }
#pragma unroll
            for (int g = 0; g < GS; ++g) {
              const uint16_t pw = __half_as_ushort(__float2half_rn(sc[g][pp]));  // exact
#pragma unroll
              for (int e = 0; e < EPL / 2; ++e)
                fma_f16_f16x2_f32(pw, vh[e], acc[g][2 * e], acc[g][2 * e + 1]);
            }
          } else {
            float vf[EPL];
#pragma unroll
            for (int kk = 0; kk < NVL; ++kk) {
              const uint4 v = *reinterpret_cast<const uint4*>(Vs + t * D + (sub + 8 * kk) * VEC);
              vec_to_float(v, &vf[kk * VEC], T());
            }
#pragma unroll
            for (int g = 0; g < GS; ++g) {
#pragma unroll
              for (int e = 0; e < EPL; ++e) acc[g][e] = fmaf(sc[g][pp], vf[e], acc[g][e]);
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
  if (aborted) {
    if (lane == 0) set_error(p.err, PA_DEVERR_TIMEOUT);
    // let copies already in flight land before the shared memory is reused
    for (; k < issued; ++k) mbar_wait_bounded(bar0 + 8 * (k % NST), (k / NST) & 1);
#pragma unroll
    for (int g = 0; g < GS; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
    }
  }

  // merge the four 8-lane groups of the warp
#pragma unroll
  for (int g = 0; g < GS; ++g) {
#pragma unroll
    for (int o = 8; o <= 16; o <<= 1) {
      const float mo = __shfl_xor_sync(FULL, m[g], o);
      const float lo = __shfl_xor_sync(FULL, l[g], o);
      const float mn = fmaxf(m[g], mo);
      const float a = exp2_safe(m[g], mn), b = exp2_safe(mo, mn);
      l[g] = l[g] * a + lo * b;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const float ao = __shfl_xor_sync(FULL, acc[g][e], o);
        acc[g][e] = acc[g][e] * a + ao * b;
      }
      m[g] = mn;
    }
  }

  // merge warps through shared memory (stages are idle now)
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);
  if (grp == 0) {
#pragma unroll
    for (int g = 0; g < GS; ++g) {
      float* r = red + (warp * GS + g) * (D + 2);
#pragma unroll
      for (int kk = 0; kk < NVL; ++kk)
#pragma unroll
        for (int i = 0; i < VEC; ++i) r[(sub + 8 * kk) * VEC + i] = acc[g][kk * VEC + i];
      if (sub == 0) {
        r[D] = m[g];
        r[D + 1] = l[g];
      }
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < GS * D; idx += NW * 32) {
    const int g = idx / D, d = idx - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red[(w * GS + g) * (D + 2) + D]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* r = red + (w * GS + g) * (D + 2);
      const float f = exp2_safe(r[D], M);
      num = fmaf(r[d], f, num);
      den = fmaf(r[D + 1], f, den);
    }
    const float o = den > 0.f ? num / den * p.v_scale : 0.f;
    const int64_t row = static_cast<int64_t>(s) * p.num_heads + h0 + g;
    if (nparts == 1) {
      store_elem(static_cast<TQ*>(p.out) + row * D + d, o);
    } else {
      p.ws_o[o_index(p, row, part) + d] = o;
      if (d == 0) {
        p.ws_m[ml_index(p, row, part)] = M;
        p.ws_l[ml_index(p, row, part)] = den;
      }
    }
  }
}

// Launch one instantiation (sets the dynamic shared-memory limit once).
template <typename T, typename TQ, int D, int BS, int GS, int NW, int NST>
cudaError_t launch_simt(const DecodeParams& p, cudaStream_t stream) {
  using C = SimtCfg<T, D, BS, GS, NW, NST>;
  constexpr auto kern = decode_simt_kernel<T, TQ, D, BS, GS, NW, NST>;
  cudaError_t attr = ensure_smem_limit<kern>(C::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  dim3 grid(p.num_heads / GS, p.num_seqs, p.max_parts - p.part_base);
  return launch_dependent(kern, grid, dim3(NW * 32), C::kSmemBytes, stream, p);
}

}  // namespace pa
