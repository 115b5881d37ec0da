// CUDA-core decode partition kernels for fp8 (e4m3) caches read with bf16 or f16
// queries / outputs.  The K scale is folded into the logit scale and the V scale into
// the output; head_dim 128 or 256 (one 16-byte vector = 16 elements per lane).
#include "decode_simt.cuh"

namespace pa {
namespace {

template <typename TQ, int D, int BS, int GS>
cudaError_t launch_auto(const DecodeParams& p, cudaStream_t st) {
  constexpr int kStage = 2 * BS * D;  // one byte per element
  constexpr int kBudget = 32768;  // small stages: more CTAs per SM hide the conversion latency
  constexpr int kW = kBudget / (2 * kStage);
  constexpr int NW = kW < 1 ? 1 : (kW > 4 ? 4 : kW);
  constexpr int kRaw = kBudget / (NW * kStage);
  constexpr int NST = kRaw < 2 ? 2 : (kRaw > 4 ? 4 : kRaw);
  return launch_simt<__nv_fp8_e4m3, TQ, D, BS, GS, NW, NST>(p, st);
}

template <typename TQ, int D, int GS>
cudaError_t by_bs(const DecodeParams& p, cudaStream_t st) {
  switch (p.block_size) {
    case 4: return launch_auto<TQ, D, 4, GS>(p, st);
    case 8: return launch_auto<TQ, D, 8, GS>(p, st);
    case 16: return launch_auto<TQ, D, 16, GS>(p, st);
    case 32: return launch_auto<TQ, D, 32, GS>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename TQ, int D>
cudaError_t by_gs(const DecodeParams& p, int gs, cudaStream_t st) {
  switch (gs) {
    case 1: return by_bs<TQ, D, 1>(p, st);
    case 2: return by_bs<TQ, D, 2>(p, st);
    case 4:
      if constexpr (D <= 128) return by_bs<TQ, D, 4>(p, st);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

template <typename TQ>
cudaError_t by_dim(const DecodeParams& p, int gs, cudaStream_t st) {
  switch (p.head_dim) {
    case 128: return by_gs<TQ, 128>(p, gs, st);
    case 256: return by_gs<TQ, 256>(p, gs, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode_simt_fp8(const DecodeParams& p, int q_dtype, int gs, cudaStream_t st) {
  return q_dtype == PA_BF16 ? by_dim<__nv_bfloat16>(p, gs, st) : by_dim<__half>(p, gs, st);
}

}  // namespace pa
