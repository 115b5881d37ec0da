// CUDA-core decode partition kernels for f16 caches: the (head_dim, block_size,
// heads-per-CTA) instantiations and the choice of warps / pipeline stages.
#include "decode_simt.cuh"

namespace pa {
namespace {

// Stage = one block's K and V runs.  kBudget bytes of stages per CTA: as many warps
// as fit with two stages each (1-4), then 2-4 stages per warp.
template <int D, int BS, int GS, int kBudget>
cudaError_t launch_budget(const DecodeParams& p, cudaStream_t st) {
  constexpr int kStage = 2 * BS * D * static_cast<int>(sizeof(__half));
  constexpr int kW = kBudget / (2 * kStage);
  constexpr int NW = kW < 1 ? 1 : (kW > 4 ? 4 : kW);
  constexpr int kRaw = kBudget / (NW * kStage);
  constexpr int NST = kRaw < 2 ? 2 : (kRaw > 4 ? 4 : kRaw);
  return launch_simt<__half, __half, D, BS, GS, NW, NST>(p, st);
}

// About 64 KiB per CTA (three CTAs per SM) for whole sequences and long partitions.
// When prefix groups cover every partition but each sequence's last one, the CTAs
// here read only those short tails (tens to a few hundred tokens): then 32 KiB CTAs,
// twice as many per SM, overlap their start-up and epilogue better.
template <int D, int BS, int GS>
cudaError_t launch_auto(const DecodeParams& p, cudaStream_t st) {
  if (p.part_base > 0 && p.max_parts - p.part_base == 1)
    return launch_budget<D, BS, GS, 32768>(p, st);
  return launch_budget<D, BS, GS, 65536>(p, st);
}

template <int D, int GS>
cudaError_t by_bs(const DecodeParams& p, cudaStream_t st) {
  switch (p.block_size) {
    case 4: return launch_auto<D, 4, GS>(p, st);
    case 8: return launch_auto<D, 8, GS>(p, st);
    case 16: return launch_auto<D, 16, GS>(p, st);
    case 32: return launch_auto<D, 32, GS>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
cudaError_t by_gs(const DecodeParams& p, int gs, cudaStream_t st) {
  switch (gs) {
    case 1: return by_bs<D, 1>(p, st);
    case 2: return by_bs<D, 2>(p, st);
    case 4:
      if constexpr (D <= 128) return by_bs<D, 4>(p, st);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode_simt_f16(const DecodeParams& p, int gs, cudaStream_t st) {
  switch (p.head_dim) {
    case 64: return by_gs<64>(p, gs, st);
    case 128: return by_gs<128>(p, gs, st);
    case 256: return by_gs<256>(p, gs, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
