// CUDA-core decode partition kernels for f32 caches: the (head_dim, block_size,
// heads-per-CTA) instantiations and the choice of warps / pipeline stages.
#include "decode_simt.cuh"

namespace pa {
namespace {

// Stage = one block's K and V runs.  Up to 4 warps; 2-4 stages per warp sized so
// a CTA holds about 64 KiB of stages (three CTAs per SM at head_dim 128, block 16).
template <int D, int BS, int GS>
cudaError_t launch_auto(const DecodeParams& p, cudaStream_t st) {
  constexpr int kStage = 2 * BS * D * static_cast<int>(sizeof(float));
  constexpr int NW = kStage <= 16384 ? 4 : (kStage <= 32768 ? 2 : 1);
  constexpr int kRaw = 65536 / (NW * kStage);
  constexpr int NST = kRaw < 2 ? 2 : (kRaw > 4 ? 4 : kRaw);
  return launch_simt<float, D, BS, GS, NW, NST>(p, st);
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

cudaError_t launch_decode_simt_f32(const DecodeParams& p, int gs, cudaStream_t st) {
  switch (p.head_dim) {
    case 64: return by_gs<64>(p, gs, st);
    case 128: return by_gs<128>(p, gs, st);
    case 256: return by_gs<256>(p, gs, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
