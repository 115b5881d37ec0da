// Tensor-core decode partition kernels for f16 caches: instantiations over
// (head_dim, block_size, 8-head column tiles) and the launch with tensor maps.
#include "decode_mma.cuh"
#include "tensor_map.cuh"

namespace pa {
namespace {

template <int D, int BS, int NT>
cudaError_t launch(const DecodeParams& p, cudaStream_t st) {
  constexpr int kStage = 2 * BS * D * 2;
  constexpr int NW = kStage <= 16384 ? 4 : (kStage <= 32768 ? 2 : 1);
  constexpr int kRaw = 65536 / (NW * kStage);
  constexpr int NST = kRaw < 2 ? 2 : (kRaw > 4 ? 4 : kRaw);
  using C = MmaCfg<__half, D, BS, NT, NW, NST>;
  const uint64_t rows = static_cast<uint64_t>(p.num_blocks) * p.num_kv_heads * BS;
  if (rows > 0x7fffffffull) return cudaErrorInvalidValue;  // int32 row coordinates
  CUtensorMap tmk, tmv;
  const bool bf16 = false;
  if (!make_cache_tensor_map(&tmk, p.k_cache, rows, D, BS, bf16) ||
      !make_cache_tensor_map(&tmv, p.v_cache, rows, D, BS, bf16))
    return cudaErrorInvalidValue;
  constexpr auto kern = decode_mma_kernel<__half, D, BS, NT, NW, NST>;
  cudaError_t e = ensure_smem_limit<kern>(C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_heads / C::kHeads, p.num_seqs, p.max_parts);
  kern<<<grid, NW * 32, C::kSmemBytes, st>>>(p, tmk, tmv);
  return cudaGetLastError();
}

template <int D, int NT>
cudaError_t by_bs(const DecodeParams& p, cudaStream_t st) {
  switch (p.block_size) {
    case 16: return launch<D, 16, NT>(p, st);
    case 32: return launch<D, 32, NT>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
cudaError_t by_nt(const DecodeParams& p, cudaStream_t st) {
  switch ((p.num_heads / p.num_kv_heads) / 8) {
    case 1: return by_bs<D, 1>(p, st);
    case 2: return by_bs<D, 2>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode_mma_f16(const DecodeParams& p, cudaStream_t st) {
  switch (p.head_dim) {
    case 64: return by_nt<64>(p, st);
    case 128: return by_nt<128>(p, st);
    case 256: return by_nt<256>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
