// Tensor-core decode partition kernels for fp8 (e4m3) caches with grouped-query
// heads: the codes arrive by TMA, ldmatrix loads them as MMA fragments and they are
// converted exactly to f16 in registers; q (bf16 or f16) becomes f16 operands, P is
// f16, accumulators float32.
#include "decode_mma.cuh"
#include "tensor_map.cuh"

namespace pa {
namespace {

template <typename TQ, int D, int BS, int NT, bool CHUNK>
cudaError_t launch(const DecodeParams& p, cudaStream_t st) {
  // about 32 KiB of fp8 stages per CTA: warps with two stages each (1-4), then 2-4
  // stages; small CTAs, so that several per SM hide the conversion work
  constexpr int kStage = 2 * BS * D;      // fp8 K + V
  constexpr int kBudget = 32768;
  constexpr int kW = kBudget / (2 * kStage);
  constexpr int NW = kW < 1 ? 1 : (kW > 4 ? 4 : kW);
  constexpr int kRaw = kBudget / (NW * kStage);
  constexpr int NST = kRaw < 2 ? 2 : (kRaw > 4 ? 4 : kRaw);
  using C = MmaCfg<__half, D, BS, NT, NW, NST, true>;
  const uint64_t rows = static_cast<uint64_t>(p.num_blocks) * p.num_kv_heads * BS;
  if (rows > 0x7fffffffull) return cudaErrorInvalidValue;  // int32 row coordinates
  CUtensorMap tmk, tmv;
  if (!make_cache_tensor_map(&tmk, p.k_cache, rows, D, BS, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1) ||
      !make_cache_tensor_map(&tmv, p.v_cache, rows, D, BS, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1))
    return cudaErrorInvalidValue;
  constexpr auto kern = decode_mma_kernel<__half, TQ, D, BS, NT, NW, NST, false, true, CHUNK>;
  cudaError_t e = ensure_smem_limit<kern>(C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int step = p.part_step > 1 ? p.part_step : 1;
  dim3 grid(p.num_heads / C::kHeads, p.num_seqs, (p.max_parts - p.part_base + step - 1) / step);
  return launch_dependent(kern, grid, dim3(NW * 32), C::kSmemBytes, st, p, tmk, tmv);
}

template <typename TQ, int D, int NT, bool CHUNK>
cudaError_t by_bs(const DecodeParams& p, cudaStream_t st) {
  switch (p.block_size) {
    case 16: return launch<TQ, D, 16, NT, CHUNK>(p, st);
    case 32: return launch<TQ, D, 32, NT, CHUNK>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename TQ>
cudaError_t by_shape(const DecodeParams& p, cudaStream_t st) {
  const int nt = (p.num_heads / p.num_kv_heads) / 8;
  // several partitions per CTA (p.part_step > 1) only where the kernel folds them
  const bool chunk = p.part_step > 1;
  switch (p.head_dim * 4 + nt) {
    case 128 * 4 + 1: return chunk ? by_bs<TQ, 128, 1, true>(p, st) : by_bs<TQ, 128, 1, false>(p, st);
    case 128 * 4 + 2: return chunk ? cudaErrorInvalidValue : by_bs<TQ, 128, 2, false>(p, st);
    case 256 * 4 + 1: return chunk ? cudaErrorInvalidValue : by_bs<TQ, 256, 1, false>(p, st);
    case 256 * 4 + 2: return chunk ? cudaErrorInvalidValue : by_bs<TQ, 256, 2, false>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode_mma_fp8(const DecodeParams& p, int q_dtype, cudaStream_t st) {
  return q_dtype == PA_BF16 ? by_shape<__nv_bfloat16>(p, st) : by_shape<__half>(p, st);
}

}  // namespace pa
