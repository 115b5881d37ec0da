// Tensor-core decode partition kernels for bf16 caches: instantiations over
// (head_dim, block_size, 8-head column tiles) and the launch with tensor maps.
#include "decode_mma.cuh"
#include "tensor_map.cuh"

namespace pa {
namespace {

template <int D, int BS, int NT, bool GROUP, bool CHUNK>
cudaError_t launch(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  // about 64 KiB of stages per CTA: warps with two stages each (1-4), then 2-4 stages;
  // about 16 KiB (one warp) for a grouped call, whose many short own partitions want
  // small CTAs
  constexpr int kStage = 2 * BS * D * 2;
  constexpr int kBudget = GROUP ? 16384 : 65536;
  constexpr int kW = kBudget / (2 * kStage);
  constexpr int NW = kW < 1 ? 1 : (kW > 4 ? 4 : kW);
  constexpr int kRaw = kBudget / (NW * kStage);
  constexpr int NST = kRaw < 2 ? 2 : (kRaw > 4 ? 4 : kRaw);
  using C = MmaCfg<__nv_bfloat16, D, BS, NT, NW, NST, false, !GROUP>;
  const uint64_t rows = static_cast<uint64_t>(p.num_blocks) * p.num_kv_heads * BS;
  if (rows > 0x7fffffffull) return cudaErrorInvalidValue;  // int32 row coordinates
  CUtensorMap tmk, tmv;
  const bool bf16 = true;
  const CUtensorMapDataType dt =
      bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (!make_cache_tensor_map(&tmk, p.k_cache, rows, D, BS, dt, 2) ||
      !make_cache_tensor_map(&tmv, p.v_cache, rows, D, BS, dt, 2))
    return cudaErrorInvalidValue;
  constexpr auto kern = decode_mma_kernel<__nv_bfloat16, __nv_bfloat16, D, BS, NT, NW, NST, GROUP, false, CHUNK>;
  cudaError_t e = ensure_smem_limit<kern>(C::kSmemBytes);
  if (e != cudaSuccess) return e;
  return launch_dependent(kern, grid, dim3(NW * 32), C::kSmemBytes, st, p, tmk, tmv);
}

template <int D, int NT, bool GROUP, bool CHUNK>
cudaError_t by_bs(const DecodeParams& p, dim3 grid, cudaStream_t st) {
  switch (p.block_size) {
    case 16: return launch<D, 16, NT, GROUP, CHUNK>(p, grid, st);
    case 32: return launch<D, 32, NT, GROUP, CHUNK>(p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

// several partitions per CTA (p.part_step > 1) only where the kernel folds them
// (head_dim / 16 k-steps times column tiles at most 8)
template <bool GROUP>
cudaError_t by_shape(const DecodeParams& p, int nt, dim3 grid, cudaStream_t st) {
  const bool chunk = !GROUP && p.part_step > 1;
  switch (p.head_dim * 4 + nt) {
    case 64 * 4 + 1:
      return chunk ? by_bs<64, 1, GROUP, !GROUP>(p, grid, st) : by_bs<64, 1, GROUP, false>(p, grid, st);
    case 64 * 4 + 2:
      return chunk ? by_bs<64, 2, GROUP, !GROUP>(p, grid, st) : by_bs<64, 2, GROUP, false>(p, grid, st);
    case 128 * 4 + 1:
      return chunk ? by_bs<128, 1, GROUP, !GROUP>(p, grid, st)
                   : by_bs<128, 1, GROUP, false>(p, grid, st);
    case 128 * 4 + 2:
      return chunk ? cudaErrorInvalidValue : by_bs<128, 2, GROUP, false>(p, grid, st);
    case 256 * 4 + 1:
      return chunk ? cudaErrorInvalidValue : by_bs<256, 1, GROUP, false>(p, grid, st);
    case 256 * 4 + 2:
      return chunk ? cudaErrorInvalidValue : by_bs<256, 2, GROUP, false>(p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// Per-sequence partitions: 8*NT query heads of one kv head per CTA (NT = group / 8).
cudaError_t launch_decode_mma_bf16(const DecodeParams& p, cudaStream_t st) {
  const int nt = (p.num_heads / p.num_kv_heads) / 8;
  const int step = p.part_step > 1 ? p.part_step : 1;
  dim3 grid(p.num_heads / (8 * nt), p.num_seqs, (p.max_parts - p.part_base + step - 1) / step);
  return by_shape<false>(p, nt, grid, st);
}

// A grouped call in one grid: the groups' shared partitions (p.num_chunks chunks,
// p.group_zparts partitions each), then every sequence's own partitions from
// p.part_base on; launched to overlap the kernel before it on the stream.
cudaError_t launch_decode_grouped_bf16(const DecodeParams& p, cudaStream_t st) {
  const int cols = p.max_members * (p.num_heads / p.num_kv_heads);
  const int nt = cols <= 8 ? 1 : 2;
  const int64_t n = static_cast<int64_t>(p.num_kv_heads) *
                    (static_cast<int64_t>(p.num_chunks) * p.group_zparts +
                     static_cast<int64_t>(p.num_seqs) * (p.max_parts - p.part_base));
  if (n <= 0 || n > 0x7fffffffLL) return cudaErrorInvalidValue;
  return by_shape<true>(p, nt, dim3(static_cast<unsigned>(n)), st);
}

}  // namespace pa
