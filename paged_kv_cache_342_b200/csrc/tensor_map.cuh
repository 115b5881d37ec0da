// Tensor maps for the TMA loads of the tensor-core decode kernel.  The encoder is
// the driver's cuTensorMapEncodeTiled, reached through the runtime's driver
// entry-point query so the library does not link libcuda directly.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace pa {

// A cache tensor [rows = num_blocks*num_kv_heads*block_size, head_dim] of
// elem_bytes-byte elements, loaded in boxes of 128 bytes x block_size rows with the
// 128-byte swizzle.  Returns false if the encoder is unavailable or rejects the shape.
bool make_cache_tensor_map(CUtensorMap* map, const void* base, uint64_t rows, int head_dim,
                           int block_size, CUtensorMapDataType dtype, int elem_bytes);

}  // namespace pa
