// Shared pieces of the tcgen05 attention kernels (head dim 64, 128-row tiles).
#pragma once

#include <cuda.h>

#include "tc_util.cuh"

namespace gpt2k {
namespace attn {

constexpr int kHD = 64;
constexpr int kTile = 128;  // query / key rows per tile
constexpr int kBox = 16384;  // 128 rows x 64 bf16, 128-byte swizzle
constexpr int kComputeThreads = 256;  // two threads per row (warps w, w+4)

// bf16 x bf16 -> fp32, M = 128, N = n, A K-major, B K- or MN-major
__host__ __device__ constexpr uint32_t idesc(int n, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Tensor map over a [B][T][cols] bf16 array: box = 64 columns x 128 rows of
// one sequence (rows past T read as zero).
cudaError_t seq_map(CUtensorMap* tm, const void* base, int B, int T, int cols);

}  // namespace attn
}  // namespace gpt2k
