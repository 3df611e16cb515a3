// Second stages of the two-stage column reductions (layernorm backward
// partials, column sums): one block of 32 x 32 threads per 32 columns, each
// column summed over the partial rows in a fixed order, so that the result
// is the same whether the stage runs at once or later in a grouped launch.
#pragma once

#include "common.cuh"

namespace gpt2k {

// dst_j[c] += sum over b < nblk of partials[b * nsums * C + j * C + c] for the
// 32 columns col = blk * 32 + tx of the nsums * C, with j = col / C: thread
// (tx, ty) takes blocks ty, ty + 32, ... into four running sums combined in a
// fixed order, then the 32 sums are added in ty order.
__device__ __forceinline__ void ln_reduce_block(float* dg, float* db, float* dsum3,
                                                const float* __restrict__ partials, int nblk,
                                                int nsums, int C, int blk) {
  __shared__ float red[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int col = blk * 32 + tx;  // over nsums * C
  const size_t stride = (size_t)nsums * C;
  float s[4] = {0.f, 0.f, 0.f, 0.f};
  if (col < nsums * C) {
    const float* p = partials + col;
    int b = ty;
    for (; b + 96 < nblk; b += 128) {
      s[0] += p[(size_t)b * stride];
      s[1] += p[(size_t)(b + 32) * stride];
      s[2] += p[(size_t)(b + 64) * stride];
      s[3] += p[(size_t)(b + 96) * stride];
    }
    for (int k = 0; b < nblk; b += 32, ++k) s[k] += p[(size_t)b * stride];
  }
  red[ty][tx] = (s[0] + s[1]) + (s[2] + s[3]);
  __syncthreads();
  if (ty == 0 && col < nsums * C) {
    float t = 0.f;
    for (int k = 0; k < 32; ++k) t += red[k][tx];
    const int j = col / C, c = col % C;
    float* dst = j == 0 ? dg : (j == 1 ? db : dsum3);
    dst[c] += t;
  }
}

// db[n] += sum over c < chunks of partials[c * N + n] for the 32 columns
// n = blk * 32 + tx: thread (tx, ty) sums chunks ty, ty + 32, ... in order,
// then the 32 sums are added in ty order.
__device__ __forceinline__ void colsum_reduce_block(float* db, const float* __restrict__ partials,
                                                    int chunks, int N, int blk) {
  __shared__ float red[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int n = blk * 32 + tx;
  float s = 0.f;
  if (n < N)
    for (int c = ty; c < chunks; c += 32) s += partials[(size_t)c * N + n];
  red[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && n < N) {
    float t = 0.f;
    for (int k = 0; k < 32; ++k) t += red[k][tx];
    db[n] += t;
  }
}

}  // namespace gpt2k
