// LayerNorm forward and backward: one warp per row, 16-byte vector loads,
// fp32 statistics (biased variance, eps = 1e-5).  The backward's dgamma /
// dbeta column sums are accumulated per warp in registers over a fixed row
// assignment, reduced per block in warp order, and summed over blocks in
// block order: no atomics, fixed summation order.

#include "kernels.h"

namespace gpt2k {

namespace {

constexpr float kLnEps = 1e-5f;

// kMaxChunks = ceil(C / 256): the 8-element chunks each lane owns.
template <int kMaxChunks>
__global__ void ln_fwd_kernel(act_t* __restrict__ y, float* __restrict__ mean,
                              float* __restrict__ rstd, const act_t* __restrict__ x,
                              const float* __restrict__ g, const float* __restrict__ b, int M,
                              int C) {
  const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (row >= M) return;
  const int lane = threadIdx.x & 31;
  const act_t* xr = x + (size_t)row * C;
  float v[kMaxChunks][8];
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const int c = (k * 32 + lane) * 8;
    if (c < C) {
      load8(xr + c, v[k]);
#pragma unroll
      for (int i = 0; i < 8; ++i) s += v[k][i];
    }
  }
  const float mu = warp_sum(s) / C;
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const int c = (k * 32 + lane) * 8;
    if (c < C) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float d = v[k][i] - mu;
        q += d * d;
      }
    }
  }
  const float rs = rsqrtf(warp_sum(q) / C + kLnEps);
  act_t* yr = y + (size_t)row * C;
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const int c = (k * 32 + lane) * 8;
    if (c < C) {
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = (v[k][i] - mu) * rs * g[c + i] + b[c + i];
      store8(yr + c, o);
    }
  }
  if (lane == 0) {
    mean[row] = mu;
    rstd[row] = rs;
  }
}

// grid = kLnBlocks blocks of 8 warps; warp w of block blk handles rows
// (blk * 8 + w) + k * (kLnBlocks * 8).  partials[blk][0..C) = dgamma,
// partials[blk][C..2C) = dbeta.
template <int kMaxChunks>
__global__ void __launch_bounds__(256)
    ln_bwd_kernel(act_t* __restrict__ dres, const act_t* __restrict__ dy,
                  const act_t* __restrict__ x, const float* __restrict__ mean,
                  const float* __restrict__ rstd, const float* __restrict__ g,
                  float* __restrict__ partials, int M, int C, int accumulate) {
  extern __shared__ float red[];  // [8 warps][2C]
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int nw = blockDim.x / 32;
  float dg[kMaxChunks][8], db[kMaxChunks][8], gv[kMaxChunks][8];
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dg[k][i] = 0.f;
      db[k][i] = 0.f;
      const int c = (k * 32 + lane) * 8 + i;
      gv[k][i] = c < C ? g[c] : 0.f;
    }
  for (int row = blockIdx.x * nw + warp; row < M; row += gridDim.x * nw) {
    const act_t* xr = x + (size_t)row * C;
    const act_t* dyr = dy + (size_t)row * C;
    const float mu = mean[row], rs = rstd[row];
    float xh[kMaxChunks][8], dxh[kMaxChunks][8];
    float a = 0.f, bsum = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxChunks; ++k) {
      const int c = (k * 32 + lane) * 8;
      if (c < C) {
        float xv[8], dv[8];
        load8(xr + c, xv);
        load8(dyr + c, dv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          xh[k][i] = (xv[i] - mu) * rs;
          dxh[k][i] = dv[i] * gv[k][i];
          a += dxh[k][i];
          bsum += dxh[k][i] * xh[k][i];
          dg[k][i] += dv[i] * xh[k][i];
          db[k][i] += dv[i];
        }
      }
    }
    a = warp_sum(a) / C;
    bsum = warp_sum(bsum) / C;
    act_t* dr = dres + (size_t)row * C;
#pragma unroll
    for (int k = 0; k < kMaxChunks; ++k) {
      const int c = (k * 32 + lane) * 8;
      if (c < C) {
        float o[8];
        if (accumulate) load8(dr + c, o);
        else {
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] += rs * (dxh[k][i] - a - xh[k][i] * bsum);
        store8(dr + c, o);
      }
    }
  }
  // block reduction of the column partials in warp order
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const int c = (k * 32 + lane) * 8;
    if (c < C) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        red[(size_t)warp * 2 * C + c + i] = dg[k][i];
        red[(size_t)warp * 2 * C + C + c + i] = db[k][i];
      }
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < 2 * C; j += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < nw; ++w) s += red[(size_t)w * 2 * C + j];
    partials[(size_t)blockIdx.x * 2 * C + j] = s;
  }
}

// dg[c] += sum_blk partials[blk][c]; db[c] += sum_blk partials[blk][C + c]
__global__ void ln_bwd_reduce_kernel(float* __restrict__ dg, float* __restrict__ db,
                                     const float* __restrict__ partials, int nblk, int C) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= 2 * C) return;
  float s = 0.f;
  for (int b = 0; b < nblk; ++b) s += partials[(size_t)b * 2 * C + j];
  if (j < C) dg[j] += s;
  else db[j - C] += s;
}

}  // namespace

void layernorm_fwd(act_t* y, float* mean, float* rstd, const act_t* x, const float* g,
                   const float* b, int M, int C, cudaStream_t s) {
  const int warps = 8;
  const int grid = (M + warps - 1) / warps;
  switch ((C + 255) / 256) {
#define GPT2_LNF(N) \
  case N: ln_fwd_kernel<N><<<grid, warps * 32, 0, s>>>(y, mean, rstd, x, g, b, M, C); break;
    GPT2_LNF(1) GPT2_LNF(2) GPT2_LNF(3) GPT2_LNF(4) GPT2_LNF(5) GPT2_LNF(6) GPT2_LNF(7) GPT2_LNF(8)
#undef GPT2_LNF
    default: break;
  }
  note_launch();
}

template <int N>
static void ln_bwd_launch(act_t* dres, const act_t* dy, const act_t* x, const float* mean,
                          const float* rstd, const float* g, float* partials, int M, int C,
                          int accumulate, cudaStream_t s) {
  const size_t smem = (size_t)8 * 2 * C * sizeof(float);
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(ln_bwd_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * 2 * 2048 * 4);
    attr = true;
  }
  ln_bwd_kernel<N><<<kLnBlocks, 256, smem, s>>>(dres, dy, x, mean, rstd, g, partials, M, C, accumulate);
}

void layernorm_bwd(act_t* dres, const act_t* dy, const act_t* x, const float* mean,
                   const float* rstd, const float* g, float* dg, float* db, float* partials,
                   int M, int C, int accumulate, cudaStream_t s) {
  switch ((C + 255) / 256) {
#define GPT2_LNB(N) \
  case N: ln_bwd_launch<N>(dres, dy, x, mean, rstd, g, partials, M, C, accumulate, s); break;
    GPT2_LNB(1) GPT2_LNB(2) GPT2_LNB(3) GPT2_LNB(4) GPT2_LNB(5) GPT2_LNB(6) GPT2_LNB(7) GPT2_LNB(8)
#undef GPT2_LNB
    default: break;
  }
  ln_bwd_reduce_kernel<<<(2 * C + 255) / 256, 256, 0, s>>>(dg, db, partials, kLnBlocks, C);
  note_launch(2);
}

}  // namespace gpt2k
