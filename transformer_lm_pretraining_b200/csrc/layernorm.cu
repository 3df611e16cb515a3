// LayerNorm forward and backward: one warp per row, 16-byte vector loads,
// fp32 statistics (biased variance, eps = 1e-5).
//
// The backward's column sums -- dgamma, dbeta and, optionally, the column
// sum of the residual gradient it writes (the bias gradient of the
// projection that produced that residual) -- are accumulated per warp in
// registers over a fixed row assignment, reduced per block in warp order,
// and summed over blocks in block order: no atomics, fixed summation order.

#include "kernels.h"
#include "reduce.cuh"
#include "tc_util.cuh"

namespace gpt2k {

namespace {

constexpr float kLnEps = 1e-5f;

// kChunks = ceil(C / 256): the 8-element chunks each lane owns.
template <int kChunks>
__global__ void __launch_bounds__(256)
    ln_fwd_kernel(act_t* __restrict__ y, float* __restrict__ mean, float* __restrict__ rstd,
                  const act_t* __restrict__ x, const float* __restrict__ g,
                  const float* __restrict__ b, int M, int C) {
  pdl_start();
  const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (row >= M) return;
  const int lane = threadIdx.x & 31;
  const act_t* xr = x + (size_t)row * C;
  float v[kChunks][8];
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kChunks; ++k) {
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
  for (int k = 0; k < kChunks; ++k) {
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
  for (int k = 0; k < kChunks; ++k) {
    const int c = (k * 32 + lane) * 8;
    if (c < C) {
      float gg[8], bb[8], o[8];
      load8(g + c, gg);
      load8(b + c, bb);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = (v[k][i] - mu) * rs * gg[i] + bb[i];
      store8(yr + c, o);
    }
  }
  if (lane == 0) {
    mean[row] = mu;
    rstd[row] = rs;
  }
}

// 8 activations as loaded (16 bytes in the bf16 build): rows are kept in
// this form and converted where used.
struct alignas(16) Pack8 {
  act_t v[8];
};

// Team kernels: TEAMS teams of TPR threads per block, one row per team at a
// time, 8 columns per thread; row sums go through a warp shuffle and, across
// the team's warps, shared memory behind a named barrier of the team alone:
// no block-wide barrier in the row loop.
template <int TPR>
constexpr int ln_teams() {
  return TPR >= 256 ? 2 : (768 / TPR > 8 ? 8 : 768 / TPR);
}
constexpr int kLnStages = 4;  // rows in flight per team

// Bounded wait for the bulk copies of a slot: the copies always complete, so
// the limit only guards against a broken device; after it the row is
// processed with whatever the slot holds and the kernel still ends.
__device__ __forceinline__ void ln_slot_wait(uint32_t bar, uint32_t parity) {
  if (tc::mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = tc::global_ns();
  while (!tc::mbar_try_wait(bar, parity))
    if (tc::global_ns() - t0 > tc::kWaitLimitNs) return;
}

// Chan, Golub & LeVeque (1979), parallel variance: parts a, b of sizes na, nb
// with means ma, mb and squared-deviation sums Sa, Sb form a union of mean
// ma + d nb / n and sum Sa + Sb + d^2 na nb / n, d = mb - ma.  For equal
// sizes, written symmetrically so that both partners of a butterfly step get
// the same bits.
__device__ __forceinline__ void chan_merge(float& mean, float& m2, float n, float mean_b, float m2_b) {
  const float d = mean_b - mean;
  mean = 0.5f * (mean + mean_b);
  m2 = (m2 + m2_b) + d * d * (0.5f * n);
}

// The forward: each team keeps the loads of its next kRegDepth rows in
// flight in registers (plain 16-byte loads; measured faster than bulk-copy
// staging for this one-input kernel when the input is in L2, as the
// residual stream is right after the GEMM that wrote it).  The row's mean
// and sum of squared deviations come from each thread's own 8 values
// (two-pass, exact) combined with chan_merge over the warp and, in warp
// order, across the team's warps.
constexpr int kRegDepth = 4;
template <int TPR>
__global__ void __launch_bounds__(TPR * ln_teams<TPR>())
    ln_fwd_reg_kernel(act_t* __restrict__ y, float* __restrict__ mean, float* __restrict__ rstd,
                      const act_t* __restrict__ x, const float* __restrict__ g,
                      const float* __restrict__ b, int M) {
  pdl_start();
  constexpr int TEAMS = ln_teams<TPR>();
  constexpr int WPR = TPR / 32;
  constexpr int C = 8 * TPR;
  __shared__ float red[TEAMS][2][WPR][2];
  const int team = threadIdx.x / TPR, tc = threadIdx.x % TPR;
  const int wr = tc / 32, lane = threadIdx.x & 31;
  const int c = tc * 8;
  const int stride = gridDim.x * TEAMS;
  const int row0 = blockIdx.x * TEAMS + team;
  float gg[8], bb[8];
  load8(g + c, gg);
  load8(b + c, bb);
  Pack8 buf[kRegDepth];
#pragma unroll
  for (int i = 0; i < kRegDepth; ++i) {
    const int row = row0 + i * stride;
    if (row < M) buf[i] = *reinterpret_cast<const Pack8*>(x + (size_t)row * C + c);
  }
  for (int k = 0;; k += kRegDepth) {
#pragma unroll
    for (int i = 0; i < kRegDepth; ++i) {
      const int row = row0 + (k + i) * stride;
      if (row >= M) return;  // uniform over the team
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = to_f(buf[i].v[e]);
      const int nrow = row + kRegDepth * stride;
      if (nrow < M) buf[i] = *reinterpret_cast<const Pack8*>(x + (size_t)nrow * C + c);
      float mu = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) mu += v[e];
      mu *= 0.125f;
      float m2 = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) m2 = fmaf(v[e] - mu, v[e] - mu, m2);
      float n = 8.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float mb = __shfl_xor_sync(0xffffffffu, mu, o);
        const float sb = __shfl_xor_sync(0xffffffffu, m2, o);
        chan_merge(mu, m2, n, mb, sb);
        n *= 2.f;
      }
      if (WPR > 1) {
        float* rr = &red[team][(k + i) & 1][0][0];
        if (lane == 0) {
          rr[2 * wr] = mu;
          rr[2 * wr + 1] = m2;
        }
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "n"(TPR) : "memory");
        mu = rr[0];
        m2 = rr[1];
        float na = 256.f;
#pragma unroll
        for (int w = 1; w < WPR; ++w) {
          const float d = rr[2 * w] - mu;
          const float nn = na + 256.f;
          mu = fmaf(d, 256.f / nn, mu);
          m2 = m2 + rr[2 * w + 1] + d * d * (na * 256.f / nn);
          na = nn;
        }
      }
      const float rs = rsqrtf(m2 * (1.0f / C) + kLnEps);
      Pack8 q;
#pragma unroll
      for (int e = 0; e < 8; ++e) q.v[e] = from_f<act_t>(fmaf((v[e] - mu) * rs, gg[e], bb[e]));
      *reinterpret_cast<Pack8*>(y + (size_t)row * C + c) = q;
      if (tc == 0) {
        mean[row] = mu;
        rstd[row] = rs;
      }
    }
  }
}

template <int TPR>
void ln_fwd_reg_launch(act_t* y, float* mean, float* rstd, const act_t* x, const float* g,
                       const float* b, int M, cudaStream_t s) {
  constexpr int threads = TPR * ln_teams<TPR>();
  static int grid = 0;
  if (!grid) {
    int per_sm = 0, sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ln_fwd_reg_kernel<TPR>, threads, 0);
    grid = per_sm * sms;
    if (grid < 1) grid = sms;
  }
  launch_kernel(ln_fwd_reg_kernel<TPR>, grid, threads, 0, s, y, mean, rstd, x, g, b, M);
}

// grid = nblk blocks of 8 warps; warp w of block blk handles rows
// (blk * 8 + w) + k * (nblk * 8).  partials[blk][0][..C) = dgamma,
// [1] = dbeta, [2] = column sums of the written dres (when NSUMS == 3).
// The per-column running sums live in shared memory, one private slice per
// warp (each lane owns its columns, so no two threads touch the same word),
// which keeps the row loop's register footprint small enough for several
// blocks per SM.

template <int kChunks, int NSUMS>
__global__ void __launch_bounds__(256, 2)
    ln_bwd_kernel(act_t* __restrict__ dres, const act_t* __restrict__ dy,
                  const act_t* __restrict__ x, const float* __restrict__ mean,
                  const float* __restrict__ rstd, const float* __restrict__ g,
                  float* __restrict__ partials, int M, int C, int accumulate) {
  pdl_start();
  extern __shared__ float red[];  // [8 warps][NSUMS][C]
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int nw = blockDim.x / 32;
  float* mine = red + (size_t)warp * NSUMS * C;
  for (int i = lane; i < NSUMS * C; i += 32) mine[i] = 0.f;
  __syncwarp();
  for (int row = blockIdx.x * nw + warp; row < M; row += gridDim.x * nw) {
    const act_t* xr = x + (size_t)row * C;
    const act_t* dyr = dy + (size_t)row * C;
    act_t* dr = dres + (size_t)row * C;
    // every load of the row is issued before any of it is used
    Pack8 px[kChunks], pd[kChunks], po[kChunks];
#pragma unroll
    for (int k = 0; k < kChunks; ++k) {
      const int c = (k * 32 + lane) * 8;
      if (c < C) {
        px[k] = *reinterpret_cast<const Pack8*>(xr + c);
        pd[k] = *reinterpret_cast<const Pack8*>(dyr + c);
        if (accumulate) po[k] = *reinterpret_cast<const Pack8*>(dr + c);
      }
    }
    const float mu = mean[row], rs = rstd[row];
    float a = 0.f, bsum = 0.f;
#pragma unroll
    for (int k = 0; k < kChunks; ++k) {
      const int c = (k * 32 + lane) * 8;
      if (c < C) {
        float gg[8], s0[8], s1[8];
        load8(g + c, gg);
        load8(mine + c, s0);
        load8(mine + C + c, s1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float xh = (to_f(px[k].v[i]) - mu) * rs;
          const float d = to_f(pd[k].v[i]);
          const float dxh = d * gg[i];
          a += dxh;
          bsum += dxh * xh;
          s0[i] += d * xh;
          s1[i] += d;
        }
        store8(mine + c, s0);
        store8(mine + C + c, s1);
      }
    }
    a = warp_sum(a) / C;
    bsum = warp_sum(bsum) / C;
#pragma unroll
    for (int k = 0; k < kChunks; ++k) {
      const int c = (k * 32 + lane) * 8;
      if (c < C) {
        float gg[8], o[8];
        load8(g + c, gg);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float xh = (to_f(px[k].v[i]) - mu) * rs;
          const float dxh = to_f(pd[k].v[i]) * gg[i];
          o[i] = (accumulate ? to_f(po[k].v[i]) : 0.f) + rs * (dxh - a - xh * bsum);
        }
        if (NSUMS == 3) {
          // the bias gradient sums the values as stored (activation dtype)
          float s2[8];
          load8(mine + 2 * C + c, s2);
#pragma unroll
          for (int i = 0; i < 8; ++i) s2[i] += to_f(from_f<act_t>(o[i]));
          store8(mine + 2 * C + c, s2);
        }
        store8(dr + c, o);
      }
    }
  }
  __syncthreads();
  // block reduction of each column sum in warp order
  for (int i = threadIdx.x; i < NSUMS * C; i += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < nw; ++w) s += red[(size_t)w * NSUMS * C + i];
    partials[(size_t)blockIdx.x * NSUMS * C + i] = s;
  }
}

// The backward stages its rows through shared memory: one thread of each
// team keeps kLnStages of the team's next rows in flight, a slot holding the
// row of x, of dy and (when accumulating) of dres, brought by one
// cp.async.bulk each and completing on the slot's mbarrier, so the bytes in
// flight do not depend on registers; a slot is refilled once every thread
// of the team has passed the team's named barrier (or, for one-warp rows,
// its __syncwarp).  mean and rstd of the next rows are loaded into registers
// ahead.
// Every thread keeps the column sums of its 8 columns (and gamma) in
// registers across its rows.  partials[blk][0..NSUMS) as the per-warp
// kernel (teams added in team order).
template <int TPR>
constexpr int ln_bwd_teams() {
  return TPR >= 256 ? 2 : (384 / TPR > 8 ? 8 : 384 / TPR);
}

template <int TPR, int NSUMS>
__global__ void __launch_bounds__(TPR * ln_bwd_teams<TPR>())
    ln_bwd_staged_kernel(act_t* __restrict__ dres, const act_t* __restrict__ dy,
                         const act_t* __restrict__ x, const float* __restrict__ mean,
                         const float* __restrict__ rstd, const float* __restrict__ g,
                         float* __restrict__ partials, int M, int accumulate) {
  pdl_start();
  constexpr int TEAMS = ln_bwd_teams<TPR>();
  constexpr int WPR = TPR / 32;
  constexpr int C = 8 * TPR;
  constexpr uint32_t kRowBytes = C * sizeof(act_t);
  constexpr uint32_t kSlotBytes = 3 * kRowBytes;  // x | dy | dres
  extern __shared__ __align__(128) uint8_t ln_smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(ln_smem + (size_t)TEAMS * kLnStages * kSlotBytes);
  float* sums = reinterpret_cast<float*>(bars + TEAMS * kLnStages);  // [TEAMS][NSUMS][C] at the end
  __shared__ float red[TEAMS][2][WPR][2];
  const int team = threadIdx.x / TPR, tc = threadIdx.x % TPR;
  const int wr = tc / 32, lane = threadIdx.x & 31;
  const int c = tc * 8;
  const int stride = gridDim.x * TEAMS;
  const int row0 = blockIdx.x * TEAMS + team;
  const uint32_t bar0 = tc::smem_u32(bars + team * kLnStages);
  uint8_t* slots = ln_smem + (size_t)team * kLnStages * kSlotBytes;
  const uint32_t slot0 = tc::smem_u32(slots);
  if (threadIdx.x == 0) {
    for (int i = 0; i < TEAMS * kLnStages; ++i) tc::mbar_init(tc::smem_u32(bars + i), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  auto issue = [&](int k) {  // row k of this team into slot k % kLnStages
    const int row = row0 + k * stride;
    if (row >= M) return;
    const uint32_t bar = bar0 + 8 * (k % kLnStages);
    const uint32_t dst = slot0 + (uint32_t)(k % kLnStages) * kSlotBytes;
    tc::mbar_expect_tx(bar, accumulate ? 3 * kRowBytes : 2 * kRowBytes);
    tc::bulk_load_1d(dst, x + (size_t)row * C, kRowBytes, bar);
    tc::bulk_load_1d(dst + kRowBytes, dy + (size_t)row * C, kRowBytes, bar);
    if (accumulate) tc::bulk_load_1d(dst + 2 * kRowBytes, dres + (size_t)row * C, kRowBytes, bar);
  };
  if (tc == 0)
    for (int k = 0; k < kLnStages; ++k) issue(k);
  float gg[8], s0[8], s1[8], s2[8];
  load8(g + c, gg);
#pragma unroll
  for (int i = 0; i < 8; ++i) s0[i] = s1[i] = s2[i] = 0.f;
  // mean and rstd one row ahead
  float mu_n = 0.f, rs_n = 0.f;
  if (row0 < M) {
    mu_n = mean[row0];
    rs_n = rstd[row0];
  }
  for (int k = 0;; ++k) {
    const int row = row0 + k * stride;
    if (row >= M) break;  // uniform over the team
    const float crs = rs_n, nmr = -mu_n * rs_n;
    if (row + stride < M) {
      mu_n = mean[row + stride];
      rs_n = rstd[row + stride];
    }
    const int st = k % kLnStages;
    ln_slot_wait(bar0 + 8 * st, (uint32_t)(k / kLnStages) & 1u);
    const uint8_t* slot = slots + (size_t)st * kSlotBytes;
    const Pack8 cx = *reinterpret_cast<const Pack8*>(slot + c * sizeof(act_t));
    const Pack8 cd = *reinterpret_cast<const Pack8*>(slot + kRowBytes + c * sizeof(act_t));
    Pack8 co;
    if (accumulate) co = *reinterpret_cast<const Pack8*>(slot + 2 * kRowBytes + c * sizeof(act_t));
    float xh[8], dxh[8], a = 0.f, bsum = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      xh[i] = fmaf(to_f(cx.v[i]), crs, nmr);
      const float d = to_f(cd.v[i]);
      dxh[i] = d * gg[i];
      a += dxh[i];
      bsum = fmaf(dxh[i], xh[i], bsum);
      s0[i] = fmaf(d, xh[i], s0[i]);
      s1[i] += d;
    }
    a = warp_sum(a);
    bsum = warp_sum(bsum);
    if (WPR > 1) {
      float* rr = &red[team][k & 1][0][0];
      if (lane == 0) {
        rr[2 * wr] = a;
        rr[2 * wr + 1] = bsum;
      }
      asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "n"(TPR) : "memory");
      a = 0.f;
      bsum = 0.f;
#pragma unroll
      for (int w = 0; w < WPR; ++w) {
        a += rr[2 * w];
        bsum += rr[2 * w + 1];
      }
    } else {
      __syncwarp();
    }
    if (tc == 0) issue(k + kLnStages);  // every thread of the team has read the slot
    a *= 1.0f / C;
    bsum *= 1.0f / C;
    Pack8 q;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float t = fmaf(-xh[i], bsum, dxh[i] - a);
      const float o = accumulate ? fmaf(crs, t, to_f(co.v[i])) : crs * t;
      q.v[i] = from_f<act_t>(o);
      if (NSUMS == 3) s2[i] += to_f(q.v[i]);  // the bias gradient sums the values as stored
    }
    *reinterpret_cast<Pack8*>(dres + (size_t)row * C + c) = q;
  }
  // block reduction over the teams, in team order
  float* mine = sums + (size_t)team * NSUMS * C;
  store8(mine + c, s0);
  store8(mine + C + c, s1);
  if (NSUMS == 3) store8(mine + 2 * C + c, s2);
  __syncthreads();
  for (int i = threadIdx.x; i < NSUMS * C; i += blockDim.x) {
    float t = 0.f;
    for (int k = 0; k < TEAMS; ++k) t += sums[(size_t)k * NSUMS * C + i];
    partials[(size_t)blockIdx.x * NSUMS * C + i] = t;
  }
}

template <int TPR, int S>
int ln_bwd_staged_launch(act_t* dres, const act_t* dy, const act_t* x, const float* mean,
                         const float* rstd, const float* g, float* partials, int M,
                         int accumulate, cudaStream_t s) {
  constexpr int TEAMS = ln_bwd_teams<TPR>();
  constexpr int threads = TPR * TEAMS;
  constexpr size_t smem = (size_t)TEAMS * kLnStages * (3 * 8 * TPR * sizeof(act_t) + 8) +
                          (size_t)TEAMS * S * 8 * TPR * sizeof(float);
  static int grid = 0;
  if (!grid) {
    cudaFuncSetAttribute(ln_bwd_staged_kernel<TPR, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    int per_sm = 0, sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ln_bwd_staged_kernel<TPR, S>, threads,
                                                  smem);
    grid = per_sm * sms;
    if (grid < 1 || grid > kLnBlocks) grid = kLnBlocks;
  }
  launch_kernel(ln_bwd_staged_kernel<TPR, S>, grid, threads, smem, s, dres, dy, x, mean, rstd, g, partials,
                                                           M, accumulate);
  return grid;
}

// out_j[c] += sum over blocks of partials[blk][j][c] in a fixed order:
// thread (tx, ty) of a 32 x 32 block takes column tx of a 32-column group
// and blocks ty, ty+32, ... (four independent running sums, combined in a
// fixed order); the 32 partial sums are then added in ty order.
__global__ void __launch_bounds__(1024)
    ln_bwd_reduce_kernel(float* __restrict__ dg, float* __restrict__ db, float* __restrict__ dsum3,
                         const float* __restrict__ partials, int nblk, int nsums, int C) {
  pdl_start();
  ln_reduce_block(dg, db, dsum3, partials, nblk, nsums, C, blockIdx.x);
}

// Launches one wave: as many blocks as are resident at once (at most
// kLnBlocks), so no block waits for a second wave.  Returns the grid used.
template <int N, int S>
int ln_bwd_launch(act_t* dres, const act_t* dy, const act_t* x, const float* mean,
                  const float* rstd, const float* g, float* partials, int M, int C,
                  int accumulate, cudaStream_t s) {
  const size_t smem = (size_t)8 * S * C * sizeof(float);
  static bool attr = false;
  static int grid_c = -1, grid = kLnBlocks;
  if (!attr) {
    cudaFuncSetAttribute(ln_bwd_kernel<N, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         8 * S * 2048 * 4 > 227 * 1024 ? 227 * 1024 : 8 * S * 2048 * 4);
    attr = true;
  }
  if (grid_c != C) {
    int per_sm = 0, sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ln_bwd_kernel<N, S>, 256, smem);
    grid = per_sm * sms;
    if (grid < 1 || grid > kLnBlocks) grid = kLnBlocks;
    grid_c = C;
  }
  launch_kernel(ln_bwd_kernel<N, S>, grid, 256, smem, s, dres, dy, x, mean, rstd, g, partials, M, C,
                                              accumulate);
  return grid;
}

}  // namespace

void layernorm_fwd(act_t* y, float* mean, float* rstd, const act_t* x, const float* g,
                   const float* b, int M, int C, cudaStream_t s) {
  switch (C) {  // widths with a team kernel
#define GPT2_LNFT(W)                                           \
  case W:                                                    \
    ln_fwd_reg_launch<W / 8>(y, mean, rstd, x, g, b, M, s); \
    note_launch();                                           \
    return;
    GPT2_LNFT(256) GPT2_LNFT(512) GPT2_LNFT(768) GPT2_LNFT(1024) GPT2_LNFT(2048)
#undef GPT2_LNFT
    default: break;
  }
  const int warps = 8;
  const int grid = (M + warps - 1) / warps;
  switch ((C + 255) / 256) {
#define GPT2_LNF(N) \
  case N: launch_kernel(ln_fwd_kernel<N>, grid, warps * 32, 0, s, y, mean, rstd, x, g, b, M, C); break;
    GPT2_LNF(1) GPT2_LNF(2) GPT2_LNF(3) GPT2_LNF(4) GPT2_LNF(5) GPT2_LNF(6) GPT2_LNF(7) GPT2_LNF(8)
#undef GPT2_LNF
    default: break;
  }
  note_launch();
}

void layernorm_bwd(act_t* dres, const act_t* dy, const act_t* x, const float* mean,
                   const float* rstd, const float* g, float* dg, float* db, float* dbias_out,
                   float* partials, int M, int C, int accumulate, cudaStream_t s,
                   ReduceJob* defer) {
  const int nsums = dbias_out ? 3 : 2;
  int nblk = kLnBlocks;
  switch (C * 4 + nsums) {  // widths with a row-group kernel
#define GPT2_LNR(W)                                                                            \
  case 4 * W + 2:                                                                              \
    nblk = ln_bwd_staged_launch<W / 8, 2>(dres, dy, x, mean, rstd, g, partials, M, accumulate, s); \
    goto reduce;                                                                               \
  case 4 * W + 3:                                                                              \
    nblk = ln_bwd_staged_launch<W / 8, 3>(dres, dy, x, mean, rstd, g, partials, M, accumulate, s); \
    goto reduce;
    GPT2_LNR(256) GPT2_LNR(512) GPT2_LNR(768) GPT2_LNR(1024) GPT2_LNR(2048)
#undef GPT2_LNR
    default: break;
  }
  switch ((C + 255) / 256 * 4 + nsums) {
#define GPT2_LNB(N)                                                                          \
  case 4 * N + 2:                                                                            \
    nblk = ln_bwd_launch<N, 2>(dres, dy, x, mean, rstd, g, partials, M, C, accumulate, s);   \
    break;                                                                                   \
  case 4 * N + 3:                                                                            \
    nblk = ln_bwd_launch<N, 3>(dres, dy, x, mean, rstd, g, partials, M, C, accumulate, s);   \
    break;
    GPT2_LNB(1) GPT2_LNB(2) GPT2_LNB(3) GPT2_LNB(4) GPT2_LNB(5) GPT2_LNB(6) GPT2_LNB(7) GPT2_LNB(8)
#undef GPT2_LNB
    default: break;
  }
reduce:
  if (defer) {
    *defer = ReduceJob{{dg, db, dbias_out}, partials, nblk, nsums, C, REDUCE_LN};
    note_launch();
    return;
  }
  launch_kernel(ln_bwd_reduce_kernel, (nsums * C + 31) / 32, 1024, 0, s, dg, db, dbias_out, partials, nblk,
                                                               nsums, C);
  note_launch(2);
}

}  // namespace gpt2k
