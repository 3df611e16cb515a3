// Bias-gradient column sums, the fused softmax cross-entropy, the mean
// loss, parameter init, the global gradient norm and AdamW.

#include <atomic>

#include <cuda_fp16.h>

#include "kernels.h"
#include "reduce.cuh"
#include "tc_util.cuh"

namespace gpt2k {

// ------------------------------------------------------------ layout --
Layout make_layout(int L, int H, int C, int V, int Vp, int Tmax) {
  Layout g;
  g.L = L; g.H = H; g.C = C; g.V = V; g.Vp = Vp; g.Tmax = Tmax;
  const size_t l = (size_t)L, c = (size_t)C;
  g.num[T_WTE] = (size_t)Vp * c;
  g.num[T_WPE] = (size_t)Tmax * c;
  g.num[T_LN1G] = l * c;
  g.num[T_LN1B] = l * c;
  g.num[T_WQKV] = l * 3 * c * c;
  g.num[T_BQKV] = l * 3 * c;
  g.num[T_WO] = l * c * c;
  g.num[T_BO] = l * c;
  g.num[T_LN2G] = l * c;
  g.num[T_LN2B] = l * c;
  g.num[T_WFC] = l * 4 * c * c;
  g.num[T_BFC] = l * 4 * c;
  g.num[T_WP] = l * 4 * c * c;
  g.num[T_BP] = l * c;
  g.num[T_LNFG] = c;
  g.num[T_LNFB] = c;
  size_t o = 0;
  for (int i = 0; i < T_COUNT; ++i) {
    g.off[i] = o;
    o += g.num[i];
  }
  g.total = o;
  return g;
}

static std::atomic<long> g_launches{0};
static int g_pdl = 1;
bool pdl_enabled() { return g_pdl != 0; }
int set_pdl(int enable) {
  const int prev = g_pdl;
  g_pdl = enable ? 1 : 0;
  return prev;
}

void note_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
long launch_count() { return g_launches.load(std::memory_order_relaxed); }

bool tensor_decayed(int t) {
  return t == T_WTE || t == T_WPE || t == T_WQKV || t == T_WO || t == T_WFC || t == T_WP;
}

namespace {

// ------------------------------------------------------------ colsum --
// partials[chunk][n] = sum over the chunk's rows of dy[m, n] (row set of
// warp w: r0 + w, r0 + w + 8, ...; then the 8 warps in order).  A warp
// covers 256 columns, 8 per lane (16-byte loads); N % 8 == 0.
__global__ void __launch_bounds__(256)
    colsum_partial_kernel(float* __restrict__ partials, const act_t* __restrict__ dy, int M, int N,
                          int rows_per_chunk) {
  pdl_start();
  __shared__ float red[8][256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int n = blockIdx.x * 256 + lane * 8;
  const int r0 = blockIdx.y * rows_per_chunk;
  const int r1 = min(M, r0 + rows_per_chunk);
  float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (n < N) {
    int r = r0 + w;
    // eight rows in flight, loaded as raw 16-byte vectors and converted after
    struct alignas(16) Row8 {
      act_t v[8];
    };
    for (; r < r1; r += 64) {  // one round trip per 8 rows, the last batch guarded
      Row8 q[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (r + 8 * k < r1) {
          q[k] = *reinterpret_cast<const Row8*>(dy + (size_t)(r + 8 * k) * N + n);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) q[k].v[i] = from_f<act_t>(0.f);
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k)
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i] += to_f(q[k].v[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[w][lane * 8 + i] = s[i];
  __syncthreads();
  const int col = blockIdx.x * 256 + threadIdx.x;
  if (col < N) {
    float t = 0.f;
    for (int k = 0; k < 8; ++k) t += red[k][threadIdx.x];
    partials[(size_t)blockIdx.y * N + col] = t;
  }
}

// db[n] += sum over chunks of partials[chunk][n] in a fixed order
// (colsum_reduce_block).
__global__ void __launch_bounds__(1024)
    colsum_reduce_kernel(float* __restrict__ db, const float* __restrict__ partials, int chunks,
                         int N) {
  pdl_start();
  colsum_reduce_block(db, partials, chunks, N, blockIdx.x);
}

// Every job of the list: block b belongs to the first job k with
// b < group_end[k] and reduces that job's 32-column group b - group_end[k - 1].
__global__ void __launch_bounds__(1024) reduce_jobs_kernel(const __grid_constant__ ReduceJobs jobs) {
  pdl_start();
  int k = 0;
  while (k + 1 < jobs.n && (int)blockIdx.x >= jobs.group_end[k]) ++k;
  const ReduceJob& j = jobs.job[k];
  const int grp = (int)blockIdx.x - (k ? jobs.group_end[k - 1] : 0);
  if (j.kind == REDUCE_LN) ln_reduce_block(j.dst[0], j.dst[1], j.dst[2], j.partials, j.nrows, j.nsums, j.C, grp);
  else colsum_reduce_block(j.dst[0], j.partials, j.nrows, j.C, grp);
}

// -------------------------------------------------------- classifier --
// One block per row.  Pass 1: max and sum of exp over the first V logits
// (per-thread online, then block reduction in fixed order).  Pass 2:
// z <- (exp(z - lse) - [col == tgt]) / M for col < V, 0 for padding.
constexpr int kClsThreads = 512;

__device__ __forceinline__ void online_merge(float& m, float& s, float m2, float s2) {
  if (m2 > m) {
    s = s * __expf(m - m2) + s2;
    m = m2;
  } else if (m2 > -INFINITY) {
    s += s2 * __expf(m2 - m);
  }
}

__global__ void __launch_bounds__(kClsThreads)
    classifier_kernel(act_t* __restrict__ logits, float* __restrict__ losses,
                      const int* __restrict__ tgt, int M, int V, int Vp, int write_grad,
                      int* err) {
  pdl_start();
  const int row = blockIdx.x;
  act_t* z = logits + (size_t)row * Vp;
  const int vec = (Vp % 8 == 0) ? 8 : 1;
  float mx = -INFINITY, sm = 0.f;
  if (vec == 8) {
    for (int c = threadIdx.x * 8; c < Vp; c += kClsThreads * 8) {
      float v[8];
      load8(z + c, v);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (c + i < V) online_merge(mx, sm, v[i], 1.f);
    }
  } else {
    for (int c = threadIdx.x; c < V; c += kClsThreads) online_merge(mx, sm, to_f(z[c]), 1.f);
  }
  // warp then block reduction (fixed order)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, mx, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, sm, o);
    online_merge(mx, sm, m2, s2);
  }
  __shared__ float wm[kClsThreads / 32], ws[kClsThreads / 32];
  __shared__ float lse_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    wm[warp] = mx;
    ws[warp] = sm;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = wm[0], s = ws[0];
    for (int w = 1; w < kClsThreads / 32; ++w) online_merge(m, s, wm[w], ws[w]);
    lse_s = m + logf(s);
  }
  __syncthreads();
  const float lse = lse_s;
  int t = tgt[row];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) atomicOr(err, ERR_TARGET);
    t = 0;
  }
  if (threadIdx.x == 0) losses[row] = lse - to_f(z[t]);
  if (!write_grad) return;
  __syncthreads();  // the target logit is read before it is overwritten
  const float inv = 1.0f / (float)M;
  if (vec == 8) {
    for (int c = threadIdx.x * 8; c < Vp; c += kClsThreads * 8) {
      float v[8];
      load8(z + c, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int col = c + i;
        v[i] = col < V ? (__expf(v[i] - lse) - (col == t ? 1.f : 0.f)) * inv : 0.f;
      }
      store8(z + c, v);
    }
  } else {
    for (int c = threadIdx.x; c < Vp; c += kClsThreads) {
      const float v = to_f(z[c]);
      z[c] = from_f<act_t>(c < V ? (__expf(v - lse) - (c == t ? 1.f : 0.f)) * inv : 0.f);
    }
  }
}

// Persistent variant for rows that fit twice in shared memory: persistent
// CTAs take rows blockIdx.x, + gridDim.x, ...; each row arrives with one
// bulk copy into a shared-memory row buffer, so HBM sees one read and one
// write of the logits.  Three passes over shared memory: the max (on
// packed bf16 pairs); the exponentials e = exp(z - max), summed in fp32
// (per-thread partials over a fixed column assignment, then warps in order)
// and kept in place as fp16; then z <- e / sum / M - onehot / M written
// straight to global memory (skipped when write_grad == 0).  Separate max
// and sum passes keep every exponential independent of the others (a
// running max would chain them), and each logit is exponentiated once.
// The bf16 build only (rows of 2-byte logits).
// Configurations: one CTA of 1024 threads per SM with two row buffers (a
// row loads while the previous one is computed), or two CTAs of 512 threads
// per SM with one buffer each, whose loads and barrier-separated passes
// interleave.  Measured at M 16384 x Vpad 50304: 709 us (4.65 TB/s) for the
// first, 548 us (6.0 TB/s) for the second.
constexpr int kClsCtasPerSm = 2;  // 1: <1024 threads, 2 buffers>; 2: <512, 1> twice

template <int THREADS>
__device__ __forceinline__ float block_reduce_cls(float v, float* red, bool is_max) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < THREADS / 32; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  __syncthreads();  // red is reused by the next reduction
  return r;
}

template <int THREADS, int NB>
__global__ void __launch_bounds__(THREADS, 2048 / THREADS / 1 > 2 ? 2 : 2048 / THREADS)
    classifier_bulk_kernel(act_t* __restrict__ logits, float* __restrict__ losses,
                           const int* __restrict__ tgt, int M, int V, int Vp, int write_grad,
                           int* err) {
  pdl_start();
  using namespace tc;
  extern __shared__ __align__(128) uint8_t cls_smem[];
  __shared__ float red[THREADS / 32];
  __shared__ uint64_t bars[NB];
  __shared__ int abort_s;
  const uint32_t row_bytes = (uint32_t)Vp * sizeof(act_t);
  const uint32_t buf_stride = (row_bytes + 127u) & ~127u;
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int b = 0; b < NB; ++b) mbar_init(smem_u32(&bars[b]), 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  auto issue = [&](int b, int r) {
    const uint32_t bar = smem_u32(&bars[b]);
    mbar_expect_tx(bar, row_bytes);
    bulk_load_1d(smem_u32(cls_smem + b * buf_stride), logits + (size_t)r * Vp, row_bytes, bar);
  };
  if (tid == 0) {
    for (int b = 0; b < NB; ++b)
      if (blockIdx.x + b * gridDim.x < M) issue(b, blockIdx.x + b * gridDim.x);
  }
  const float inv = 1.0f / (float)M;
  constexpr float kLog2e = 1.4426950408889634f;
  uint32_t phase = 0;  // bit b: parity of buffer b's next fill
  int it = 0;
  for (int row = blockIdx.x; row < M; row += gridDim.x, ++it) {
    const int b = it % NB;
    const bool got = mbar_wait(smem_u32(&bars[b]), (phase >> b) & 1u, &abort_s, err);
    if (!__syncthreads_and(got)) break;
    phase ^= 1u << b;
    uint8_t* zb = cls_smem + b * buf_stride;
    const act_t* z = reinterpret_cast<const act_t*>(zb);
    int t = tgt[row];
    if (t < 0 || t >= V) {
      if (tid == 0) atomicOr(err, ERR_TARGET);
      t = 0;
    }
    const float zt = to_f(z[t]);  // read before pass 2 overwrites the row
    // pass 1: the max over columns < V, on packed bf16 pairs
    float mx = -INFINITY;
    {
      __nv_bfloat162 m2 = __floats2bfloat162_rn(-INFINITY, -INFINITY);
      for (int c = tid * 8; c < Vp; c += THREADS * 8) {
        if (c + 8 <= V) {
          const uint4 u = *reinterpret_cast<const uint4*>(z + c);
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
          m2 = __hmax2(__hmax2(m2, h2[0]), __hmax2(h2[1], __hmax2(h2[2], h2[3])));
        } else {
          for (int i = 0; i < 8 && c + i < V; ++i) mx = fmaxf(mx, to_f(z[c + i]));
        }
      }
      mx = fmaxf(mx, fmaxf(__low2float(m2), __high2float(m2)));
    }
    mx = block_reduce_cls<THREADS>(mx, red, true);
    const float mx2 = mx * kLog2e;
    // pass 2: e = exp(z - max) summed in fp32 and kept in place as fp16
    // (0 for the padded columns), so that pass 3 needs no exponential
    float sm = 0.f;
    for (int c = tid * 8; c < Vp; c += THREADS * 8) {
      float v[8];
      load8(z + c, v);
      if (c + 8 <= V) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[i] = fast_exp2(fmaf(v[i], kLog2e, -mx2));
          sm += v[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[i] = c + i < V ? fast_exp2(fmaf(v[i], kLog2e, -mx2)) : 0.f;
          sm += v[i];
        }
      }
      uint4 o;
      __half2* o2 = reinterpret_cast<__half2*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) o2[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
      *reinterpret_cast<uint4*>(zb + (size_t)c * 2) = o;
    }
    sm = block_reduce_cls<THREADS>(sm, red, false);
    const float lse = mx + logf(sm);
    if (tid == 0) losses[row] = lse - zt;
    if (write_grad) {
      // pass 3: z <- e / sum / M, minus 1 / M at the target
      const float sc = inv / sm;
      act_t* out = logits + (size_t)row * Vp;
      for (int c = tid * 8; c < Vp; c += THREADS * 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(zb + (size_t)c * 2);
        const __half2* e2 = reinterpret_cast<const __half2*>(&u);
        float v[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(e2[i]);
          v[2 * i] = f.x * sc;
          v[2 * i + 1] = f.y * sc;
        }
        if (t >= c && t < c + 8) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (c + i == t) v[i] -= inv;
        }
        store8(out + c, v);
      }
    }
    __syncthreads();  // every read of buffer b is done
    if (tid == 0 && row + NB * gridDim.x < M) {
      fence_async_smem();
      issue(b, row + NB * gridDim.x);
    }
  }
  // copies still in flight land before the shared memory is released
  if (tid == 0) {
    const uint64_t t0 = global_ns();
    for (int k = 0; k < NB; ++k) {
      const int r = blockIdx.x + (it + k) * gridDim.x;
      if (r >= M) break;
      while (!mbar_try_wait(smem_u32(&bars[(it + k) % NB]), (phase >> ((it + k) % NB)) & 1u) &&
             global_ns() - t0 < kWaitLimitNs) {
      }
    }
  }
}

__global__ void mean_loss_kernel(float* out, const float* __restrict__ losses, int M) {
  pdl_start();
  __shared__ float red[1024];
  float s = 0.f;
  for (int i = threadIdx.x; i < M; i += blockDim.x) s += losses[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[0] = red[0] / (float)M;
}

// -------------------------------------------------------------- init --
// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): output n of a generator
// seeded with s is mix(s + n * 0x9E3779B97F4A7C15).  Tensor t uses the
// generator seeded with output t+1 of the master generator seeded with
// `seed`; element i takes outputs 2i+1, 2i+2 as the two uniforms of one
// Box-Muller normal (cosine branch), evaluated in double, rounded once.

struct InitSeg {
  size_t off, count;  // elements [off, off + count) get normals
  uint64_t tseed;
  double sd;
};
struct InitTable {
  InitSeg seg[6];
  int n;
};

__global__ void init_normal_kernel(float* __restrict__ p, InitTable tab) {
  pdl_start();
  const InitSeg sg = tab.seg[blockIdx.y];
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < sg.count;
       i += (size_t)gridDim.x * blockDim.x) {
    const uint64_t r1 = sm64_out(sg.tseed, 2 * i + 1);
    const uint64_t r2 = sm64_out(sg.tseed, 2 * i + 2);
    const double u1 = (double)((r1 >> 11) + 1) * 0x1.0p-53;
    const double u2 = (double)(r2 >> 11) * 0x1.0p-53;
    const double z = sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
    p[sg.off + i] = (float)(sg.sd * z);
  }
}

__global__ void fill_kernel(float* p, size_t n, float v) {
  pdl_start();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    p[i] = v;
}

template <class TO, class TI>
__global__ void convert_kernel(TO* __restrict__ out, const TI* __restrict__ in, size_t n) {
  pdl_start();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    out[i] = from_f<TO>(to_f(in[i]));
}

// -------------------------------------------------------- grad norm --
// Stage 1: block b sums g^2 over the fixed strided set of float4s
// i = b * 256 + tid + k * (gridDim.x * 256) in double, then reduces over the
// block in a fixed tree.  Stage 2 (one block) adds the block sums in order.
__global__ void __launch_bounds__(256) norm_partial_kernel(double* __restrict__ partials,
                                                           const float* __restrict__ g,
                                                           size_t n) {
  pdl_start();
  __shared__ double red[256];
  double s = 0.0;
  const size_t n4 = n / 4;
  const float4* g4 = reinterpret_cast<const float4*>(g);
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n4; i += (size_t)gridDim.x * 256) {
    const float4 v = g4[i];
    s += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
  }
  if (blockIdx.x == 0)
    for (size_t i = n4 * 4 + threadIdx.x; i < n; i += 256) s += (double)g[i] * g[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) partials[blockIdx.x] = red[0];
}

// The sum of the nblk block partials, in a fixed order: thread t of 256 adds
// partials t, t + 256, ..., then a fixed tree over the threads.
__device__ __forceinline__ double partials_sum(const double* __restrict__ partials, int nblk) {
  __shared__ double red[256];
  double s = 0.0;
  for (int b = threadIdx.x; b < nblk; b += 256) s += partials[b];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  return red[0];
}

__global__ void __launch_bounds__(256) sumsq_final_kernel(double* __restrict__ out,
                                                          const double* __restrict__ partials,
                                                          int nblk) {
  pdl_start();
  const double s = partials_sum(partials, nblk);
  if (threadIdx.x == 0) *out = s;
}

__global__ void clip_from_sumsq_kernel(float* __restrict__ scalars, const double* __restrict__ sumsq,
                                       float max_norm) {
  pdl_start();
  const float nrm = (float)sqrt(*sumsq);
  scalars[S_NORM] = nrm;
  scalars[S_CLIP] = (nrm > max_norm) ? max_norm / (nrm + 1e-6f) : 1.0f;
}

__global__ void __launch_bounds__(256) norm_final_kernel(float* __restrict__ scalars,
                                                         const double* __restrict__ partials,
                                                         int nblk, float max_norm) {
  pdl_start();
  const double s = partials_sum(partials, nblk);
  if (threadIdx.x != 0) return;
  const float nrm = (float)sqrt(s);
  scalars[S_NORM] = nrm;
  scalars[S_CLIP] = (nrm > max_norm) ? max_norm / (nrm + 1e-6f) : 1.0f;
}

// ------------------------------------------------------------- AdamW --
struct DecayTable {
  size_t begin[T_COUNT];
  size_t end[T_COUNT];
  int n;
};

// One float4 of the update (elements i .. i + 3 of the flat order).
__device__ __forceinline__ void adamw4(float4& pp, const float4 gg, float4& mm, float4& vv, float4& out,
                                       const AdamArgs& a, float wd, float clip, float lr, float ibc1,
                                       float ibc2) {
  float* pe = &pp.x;
  const float* ge = &gg.x;
  float* me = &mm.x;
  float* ve = &vv.x;
  float* oe = &out.x;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float gr = ge[j] * clip;
    me[j] = a.b1 * me[j] + (1.f - a.b1) * gr;
    ve[j] = a.b2 * ve[j] + (1.f - a.b2) * gr * gr;
    const float mh = me[j] * ibc1;
    const float vh = ve[j] * ibc2;
    pe[j] -= lr * (mh / (sqrtf(vh) + a.eps) + wd * pe[j]);
    oe[j] = pe[j];
  }
}

__device__ __forceinline__ float adamw_decay(size_t i, const DecayTable& dt, float wd) {
  float r = 0.f;
  for (int k = 0; k < dt.n; ++k)
    if (i >= dt.begin[k] && i < dt.end[k]) r = wd;
  return r;
}

// Each thread takes two float4 per pass (all eight loads issued before the
// arithmetic), so more bytes are in flight per thread.
__global__ void __launch_bounds__(256)
    adamw_kernel(float* __restrict__ p, act_t* __restrict__ pact, const float* __restrict__ g,
                 float* __restrict__ m, float* __restrict__ v, size_t base, size_t n, AdamArgs a,
                 DecayTable dt, const float* __restrict__ scalars) {
  pdl_start();
  const float nrm = scalars[S_NORM];
  if (!isfinite(nrm)) return;  // never apply a non-finite update
  const float clip = scalars[S_CLIP];
  const float lr = scalars[S_LR];
  const float ibc1 = 1.f / scalars[S_BC1], ibc2 = 1.f / scalars[S_BC2];
  const size_t n4 = n / 4;
  p += base;
  pact += base;
  g += base;
  m += base;
  v += base;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i4 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i4 < n4; i4 += 2 * stride) {
    const size_t j4 = i4 + stride;
    const bool two = j4 < n4;
    float4 pp[2], gg[2], mm[2], vv[2], out[2];
    pp[0] = reinterpret_cast<float4*>(p)[i4];
    gg[0] = reinterpret_cast<const float4*>(g)[i4];
    mm[0] = reinterpret_cast<float4*>(m)[i4];
    vv[0] = reinterpret_cast<float4*>(v)[i4];
    if (two) {
      pp[1] = reinterpret_cast<float4*>(p)[j4];
      gg[1] = reinterpret_cast<const float4*>(g)[j4];
      mm[1] = reinterpret_cast<float4*>(m)[j4];
      vv[1] = reinterpret_cast<float4*>(v)[j4];
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h == 1 && !two) break;
      const size_t k4 = h ? j4 : i4;
      adamw4(pp[h], gg[h], mm[h], vv[h], out[h], a, adamw_decay(base + k4 * 4, dt, a.wd), clip, lr,
             ibc1, ibc2);
      reinterpret_cast<float4*>(p)[k4] = pp[h];
      reinterpret_cast<float4*>(m)[k4] = mm[h];
      reinterpret_cast<float4*>(v)[k4] = vv[h];
#if GPT2_ACT_BF16
      __nv_bfloat162 lo = __floats2bfloat162_rn(out[h].x, out[h].y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(out[h].z, out[h].w);
      uint2 packed;
      packed.x = *reinterpret_cast<uint32_t*>(&lo);
      packed.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(pact)[k4] = packed;
#else
      (void)pact;
#endif
    }
  }
}

// The step's learning rate: warmup lr_max (s + 1) / W for s < W, then a
// cosine from lr_max down to lr_min at s = S, lr_min after (condensed GPT-2
// page, section 3; the same formula as the host's gpt2_lr).
struct Sched {
  double max_lr, min_lr, warmup, max_steps;
};
__global__ void adam_prep_kernel(float* scalars, int* step, float lr, int scheduled, Sched sc,
                                 float b1, float b2) {
  pdl_start();
  const int t = *step + 1;
  *step = t;
  double l = lr;
  if (scheduled) {
    const double s = (double)(t - 1);
    if (s < sc.warmup) l = sc.max_lr * (s + 1.0) / sc.warmup;
    else if (s > sc.max_steps || sc.max_steps <= sc.warmup) l = sc.min_lr;
    else {
      const double ratio = (s - sc.warmup) / (sc.max_steps - sc.warmup);
      l = sc.min_lr + 0.5 * (1.0 + cos(3.14159265358979323846 * ratio)) * (sc.max_lr - sc.min_lr);
    }
  }
  scalars[S_LR] = (float)l;
  scalars[S_BC1] = (float)(1.0 - pow((double)b1, (double)t));
  scalars[S_BC2] = (float)(1.0 - pow((double)b2, (double)t));
}

__global__ void reset_clip_kernel(float* scalars) {
  pdl_start();
  scalars[S_NORM] = 0.f;
  scalars[S_CLIP] = 1.f;
}

int grid_for(size_t n, int threads, int max_blocks) {
  size_t b = (n + threads - 1) / threads;
  if (b > (size_t)max_blocks) b = max_blocks;
  if (b < 1) b = 1;
  return (int)b;
}

}  // namespace

void colsum_acc(float* db, const act_t* dy, int M, int N, float* partials, cudaStream_t s,
                ReduceJob* defer) {
  // as many blocks as are resident at once and no more: a block past the
  // first wave would run on its own after it
  static int per_sm = 0;
  if (!per_sm) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, colsum_partial_kernel, 256, 0);
    if (per_sm < 1) per_sm = 1;
  }
  const int colgroups = (N + 255) / 256;
  int want = per_sm * kNumSMs / colgroups;
  if (want < 1) want = 1;
  if (want > kColsumChunks) want = kColsumChunks;
  const int rows = (M + want - 1) / want;
  const int chunks = (M + rows - 1) / rows;
  dim3 g(colgroups, chunks);
  launch_kernel(colsum_partial_kernel, g, 256, 0, s, partials, dy, M, N, rows);
  note_launch();
  colsum_reduce(db, partials, chunks, N, s, defer);
}

void colsum_reduce(float* db, const float* partials, int chunks, int N, cudaStream_t s,
                   ReduceJob* defer) {
  if (defer) {
    *defer = ReduceJob{{db, nullptr, nullptr}, partials, chunks, 1, N, REDUCE_COLSUM};
    return;
  }
  launch_kernel(colsum_reduce_kernel, (N + 31) / 32, 1024, 0, s, db, partials, chunks, N);
  note_launch();
}

bool reduce_jobs_add(ReduceJobs& jobs, const ReduceJob& j) {
  if (jobs.n >= kMaxReduceJobs) return false;
  const int groups = (j.nsums * j.C + 31) / 32;
  jobs.group_end[jobs.n] = (jobs.n ? jobs.group_end[jobs.n - 1] : 0) + groups;
  jobs.job[jobs.n++] = j;
  return true;
}

void reduce_jobs_run(ReduceJobs& jobs, cudaStream_t s) {
  if (jobs.n == 0) return;
  launch_kernel(reduce_jobs_kernel, jobs.group_end[jobs.n - 1], 1024, 0, s, jobs);
  note_launch();
  jobs.n = 0;
}

void classifier(act_t* logits, float* losses, const int* tgt, int M, int V, int Vp, int write_grad,
                int* err, cudaStream_t s) {
  if (M <= 0) return;
  const size_t row_bytes = (size_t)Vp * sizeof(act_t);
  const size_t buf = (row_bytes + 127) & ~(size_t)127;
  if (sizeof(act_t) == 2 && 2 * buf <= 200 * 1024 && row_bytes % 16 == 0 &&
      (reinterpret_cast<uintptr_t>(logits) & 15) == 0) {
    // two row buffers per SM either way
    constexpr int kThr = kClsCtasPerSm == 2 ? 512 : 1024, kNb = kClsCtasPerSm == 2 ? 1 : 2;
    const size_t smem = kNb * buf;
    auto kern = classifier_bulk_kernel<kThr, kNb>;
    static size_t attr = 0;
    if (attr < smem) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      attr = smem;
    }
    int sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int slots = kClsCtasPerSm * sms;
    const int grid = M < slots ? M : slots;
    launch_kernel(kern, grid, kThr, smem, s, logits, losses, tgt, M, V, Vp, write_grad, err);
  } else {
    launch_kernel(classifier_kernel, M, kClsThreads, 0, s, logits, losses, tgt, M, V, Vp, write_grad, err);
  }
  note_launch();
}

void mean_loss(float* out, const float* losses, int M, cudaStream_t s) {
  launch_kernel(mean_loss_kernel, 1, 1024, 0, s, out, losses, M);
  note_launch();
}

namespace {
__global__ void gelu_fwd_kernel(act_t* __restrict__ g, const act_t* __restrict__ u, size_t n) {
  pdl_start();
  const size_t n8 = n / 8;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (size_t)gridDim.x * blockDim.x) {
    float v[8];
    load8(u + 8 * i, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = gelu_tanh(v[k]);
    store8(g + 8 * i, v);
  }
  for (size_t i = 8 * n8 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    g[i] = from_f<act_t>(gelu_tanh(to_f(u[i])));
}
}  // namespace

void gelu_fwd(act_t* g, const act_t* u, size_t n, cudaStream_t s) {
  if (!n) return;
  launch_kernel(gelu_fwd_kernel, grid_for(n / 8 + 1, 256, 8 * kNumSMs), 256, 0, s, g, u, n);
  note_launch();
}

void init_params(float* p, const Layout& lay, uint64_t seed, cudaStream_t s) {
  cudaMemsetAsync(p, 0, lay.total * sizeof(float), s);
  const int gains[3] = {T_LN1G, T_LN2G, T_LNFG};
  for (int t : gains)
    launch_kernel(fill_kernel, grid_for(lay.num[t], 256, 1024), 256, 0, s, p + lay.off[t], lay.num[t], 1.0f);
  InitTable tab;
  tab.n = 0;
  const double sd = 0.02, sd_res = 0.02 / sqrt(2.0 * lay.L);
  const int normals[6] = {T_WTE, T_WPE, T_WQKV, T_WO, T_WFC, T_WP};
  size_t maxc = 0;
  for (int t : normals) {
    InitSeg& sg = tab.seg[tab.n++];
    sg.off = lay.off[t];
    sg.count = (t == T_WTE) ? (size_t)lay.V * lay.C : lay.num[t];  // pad rows stay 0
    // tensor seed = output (t + 1) of the master SplitMix64 seeded with `seed`
    uint64_t z = seed + (uint64_t)(t + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    sg.tseed = z ^ (z >> 31);
    sg.sd = (t == T_WO || t == T_WP) ? sd_res : sd;
    if (sg.count > maxc) maxc = sg.count;
  }
  dim3 grid(grid_for(maxc, 256, 2048), tab.n);
  launch_kernel(init_normal_kernel, grid, 256, 0, s, p, tab);
  note_launch(4);
}

void f32_to_act(act_t* out, const float* in, size_t n, cudaStream_t s) {
  launch_kernel(convert_kernel<act_t, float>, grid_for(n, 256, 4096), 256, 0, s, out, in, n);
  note_launch();
}

void act_to_f32(float* out, const act_t* in, size_t n, cudaStream_t s) {
  launch_kernel(convert_kernel<float, act_t>, grid_for(n, 256, 4096), 256, 0, s, out, in, n);
  note_launch();
}

void grad_norm_clip(float* scalars, const float* g, size_t n, float max_norm, double* partials,
                    cudaStream_t s) {
  launch_kernel(norm_partial_kernel, kNormBlocks, 256, 0, s, partials, g, n);
  launch_kernel(norm_final_kernel, 1, 256, 0, s, scalars, partials, kNormBlocks, max_norm);
  note_launch(2);
}

void grad_sumsq(double* out, const float* g, size_t n, double* partials, cudaStream_t s) {
  launch_kernel(norm_partial_kernel, kNormBlocks, 256, 0, s, partials, g, n);
  launch_kernel(sumsq_final_kernel, 1, 256, 0, s, out, partials, kNormBlocks);
  note_launch(2);
}

void clip_from_sumsq(float* scalars, const double* sumsq, float max_norm, cudaStream_t s) {
  launch_kernel(clip_from_sumsq_kernel, 1, 1, 0, s, scalars, sumsq, max_norm);
  note_launch();
}

void adam_prep(float* scalars, int* step, float lr, bool scheduled, const double* sched, float b1,
               float b2, cudaStream_t s) {
  Sched sc{0.0, 0.0, 1.0, 1.0};
  if (scheduled) sc = Sched{sched[0], sched[1], sched[2], sched[3]};
  launch_kernel(adam_prep_kernel, 1, 1, 0, s, scalars, step, lr, scheduled ? 1 : 0, sc, b1, b2);
  note_launch();
}

void reset_clip(float* scalars, cudaStream_t s) {
  launch_kernel(reset_clip_kernel, 1, 1, 0, s, scalars);
  note_launch();
}

void adamw(float* p, act_t* pact, const float* g, float* m, float* v, const Layout& lay,
           const AdamArgs& a, const float* scalars, cudaStream_t s, size_t begin, size_t end) {
  DecayTable dt;
  dt.n = 0;
  for (int t = 0; t < T_COUNT; ++t)
    if (tensor_decayed(t)) {
      dt.begin[dt.n] = lay.off[t];
      dt.end[dt.n] = lay.off[t] + lay.num[t];
      ++dt.n;
    }
  if (end > lay.total) end = lay.total;
  if (begin >= end) return;
  launch_kernel(adamw_kernel, grid_for((end - begin) / 4, 256, kNumSMs * 8), 256, 0, s, 
      p, pact, g, m, v, begin, end - begin, a, dt, scalars);
  note_launch();
}

}  // namespace gpt2k
