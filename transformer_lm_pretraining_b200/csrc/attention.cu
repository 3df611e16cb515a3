// Causal multi-head attention, forward and backward, never materialising
// the T x T score matrix.
//
// bf16 build: flash-style kernels on warp-level bf16 tensor-core MMA
// (m16n8k16, fp32 accumulate).  A CTA of 4 warps owns a 64-row tile; K/V
// (or Q/dO) tiles stream through double-buffered shared memory with
// cp.async; the forward keeps an online softmax (running max and sum in
// base 2) and stores the natural-log log-sum-exp per row.  The backward
// recomputes P from the log-sum-exp and is split in two kernels so that no
// gradient needs atomics: one per key tile (dK, dV over all later query
// tiles) and one per query tile (dQ over all earlier key tiles).
//
// Validation build: the same arithmetic in plain fp32, one warp per row.

#include "kernels.h"

namespace gpt2k {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// D[b, h, t] = sum_d dO[t, h*hd + d] * O[t, h*hd + d]
__global__ void attn_rowdot_kernel(float* __restrict__ dsum, const act_t* __restrict__ dout,
                                   const act_t* __restrict__ out, int B, int T, int C, int H) {
  pdl_start();
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)B * T * H) return;
  const int hd = C / H;
  const int h = (int)(i % H);
  const size_t m = i / H;
  const act_t* a = dout + m * C + (size_t)h * hd;
  const act_t* o = out + m * C + (size_t)h * hd;
  float s = 0.f;
  for (int d = 0; d < hd; d += 8) {
    float x[8], y[8];
    load8(a + d, x);
    load8(o + d, y);
#pragma unroll
    for (int k = 0; k < 8; ++k) s += x[k] * y[k];
  }
  const int b = (int)(m / T), t = (int)(m % T);
  dsum[((size_t)b * H + h) * T + t] = s;
}

#if GPT2_ACT_BF16

constexpr int kTile = 64;
constexpr int kWarps = 4;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool pred) {
  const int sz = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(sz)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Tile of 64 rows x HD (bf16) with a 16-byte pad per row.
template <int HD>
struct TileS {
  static constexpr int kStride = HD + 8;
  __nv_bfloat16 d[kTile * kStride];
  __device__ __forceinline__ __nv_bfloat16* row(int r) { return d + r * kStride; }
};

// Async load of rows t0 .. t0+63 (rows >= T are zero-filled) of one head's
// slice: src(t) = base + t * stride.
template <int HD>
__device__ __forceinline__ void load_tile(TileS<HD>& s, const __nv_bfloat16* base, long stride,
                                          int t0, int T) {
  constexpr int kChunks = HD / 8;
  for (int i = threadIdx.x; i < kTile * kChunks; i += kWarps * 32) {
    const int r = i / kChunks, c = (i % kChunks) * 8;
    const int t = t0 + r;
    const bool ok = t < T;
    cp_async16(s.row(r) + c, base + (size_t)(ok ? t : 0) * stride + c, ok);
  }
}

// A fragments (16 rows x HD) of rows r0.. of a tile.
template <int HD>
__device__ __forceinline__ void load_afrag(uint32_t (&f)[HD / 16][4], TileS<HD>& s, int r0) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
#pragma unroll
  for (int kc = 0; kc < HD / 16; ++kc)
    ldsm4(f[kc], s.row(r0 + (lane & 7) + 8 * (mi & 1)) + kc * 16 + 8 * (mi >> 1));
}

// acc[8][4] (16 x 64) += A (16 x HD) * X^T where X is a 64 x HD tile
// (B operand read row-wise: B[k = d][n = row] = X[row][d]).
template <int HD>
__device__ __forceinline__ void mma_abt(float (&acc)[8][4], const uint32_t (&a)[HD / 16][4],
                                        TileS<HD>& x) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
#pragma unroll
  for (int kc = 0; kc < HD / 16; ++kc)
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b[4];
      ldsm4(b, x.row(np * 16 + (lane & 7) + 8 * (mi >> 1)) + kc * 16 + 8 * (mi & 1));
      mma16816(acc[2 * np], a[kc], b[0], b[1]);
      mma16816(acc[2 * np + 1], a[kc], b[2], b[3]);
    }
}

// acc[HD/8][4] (16 x HD) += P (16 x 64, from C-fragment registers) * X where
// X is a 64 x HD tile (B[k = row][n = d] = X[row][d], transposed ldmatrix).
template <int HD>
__device__ __forceinline__ void mma_pv(float (&acc)[HD / 8][4], const float (&p)[8][4],
                                       TileS<HD>& x) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
#pragma unroll
  for (int kc = 0; kc < 4; ++kc) {
    uint32_t a[4];
    a[0] = pack_bf16(p[2 * kc][0], p[2 * kc][1]);
    a[1] = pack_bf16(p[2 * kc][2], p[2 * kc][3]);
    a[2] = pack_bf16(p[2 * kc + 1][0], p[2 * kc + 1][1]);
    a[3] = pack_bf16(p[2 * kc + 1][2], p[2 * kc + 1][3]);
#pragma unroll
    for (int dp = 0; dp < HD / 16; ++dp) {
      uint32_t b[4];
      ldsm4t(b, x.row(kc * 16 + (lane & 7) + 8 * (mi & 1)) + dp * 16 + 8 * (mi >> 1));
      mma16816(acc[2 * dp], a, b[0], b[1]);
      mma16816(acc[2 * dp + 1], a, b[2], b[3]);
    }
  }
}

template <int HD>
struct FwdSmem {
  TileS<HD> q, k[2], v[2];
};

template <int HD>
__global__ void __launch_bounds__(kWarps * 32)
    flash_fwd_kernel(__nv_bfloat16* __restrict__ att, float* __restrict__ lse,
                     const __nv_bfloat16* __restrict__ qkv, int T, int C, int H, float sl2) {
  pdl_start();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FwdSmem<HD>& sm = *reinterpret_cast<FwdSmem<HD>*>(smem_raw);
  const int qb = gridDim.x - 1 - blockIdx.x;  // heaviest tiles first
  const int b = blockIdx.y / H, h = blockIdx.y % H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const long stride = 3L * C;
  const __nv_bfloat16* qb_ = qkv + (size_t)b * T * stride + (size_t)h * HD;
  const int q0 = qb * kTile;

  load_tile<HD>(sm.q, qb_, stride, q0, T);
  load_tile<HD>(sm.k[0], qb_ + C, stride, 0, T);
  load_tile<HD>(sm.v[0], qb_ + 2 * C, stride, 0, T);
  cp_commit();

  uint32_t qf[HD / 16][4];
  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const int nkv = qb + 1;
  for (int j = 0; j < nkv; ++j) {
    const int buf = j & 1;
    if (j + 1 < nkv) {
      load_tile<HD>(sm.k[buf ^ 1], qb_ + C, stride, (j + 1) * kTile, T);
      load_tile<HD>(sm.v[buf ^ 1], qb_ + 2 * C, stride, (j + 1) * kTile, T);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (j == 0) load_afrag<HD>(qf, sm.q, warp * 16);
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
    mma_abt<HD>(s, qf, sm.k[buf]);
    // scale (base 2) and causal mask on the diagonal tile
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * kTile + nt * 8 + 2 * c4 + (e & 1);
        const int qr = q0 + warp * 16 + g + 8 * (e >> 1);
        s[nt][e] = (j == qb && key > qr) ? -INFINITY : s[nt][e] * sl2;
      }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * r], s[nt][2 * r + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(mrow[r], mx);
      const float alpha = fast_exp2(mrow[r] - mnew);
      lrow[r] *= alpha;
#pragma unroll
      for (int dt = 0; dt < HD / 8; ++dt) {
        o[dt][2 * r] *= alpha;
        o[dt][2 * r + 1] *= alpha;
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][2 * r] = fast_exp2(s[nt][2 * r] - mnew);
        s[nt][2 * r + 1] = fast_exp2(s[nt][2 * r + 1] - mnew);
        lrow[r] += s[nt][2 * r] + s[nt][2 * r + 1];
      }
      mrow[r] = mnew;
    }
    mma_pv<HD>(o, s, sm.v[buf]);
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int t = q0 + warp * 16 + g + 8 * r;
    if (t >= T) continue;
    const float inv = 1.f / lrow[r];
    __nv_bfloat16* dst = att + ((size_t)b * T + t) * C + (size_t)h * HD;
#pragma unroll
    for (int dt = 0; dt < HD / 8; ++dt)
      *reinterpret_cast<uint32_t*>(dst + dt * 8 + 2 * c4) =
          pack_bf16(o[dt][2 * r] * inv, o[dt][2 * r + 1] * inv);
    if (c4 == 0) lse[((size_t)b * H + h) * T + t] = (mrow[r] + log2f(lrow[r])) / kLog2e;
  }
}

template <int HD>
struct BwdSmem {
  TileS<HD> a, bb;        // K, V (dK/dV kernel) or Q, dO (dQ kernel)
  TileS<HD> x[2], y[2];   // streamed: Q, dO  or  K, V
  float r0[2][kTile], r1[2][kTile];  // streamed per-row lse*log2e and D
};

__device__ __forceinline__ void load_rows(float* dst, const float* src, int t0, int T, float mul) {
  for (int i = threadIdx.x; i < kTile; i += kWarps * 32) {
    const int t = t0 + i;
    dst[i] = t < T ? src[t] * mul : 0.f;
  }
}

// dK, dV for one key tile: loops over query tiles i >= j.
template <int HD>
__global__ void __launch_bounds__(kWarps * 32)
    flash_bwd_dkdv_kernel(__nv_bfloat16* __restrict__ dqkv, const __nv_bfloat16* __restrict__ qkv,
                          const __nv_bfloat16* __restrict__ dout, const float* __restrict__ lse,
                          const float* __restrict__ dsum, int T, int C, int H, float sl2,
                          float scale) {
  pdl_start();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BwdSmem<HD>& sm = *reinterpret_cast<BwdSmem<HD>*>(smem_raw);
  const int j = blockIdx.x;
  const int nq = gridDim.x;
  const int b = blockIdx.y / H, h = blockIdx.y % H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const long stride = 3L * C;
  const __nv_bfloat16* base = qkv + (size_t)b * T * stride + (size_t)h * HD;
  const __nv_bfloat16* dob = dout + (size_t)b * T * C + (size_t)h * HD;
  const float* lse_bh = lse + ((size_t)b * H + h) * T;
  const float* d_bh = dsum + ((size_t)b * H + h) * T;
  const int k0 = j * kTile;

  load_tile<HD>(sm.a, base + C, stride, k0, T);       // K
  load_tile<HD>(sm.bb, base + 2 * C, stride, k0, T);  // V
  load_tile<HD>(sm.x[0], base, stride, k0, T);        // Q of tile i = j
  load_tile<HD>(sm.y[0], dob, C, k0, T);              // dO
  load_rows(sm.r0[0], lse_bh, k0, T, kLog2e);
  load_rows(sm.r1[0], d_bh, k0, T, 1.f);
  cp_commit();

  uint32_t kf[HD / 16][4], vf[HD / 16][4];
  float dk[HD / 8][4], dv[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;

  for (int i = j; i < nq; ++i) {
    const int buf = (i - j) & 1;
    if (i + 1 < nq) {
      const int t1 = (i + 1) * kTile;
      load_tile<HD>(sm.x[buf ^ 1], base, stride, t1, T);
      load_tile<HD>(sm.y[buf ^ 1], dob, C, t1, T);
      load_rows(sm.r0[buf ^ 1], lse_bh, t1, T, kLog2e);
      load_rows(sm.r1[buf ^ 1], d_bh, t1, T, 1.f);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (i == j) {
      load_afrag<HD>(kf, sm.a, warp * 16);
      load_afrag<HD>(vf, sm.bb, warp * 16);
    }
    // S^T (16 keys x 64 queries) = K Q^T
    float st[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a) st[a][0] = st[a][1] = st[a][2] = st[a][3] = 0.f;
    mma_abt<HD>(st, kf, sm.x[buf]);
    // P^T = exp2(S^T * sl2 - lse2[q]), causal: q >= key
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ql = nt * 8 + 2 * c4 + (e & 1);
        const int q = i * kTile + ql;
        const int key = k0 + warp * 16 + g + 8 * (e >> 1);
        const bool live = q < T && q >= key;
        st[nt][e] = live ? fast_exp2(st[nt][e] * sl2 - sm.r0[buf][ql]) : 0.f;
      }
    // dV += P^T dO
    mma_pv<HD>(dv, st, sm.y[buf]);
    // dP^T (16 keys x 64 queries) = V dO^T
    float dpt[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a) dpt[a][0] = dpt[a][1] = dpt[a][2] = dpt[a][3] = 0.f;
    mma_abt<HD>(dpt, vf, sm.y[buf]);
    // dS^T = P^T (dP^T - D[q])
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ql = nt * 8 + 2 * c4 + (e & 1);
        dpt[nt][e] = st[nt][e] * (dpt[nt][e] - sm.r1[buf][ql]);
      }
    // dK += dS^T Q
    mma_pv<HD>(dk, dpt, sm.x[buf]);
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int t = k0 + warp * 16 + g + 8 * r;
    if (t >= T) continue;
    __nv_bfloat16* dst = dqkv + ((size_t)b * T + t) * stride + (size_t)h * HD;
#pragma unroll
    for (int dt = 0; dt < HD / 8; ++dt) {
      *reinterpret_cast<uint32_t*>(dst + C + dt * 8 + 2 * c4) =
          pack_bf16(dk[dt][2 * r] * scale, dk[dt][2 * r + 1] * scale);
      *reinterpret_cast<uint32_t*>(dst + 2 * C + dt * 8 + 2 * c4) =
          pack_bf16(dv[dt][2 * r], dv[dt][2 * r + 1]);
    }
  }
}

// dQ for one query tile: loops over key tiles j <= i.
template <int HD>
__global__ void __launch_bounds__(kWarps * 32)
    flash_bwd_dq_kernel(__nv_bfloat16* __restrict__ dqkv, const __nv_bfloat16* __restrict__ qkv,
                        const __nv_bfloat16* __restrict__ dout, const float* __restrict__ lse,
                        const float* __restrict__ dsum, int T, int C, int H, float sl2,
                        float scale) {
  pdl_start();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BwdSmem<HD>& sm = *reinterpret_cast<BwdSmem<HD>*>(smem_raw);
  const int i = gridDim.x - 1 - blockIdx.x;  // heaviest tiles first
  const int b = blockIdx.y / H, h = blockIdx.y % H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const long stride = 3L * C;
  const __nv_bfloat16* base = qkv + (size_t)b * T * stride + (size_t)h * HD;
  const __nv_bfloat16* dob = dout + (size_t)b * T * C + (size_t)h * HD;
  const float* lse_bh = lse + ((size_t)b * H + h) * T;
  const float* d_bh = dsum + ((size_t)b * H + h) * T;
  const int q0 = i * kTile;

  load_tile<HD>(sm.a, base, stride, q0, T);   // Q
  load_tile<HD>(sm.bb, dob, C, q0, T);        // dO
  load_tile<HD>(sm.x[0], base + C, stride, 0, T);      // K
  load_tile<HD>(sm.y[0], base + 2 * C, stride, 0, T);  // V
  cp_commit();

  float lse2[2], drow[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int t = q0 + warp * 16 + g + 8 * r;
    lse2[r] = t < T ? lse_bh[t] * kLog2e : 0.f;
    drow[r] = t < T ? d_bh[t] : 0.f;
  }
  uint32_t qf[HD / 16][4], dof[HD / 16][4];
  float dq[HD / 8][4];
#pragma unroll
  for (int a = 0; a < HD / 8; ++a) dq[a][0] = dq[a][1] = dq[a][2] = dq[a][3] = 0.f;

  for (int j = 0; j <= i; ++j) {
    const int buf = j & 1;
    if (j + 1 <= i) {
      const int t1 = (j + 1) * kTile;
      load_tile<HD>(sm.x[buf ^ 1], base + C, stride, t1, T);
      load_tile<HD>(sm.y[buf ^ 1], base + 2 * C, stride, t1, T);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
      load_afrag<HD>(qf, sm.a, warp * 16);
      load_afrag<HD>(dof, sm.bb, warp * 16);
    }
    float s[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a) s[a][0] = s[a][1] = s[a][2] = s[a][3] = 0.f;
    mma_abt<HD>(s, qf, sm.x[buf]);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * kTile + nt * 8 + 2 * c4 + (e & 1);
        const int qr = q0 + warp * 16 + g + 8 * (e >> 1);
        const bool live = key <= qr && qr < T;
        s[nt][e] = live ? fast_exp2(s[nt][e] * sl2 - lse2[e >> 1]) : 0.f;
      }
    float dp[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a) dp[a][0] = dp[a][1] = dp[a][2] = dp[a][3] = 0.f;
    mma_abt<HD>(dp, dof, sm.y[buf]);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) dp[nt][e] = s[nt][e] * (dp[nt][e] - drow[e >> 1]);
    mma_pv<HD>(dq, dp, sm.x[buf]);
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int t = q0 + warp * 16 + g + 8 * r;
    if (t >= T) continue;
    __nv_bfloat16* dst = dqkv + ((size_t)b * T + t) * stride + (size_t)h * HD;
#pragma unroll
    for (int dt = 0; dt < HD / 8; ++dt)
      *reinterpret_cast<uint32_t*>(dst + dt * 8 + 2 * c4) =
          pack_bf16(dq[dt][2 * r] * scale, dq[dt][2 * r + 1] * scale);
  }
}

template <int HD>
cudaError_t fwd_launch(act_t* att, float* lse, const act_t* qkv, int B, int T, int C, int H,
                       cudaStream_t s) {
  const size_t smem = sizeof(FwdSmem<HD>);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(flash_fwd_kernel<HD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const float sl2 = kLog2e / sqrtf((float)HD);
  dim3 grid((T + kTile - 1) / kTile, B * H);
  launch_kernel(flash_fwd_kernel<HD>, grid, kWarps * 32, smem, s, att, lse, qkv, T, C, H, sl2);
  note_launch();
  return cudaGetLastError();
}

template <int HD>
cudaError_t bwd_launch(act_t* dqkv, float* dsum, const act_t* datt, const act_t* qkv,
                       const float* lse, int B, int T, int C, int H, cudaStream_t s) {
  const size_t smem = sizeof(BwdSmem<HD>);
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(flash_bwd_dkdv_kernel<HD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(flash_bwd_dq_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const float sl2 = kLog2e / sqrtf((float)HD);
  const float scale = 1.f / sqrtf((float)HD);
  dim3 grid((T + kTile - 1) / kTile, B * H);
  launch_kernel(flash_bwd_dkdv_kernel<HD>, grid, kWarps * 32, smem, s, dqkv, qkv, datt, lse, dsum, T, C, H,
                                                             sl2, scale);
  launch_kernel(flash_bwd_dq_kernel<HD>, grid, kWarps * 32, smem, s, dqkv, qkv, datt, lse, dsum, T, C, H,
                                                           sl2, scale);
  note_launch(2);
  return cudaGetLastError();
}

#else  // validation build: fp32, one warp per row

constexpr int kMaxT = 2048;

// Scores of row (b, h, i) against keys 0..i into sc (shared), then softmax.
__global__ void naive_fwd_kernel(float* __restrict__ att, float* __restrict__ lse,
                                 const float* __restrict__ qkv, int B, int T, int C, int H) {
  pdl_start();
  extern __shared__ float sc_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x / 32) + warp;  // over B*H*T
  if (row >= B * H * T) return;
  float* sc = sc_all + (size_t)warp * T;
  const int i = row % T, h = (row / T) % H, b = row / (T * H);
  const int hd = C / H;
  const float scale = 1.f / sqrtf((float)hd);
  const float* q = qkv + ((size_t)b * T + i) * 3 * C + (size_t)h * hd;
  float mx = -INFINITY;
  for (int j = 0; j <= i; ++j) {
    const float* k = qkv + ((size_t)b * T + j) * 3 * C + C + (size_t)h * hd;
    float d = 0.f;
    for (int e = lane; e < hd; e += 32) d += q[e] * k[e];
    d = warp_sum(d) * scale;
    if (lane == 0) sc[j] = d;
    mx = fmaxf(mx, d);
  }
  __syncwarp();
  float z = 0.f;
  for (int j = lane; j <= i; j += 32) z += expf(sc[j] - mx);
  z = warp_sum(z);
  float* y = att + ((size_t)b * T + i) * C + (size_t)h * hd;
  for (int e = lane; e < hd; e += 32) {
    float acc = 0.f;
    for (int j = 0; j <= i; ++j)
      acc += expf(sc[j] - mx) / z * qkv[((size_t)b * T + j) * 3 * C + 2 * C + (size_t)h * hd + e];
    y[e] = acc;
  }
  if (lane == 0) lse[((size_t)b * H + h) * T + i] = mx + logf(z);
}

// dQ for row i: dq = scale sum_j p_ij (dp_ij - D_i) k_j
__global__ void naive_bwd_dq_kernel(float* __restrict__ dqkv, const float* __restrict__ qkv,
                                    const float* __restrict__ dout, const float* __restrict__ lse,
                                    const float* __restrict__ dsum, int B, int T, int C, int H) {
  pdl_start();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x / 32) + warp;
  if (row >= B * H * T) return;
  const int i = row % T, h = (row / T) % H, b = row / (T * H);
  const int hd = C / H;
  const float scale = 1.f / sqrtf((float)hd);
  const float* q = qkv + ((size_t)b * T + i) * 3 * C + (size_t)h * hd;
  const float* dy = dout + ((size_t)b * T + i) * C + (size_t)h * hd;
  const float L = lse[((size_t)b * H + h) * T + i];
  const float D = dsum[((size_t)b * H + h) * T + i];
  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // hd <= 128
  for (int j = 0; j <= i; ++j) {
    const float* k = qkv + ((size_t)b * T + j) * 3 * C + C + (size_t)h * hd;
    const float* v = k + C;
    float s = 0.f, dp = 0.f;
    for (int e = lane; e < hd; e += 32) {
      s += q[e] * k[e];
      dp += dy[e] * v[e];
    }
    s = warp_sum(s);
    dp = warp_sum(dp);
    const float p = expf(s * scale - L);
    const float ds = p * (dp - D);
    for (int e = lane, u = 0; e < hd; e += 32, ++u) acc[u] += ds * k[e];
  }
  float* dq = dqkv + ((size_t)b * T + i) * 3 * C + (size_t)h * hd;
  for (int e = lane, u = 0; e < hd; e += 32, ++u) dq[e] = acc[u] * scale;
}

// dK, dV for key row j: sums over query rows i >= j
__global__ void naive_bwd_dkdv_kernel(float* __restrict__ dqkv, const float* __restrict__ qkv,
                                      const float* __restrict__ dout,
                                      const float* __restrict__ lse,
                                      const float* __restrict__ dsum, int B, int T, int C, int H) {
  pdl_start();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x / 32) + warp;
  if (row >= B * H * T) return;
  const int j = row % T, h = (row / T) % H, b = row / (T * H);
  const int hd = C / H;
  const float scale = 1.f / sqrtf((float)hd);
  const float* k = qkv + ((size_t)b * T + j) * 3 * C + C + (size_t)h * hd;
  const float* v = k + C;
  float dk[4] = {0.f, 0.f, 0.f, 0.f}, dv[4] = {0.f, 0.f, 0.f, 0.f};
  for (int i = j; i < T; ++i) {
    const float* q = qkv + ((size_t)b * T + i) * 3 * C + (size_t)h * hd;
    const float* dy = dout + ((size_t)b * T + i) * C + (size_t)h * hd;
    float s = 0.f, dp = 0.f;
    for (int e = lane; e < hd; e += 32) {
      s += q[e] * k[e];
      dp += dy[e] * v[e];
    }
    s = warp_sum(s);
    dp = warp_sum(dp);
    const float p = expf(s * scale - lse[((size_t)b * H + h) * T + i]);
    const float ds = p * (dp - dsum[((size_t)b * H + h) * T + i]);
    for (int e = lane, u = 0; e < hd; e += 32, ++u) {
      dv[u] += p * dy[e];
      dk[u] += ds * q[e];
    }
  }
  float* dst = dqkv + ((size_t)b * T + j) * 3 * C + (size_t)h * hd;
  for (int e = lane, u = 0; e < hd; e += 32, ++u) {
    dst[C + e] = dk[u] * scale;
    dst[2 * C + e] = dv[u];
  }
}

#endif

}  // namespace

cudaError_t attention_fwd(act_t* att, float* lse, const act_t* qkv, int B, int T, int C, int H,
                          int* err, cudaStream_t s) {
  const int hd = C / H;
#if GPT2_ACT_BF16
  switch (hd) {
    case 32: return fwd_launch<32>(att, lse, qkv, B, T, C, H, s);
    case 64: return attention_fwd_tc(att, lse, qkv, B, T, C, H, err, s);  // tcgen05
    case 128: return fwd_launch<128>(att, lse, qkv, B, T, C, H, s);
    default: return cudaErrorInvalidValue;
  }
#else
  if (hd > 128 || T > kMaxT) return cudaErrorInvalidValue;
  const int warps = 4;
  const size_t rows = (size_t)B * H * T;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(naive_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         warps * kMaxT * 4);
    attr = true;
  }
  launch_kernel(naive_fwd_kernel, (unsigned)((rows + warps - 1) / warps), warps * 32, warps * T * sizeof(float),
                     s, att, lse, qkv, B, T, C, H);
  note_launch();
  return cudaGetLastError();
#endif
}

size_t attention_bwd_scratch_floats(int B, int T, int H) {
  size_t n = (size_t)B * H * T;  // D = rowsum(dO * O) of every row
#if GPT2_ACT_BF16
  const size_t tc = attention_bwd_tc_scratch_floats(B, T, H);
  if (tc > n) n = tc;
#endif
  return n;
}

cudaError_t attention_bwd(act_t* dqkv, float* dsum, const act_t* datt, const act_t* qkv,
                          const act_t* att, const float* lse, int B, int T, int C, int H,
                          int* err, cudaStream_t s) {
  const int hd = C / H;
#if GPT2_ACT_BF16
  // the tcgen05 kernels form D themselves (head dim 64)
  if (hd == 64) return attention_bwd_tc(dqkv, dsum, datt, qkv, att, lse, B, T, C, H, err, s);
#endif
  const size_t n = (size_t)B * T * H;
  launch_kernel(attn_rowdot_kernel, (unsigned)((n + 255) / 256), 256, 0, s, dsum, datt, att, B, T, C, H);
  note_launch();
#if GPT2_ACT_BF16
  switch (hd) {
    case 32: return bwd_launch<32>(dqkv, dsum, datt, qkv, lse, B, T, C, H, s);
    case 128: return bwd_launch<128>(dqkv, dsum, datt, qkv, lse, B, T, C, H, s);
    default: return cudaErrorInvalidValue;
  }
#else
  if (hd > 128) return cudaErrorInvalidValue;
  const int warps = 4;
  const size_t rows = (size_t)B * H * T;
  const unsigned grid = (unsigned)((rows + warps - 1) / warps);
  launch_kernel(naive_bwd_dq_kernel, grid, warps * 32, 0, s, dqkv, qkv, datt, lse, dsum, B, T, C, H);
  launch_kernel(naive_bwd_dkdv_kernel, grid, warps * 32, 0, s, dqkv, qkv, datt, lse, dsum, B, T, C, H);
  note_launch(2);
  return cudaGetLastError();
#endif
}

}  // namespace gpt2k
