// GEMM epilogues: bias, GELU (keeping the pre-activation), residual add,
// GELU backward and fp32 (accumulating) stores.
#pragma once

#include "kernels.h"

namespace gpt2k {

struct EpiParams {
  int M, N;
  float alpha;
  act_t* out; long ldo;
  float* out32; long ldo32;
  const float* bias;
  const act_t* resid; long ldr;
  act_t* aux; long ldaux;
  int expiry_test;  // GemmArgs::expiry_test
  float* colsum;    // GemmArgs::colsum
};

// One output element (any epilogue kind).
template <int EPI>
__device__ __forceinline__ void epi_scalar(const EpiParams& e, int m, int n, float acc) {
  float v = acc * e.alpha;
  if (EPI == EPI_F32_ACC) {
    e.out32[(size_t)m * e.ldo32 + n] += v;
    return;
  }
  if (EPI == EPI_F32_STORE) {
    e.out32[(size_t)m * e.ldo32 + n] = v;
    return;
  }
  if (EPI == EPI_DGELU) {
    v *= gelu_tanh_grad(to_f(e.aux[(size_t)m * e.ldaux + n]));
    e.out[(size_t)m * e.ldo + n] = from_f<act_t>(v);
    return;
  }
  if (EPI == EPI_BIAS || EPI == EPI_BIAS_GELU || EPI == EPI_BIAS_RESID) {
    if (e.bias) v += e.bias[n];
  }
  if (EPI == EPI_BIAS_RESID) v += to_f(e.resid[(size_t)m * e.ldr + n]);
  if (EPI == EPI_BIAS_GELU) {  // GELU of u as stored, so that it can be recomputed from u
    const act_t u = from_f<act_t>(v);
    e.aux[(size_t)m * e.ldaux + n] = u;
    v = gelu_tanh(to_f(u));
  }
  e.out[(size_t)m * e.ldo + n] = from_f<act_t>(v);
}

// 32 consecutive outputs n0 .. n0+31 of row m (n0 % 32 == 0).  Vectorised
// when the whole run is in range and the leading dimensions keep 16-byte
// alignment (checked by the launcher); otherwise element by element.
template <int EPI>
__device__ __forceinline__ void epi_row32(const EpiParams& e, int m, int n0, float* v,
                                          bool vec_ok) {
  if (!(vec_ok && n0 + 32 <= e.N)) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (n0 + i < e.N) epi_scalar<EPI>(e, m, n0 + i, v[i]);
    return;
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] *= e.alpha;
  if (EPI == EPI_F32_ACC || EPI == EPI_F32_STORE) {
    float* o = e.out32 + (size_t)m * e.ldo32 + n0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float4 w = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      if (EPI == EPI_F32_ACC) {
        const float4 old = reinterpret_cast<const float4*>(o)[j];
        w.x += old.x; w.y += old.y; w.z += old.z; w.w += old.w;
      }
      reinterpret_cast<float4*>(o)[j] = w;
    }
    return;
  }
  if (EPI == EPI_DGELU) {
    const act_t* a = e.aux + (size_t)m * e.ldaux + n0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float u[8];
      load8(a + 8 * j, u);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[8 * j + i] *= gelu_tanh_grad(u[i]);
    }
  } else {
    if ((EPI == EPI_BIAS || EPI == EPI_BIAS_GELU || EPI == EPI_BIAS_RESID) && e.bias) {
      const float4* b4 = reinterpret_cast<const float4*>(e.bias + n0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 b = b4[j];
        v[4 * j] += b.x; v[4 * j + 1] += b.y; v[4 * j + 2] += b.z; v[4 * j + 3] += b.w;
      }
    }
    if (EPI == EPI_BIAS_RESID) {
      const act_t* r = e.resid + (size_t)m * e.ldr + n0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float x[8];
        load8(r + 8 * j, x);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[8 * j + i] += x[i];
      }
    }
    if (EPI == EPI_BIAS_GELU) {  // GELU of u as stored, so that it can be recomputed from u
      act_t* a = e.aux + (size_t)m * e.ldaux + n0;
#pragma unroll
      for (int j = 0; j < 4; ++j) store8(a + 8 * j, v + 8 * j);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = gelu_tanh(to_f(from_f<act_t>(v[i])));
    }
  }
  act_t* o = e.out + (size_t)m * e.ldo + n0;
#pragma unroll
  for (int j = 0; j < 4; ++j) store8(o + 8 * j, v + 8 * j);
}

// out32[i] += sum_s ws[s * stride + i], s ascending.
__global__ void splitk_reduce_kernel(float* out32, long ldo32, const float* ws, int splits,
                                     int M, int N);

}  // namespace gpt2k
