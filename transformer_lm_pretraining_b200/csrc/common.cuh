// Shared device helpers of the GPT-2 step kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#ifdef GPT2_FP32_VALIDATE
typedef float act_t;  // validation build: every activation in fp32
#define GPT2_ACT_BF16 0
#else
typedef __nv_bfloat16 act_t;  // product build: bf16 activations
#define GPT2_ACT_BF16 1
#endif

namespace gpt2k {

constexpr int kNumSMs = 148;

// Programmatic dependent launch.  Every kernel of the library starts with
// pdl_launch_dependents() (the kernel that follows it in the stream may be
// launched as soon as every CTA of this one has started, so its CTAs take
// SMs as this grid's CTAs leave and run their set-up, barriers and TMEM
// allocation, there) and calls pdl_wait() before its first access to global
// memory (it returns once the grids this one depends on have completed and
// their writes are visible; at once when the launch had no programmatic
// dependency).  So the launch latency and prologue of each kernel overlap
// the tail of the one before, and no data is read or written early.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_start() {
  pdl_launch_dependents();
  pdl_wait();
}

// Whether launches carry the programmatic-serialization attribute (default
// on; gpt2k_set_programmatic_launch).
bool pdl_enabled();

// kern<<<grid, block, smem, s>>>(args...) with the programmatic-serialization
// attribute when enabled (and a cluster of `cluster` CTAs along x when > 1).
template <typename... P, typename... A>
cudaError_t launch_kernel_cluster(void (*kern)(P...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t s, int cluster, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  int n = 0;
  if (pdl_enabled()) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = (unsigned)cluster;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = (unsigned)n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<A&&>(args)...);
}
template <typename... P, typename... A>
cudaError_t launch_kernel(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          A&&... args) {
  return launch_kernel_cluster(kern, grid, block, smem, s, 1, static_cast<A&&>(args)...);
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <class T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// 2^x with the hardware approximation (one special-function op, relative
// error ~2^-22, subnormal results flushed to 0); -inf gives 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): output n of the generator
// seeded with s is mix(s + n * 0x9E3779B97F4A7C15).
__host__ __device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__host__ __device__ __forceinline__ uint64_t sm64_out(uint64_t seed, uint64_t n) {
  return sm64_mix(seed + n * 0x9E3779B97F4A7C15ull);
}

// 8 consecutive activations <-> 8 floats (16 B of bf16 or 32 B of fp32).
__device__ __forceinline__ void load8(const float* p, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void store8(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* v) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

// Two fp32 lanes per instruction: sm_100's packed add, sub, mul and fma on f32x2.
// Each lane rounds as the scalar instruction does, so a packed sequence gives
// the same bits as the same scalar sequence, with half the instructions.
__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mov.b64 c, {%6, %7};\n\tfma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 f2_splat(float x) { return make_float2(x, x); }
// Elements i, i + 1 of a register array as a pair, and back.
__device__ __forceinline__ float2 get2(const float* v, int i) { return make_float2(v[i], v[i + 1]); }
__device__ __forceinline__ void set2(float* v, int i, float2 x) {
  v[i] = x.x;
  v[i + 1] = x.y;
}

// GPT-2's GELU: 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3), and
// its derivative (the tanh form named on the condensed GPT-2 page).
#if GPT2_ACT_BF16
// bf16 build: the same function through the identity 0.5 (1 + tanh(u)) =
// 1 / (1 + exp(-2u)) = 1 / (1 + 2^(-2 u log2 e)), with the constants folded
// so that x (1 + 2^(x (a + b x^2)))^-1 takes three multiply-adds and two
// special-function ops (ex2, rcp).  Where 2^(...) overflows to +inf the
// reciprocal is 0 and the result the limit, -0.  Accurate to a few fp32
// ulps even where 1 + tanh(u) is tiny; these epilogues are instruction-bound,
// so the count matters.
__device__ __forceinline__ float rcp_hw(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
namespace gelu_c {
constexpr float kA = -2.0f * 0.7978845608028654f * 1.4426950408889634f;  // -2 sqrt(2/pi) log2 e
constexpr float kB = kA * 0.044715f;
constexpr float k = 0.7978845608028654f;  // sqrt(2/pi)
constexpr float kc = k * 0.044715f;
constexpr float d0 = -0.5f * k, d1 = -1.5f * kc;  // d = d0 + d1 x^2
}  // namespace gelu_c
__device__ __forceinline__ float gelu_tanh(float x) {
  using namespace gelu_c;
  return x * rcp_hw(1.0f + fast_exp2(x * fmaf(x * x, kB, kA)));
}
// The derivative uses the hardware tanh (tanh.approx.f32, one special-function
// op; relative error about 2^-11, so GELU'(x) is off by at most about one
// bf16 ulp, the precision its product is stored in):
//   GELU'(x) = 0.5 (1 + t) + 0.5 x (1 - t^2) du/dx,  t = tanh(u),
//   du/dx = sqrt(2/pi) (1 + 3 * 0.044715 x^2),
// evaluated as 0.5 t + 0.5 + x d (t^2 - 1) with d = -du/dx / 2, so that every
// step is one multiply or multiply-add with a constant operand.
__device__ __forceinline__ float tanh_hw(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float gelu_tanh_grad(float x) {
  using namespace gelu_c;
  const float x2 = x * x;
  const float t = tanh_hw(x * fmaf(x2, kc, k));
  const float q = fmaf(t, t, -1.0f);
  const float xd = x * fmaf(x2, d1, d0);
  return fmaf(xd, q, fmaf(t, 0.5f, 0.5f));
}

// gelu_tanh and gelu_tanh_grad on two values (bit-identical to the scalar
// forms).
__device__ __forceinline__ float2 gelu_tanh2(float2 x) {
  using namespace gelu_c;
  const float2 a = f2_mul(x, f2_fma(f2_mul(x, x), f2_splat(kB), f2_splat(kA)));
  const float2 d = f2_add(make_float2(fast_exp2(a.x), fast_exp2(a.y)), f2_splat(1.0f));
  return f2_mul(x, make_float2(rcp_hw(d.x), rcp_hw(d.y)));
}
__device__ __forceinline__ float2 gelu_tanh_grad2(float2 x) {
  using namespace gelu_c;
  const float2 x2 = f2_mul(x, x);
  const float2 a = f2_mul(x, f2_fma(x2, f2_splat(kc), f2_splat(k)));
  const float2 t = make_float2(tanh_hw(a.x), tanh_hw(a.y));
  const float2 q = f2_fma(t, t, f2_splat(-1.0f));
  const float2 xd = f2_mul(x, f2_fma(x2, f2_splat(d1), f2_splat(d0)));
  return f2_fma(xd, q, f2_fma(t, f2_splat(0.5f), f2_splat(0.5f)));
}
#else
__device__ __forceinline__ float gelu_tanh(float x) {
  const float k = 0.7978845608028654f;
  return 0.5f * x * (1.0f + tanhf(k * (x + 0.044715f * x * x * x)));
}
__device__ __forceinline__ float gelu_tanh_grad(float x) {
  const float k = 0.7978845608028654f;
  const float th = tanhf(k * (x + 0.044715f * x * x * x));
  const float dinner = k * (1.0f + 3.0f * 0.044715f * x * x);
  return 0.5f * (1.0f + th) + 0.5f * x * (1.0f - th * th) * dinner;
}
__device__ __forceinline__ float2 gelu_tanh2(float2 x) { return make_float2(gelu_tanh(x.x), gelu_tanh(x.y)); }
__device__ __forceinline__ float2 gelu_tanh_grad2(float2 x) {
  return make_float2(gelu_tanh_grad(x.x), gelu_tanh_grad(x.y));
}
#endif

}  // namespace gpt2k
