// fp32 GEMM for the validation build (no tensor cores): 64x64 tiles staged
// through shared memory, each thread computing a 4x4 block in fp32, with the
// same epilogues as the tensor-core kernel.

#include "gemm_epi.cuh"

namespace gpt2k {

namespace {

constexpr int TS = 64;  // tile size in M and N
constexpr int TK = 16;

template <int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const float* __restrict__ A, long lda,
                                                        int a_mn, const float* __restrict__ B,
                                                        long ldb, int b_mn, int K, EpiParams ep,
                                                        int k_begin_stride, long split_stride) {
  pdl_start();
  __shared__ float sA[TK][TS + 1];
  __shared__ float sB[TK][TS + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * TS, n0 = blockIdx.x * TS;
  const int split = blockIdx.z;
  const int kb = split * k_begin_stride;
  const int ke = min(K, kb + k_begin_stride);
  float acc[4][4] = {};
  for (int k0 = kb; k0 < ke; k0 += TK) {
    for (int i = threadIdx.x; i < TK * TS; i += 256) {
      int kk, mm;
      if (a_mn) { mm = i % TS; kk = i / TS; } else { kk = i % TK; mm = i / TK; }
      const int m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < ep.M && k < ke) v = a_mn ? A[(size_t)k * lda + m] : A[(size_t)m * lda + k];
      sA[kk][mm] = v;
    }
    for (int i = threadIdx.x; i < TK * TS; i += 256) {
      int kk, nn;
      if (b_mn) { nn = i % TS; kk = i / TS; } else { kk = i % TK; nn = i / TK; }
      const int n = n0 + nn, k = k0 + kk;
      float v = 0.f;
      if (n < ep.N && k < ke) v = b_mn ? B[(size_t)k * ldb + n] : B[(size_t)n * ldb + k];
      sB[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sA[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sB[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  EpiParams e = ep;
  if (EPI == EPI_F32_STORE) e.out32 += (size_t)split * split_stride;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < ep.M && n < ep.N) epi_scalar<EPI>(e, m, n, acc[i][j]);
    }
}

}  // namespace

__global__ void splitk_reduce_kernel(float* out32, long ldo32, const float* ws, int splits, int M,
                                     int N) {
  pdl_start();
  const size_t total = (size_t)M * N;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(i / N), n = (int)(i % N);
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += ws[(size_t)k * total + i];
    out32[(size_t)m * ldo32 + n] += s;
  }
}

int gemm_set_cta_pairs(int) { return 0; }  // the fp32 validation library has no CTA pairs
bool gemm_colsum_supported() { return false; }  // the column sums run as their own pass

cudaError_t gemm(const GemmArgs& a, cudaStream_t s, int* err) {
  if (a.M2 > 0) {  // the stacked second product: one launch after the other
    GemmArgs first = a;
    first.M2 = 0;
    const cudaError_t e = gemm(first, s, err);
    if (e != cudaSuccess) return e;
    return gemm(gemm_second(a), s, err);
  }
  (void)err;
  if (a.M <= 0 || a.N <= 0 || a.K <= 0) return cudaSuccess;
  EpiParams ep{a.M, a.N, a.alpha, a.out, a.ldo, a.out32, a.ldo32, a.bias, a.resid, a.ldr, a.aux, a.ldaux};
  const int tiles = ((a.M + TS - 1) / TS) * ((a.N + TS - 1) / TS);
  int splits = 1;
  int epi = a.epi;
  if (a.epi == EPI_F32_ACC && a.max_splits > 1 && a.split_ws) {
    splits = (4 * 148 + tiles - 1) / tiles;
    if (splits > a.max_splits) splits = a.max_splits;
    if (splits > a.K / 256) splits = a.K / 256;
    while (splits > 1 && (size_t)splits * a.M * a.N > a.split_ws_floats) --splits;
    if (splits < 1) splits = 1;
  }
  int kchunk = (a.K + splits - 1) / splits;
  kchunk = (kchunk + TK - 1) / TK * TK;
  splits = (a.K + kchunk - 1) / kchunk;
  long split_stride = 0;
  if (splits > 1) {
    epi = EPI_F32_STORE;
    ep.out32 = a.split_ws;
    ep.ldo32 = a.N;
    split_stride = (long)a.M * a.N;
  }
  dim3 grid((a.N + TS - 1) / TS, (a.M + TS - 1) / TS, splits);
  switch (epi) {
#define GPT2_SIMT(E)                                                                               \
  case E:                                                                                          \
    launch_kernel(gemm_simt_kernel<E>, grid, 256, 0, s, a.A, a.lda, a.a_mn, a.B, a.ldb, a.b_mn, a.K, ep, kchunk, \
                                             split_stride);                                        \
    break;
    GPT2_SIMT(EPI_STORE)
    GPT2_SIMT(EPI_BIAS)
    GPT2_SIMT(EPI_BIAS_GELU)
    GPT2_SIMT(EPI_BIAS_RESID)
    GPT2_SIMT(EPI_DGELU)
    GPT2_SIMT(EPI_F32_ACC)
    GPT2_SIMT(EPI_F32_STORE)
#undef GPT2_SIMT
    default:
      return cudaErrorInvalidValue;
  }
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (splits > 1) {
    const size_t total = (size_t)a.M * a.N;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 1184) blocks = 1184;
    launch_kernel(splitk_reduce_kernel, blocks, 256, 0, s, a.out32, a.ldo32, a.split_ws, splits, a.M, a.N);
    note_launch();
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace gpt2k
