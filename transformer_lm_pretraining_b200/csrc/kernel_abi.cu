// Kernel-level C entry points (include/gpt2_kernels.h).

#include "../../include/gpt2.h"
#include "../../include/gpt2_kernels.h"
#include "kernels.h"

using namespace gpt2k;

namespace {

int* err_word() {
  static int* e = nullptr;
  if (!e) {
    if (cudaMalloc(&e, sizeof(int)) != cudaSuccess) return nullptr;
    cudaMemset(e, 0, sizeof(int));
  }
  return e;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int status(cudaError_t e) { return e == cudaSuccess ? GPT2_OK : (e == cudaErrorInvalidValue ? GPT2_ERR_ARG : GPT2_ERR_CUDA); }

}  // namespace

extern "C" {

int gpt2k_gemm_set_cta_pairs(int enable) { return gemm_set_cta_pairs(enable); }

int gpt2k_set_programmatic_launch(int enable) { return set_pdl(enable); }

int gpt2k_gemm(void* stream, int epi, int M, int N, int K, const void* A, long lda, int a_mn,
               const void* B, long ldb, int b_mn, float alpha, void* out, long ldo, float* out32,
               long ldo32, const float* bias, const void* resid, long ldr, void* aux, long ldaux,
               float* split_ws, size_t split_ws_floats) {
  if (M < 0 || N < 0 || K < 0 || epi < 0 || epi > EPI_F32_ACC) return GPT2_ERR_ARG;
  int* err = err_word();
  if (!err) return GPT2_ERR_CUDA;
  GemmArgs g{};
  g.M = M; g.N = N; g.K = K;
  g.A = static_cast<const act_t*>(A); g.lda = lda; g.a_mn = a_mn;
  g.B = static_cast<const act_t*>(B); g.ldb = ldb; g.b_mn = b_mn;
  g.epi = epi; g.alpha = alpha;
  g.out = static_cast<act_t*>(out); g.ldo = ldo;
  g.out32 = out32; g.ldo32 = ldo32;
  g.bias = bias;
  g.resid = static_cast<const act_t*>(resid); g.ldr = ldr;
  g.aux = static_cast<act_t*>(aux); g.ldaux = ldaux;
  g.split_ws = split_ws; g.split_ws_floats = split_ws_floats;
  g.max_splits = split_ws ? 8 : 1;
  return status(gemm(g, static_cast<cudaStream_t>(stream), err));
}

int gpt2k_gemm_expiry_test(void* stream, int M, int N, int K, const void* A, const void* B,
                           void* out, int kblock) {
  if (M < 1 || N < 1 || K < 1 || kblock < 0 || kblock >= (K + 63) / 64) return GPT2_ERR_ARG;
  int* err = err_word();
  if (!err) return GPT2_ERR_CUDA;
  GemmArgs g{};
  g.M = M; g.N = N; g.K = K;
  g.A = static_cast<const act_t*>(A); g.lda = K;
  g.B = static_cast<const act_t*>(B); g.ldb = K;
  g.epi = EPI_STORE; g.alpha = 1.f;
  g.out = static_cast<act_t*>(out); g.ldo = N;
  g.max_splits = 1;
  g.expiry_test = kblock + 1;
  return status(gemm(g, static_cast<cudaStream_t>(stream), err));
}

int gpt2k_attention_fwd(void* stream, void* att, float* lse, const void* qkv, int B, int T, int C,
                        int H) {
  if (B < 1 || T < 1 || H < 1 || C % H) return GPT2_ERR_ARG;
  int* err = err_word();
  if (!err) return GPT2_ERR_CUDA;
  return status(attention_fwd(static_cast<act_t*>(att), lse, static_cast<const act_t*>(qkv), B, T,
                              C, H, err, static_cast<cudaStream_t>(stream)));
}

size_t gpt2k_attention_bwd_scratch(int B, int T, int H) {
  if (B < 1 || T < 1 || H < 1) return 0;
  return attention_bwd_scratch_floats(B, T, H);
}

int gpt2k_attention_bwd(void* stream, void* dqkv, float* dsum, const void* datt, const void* qkv,
                        const void* att, const float* lse, int B, int T, int C, int H) {
  if (B < 1 || T < 1 || H < 1 || C % H) return GPT2_ERR_ARG;
  int* err = err_word();
  if (!err) return GPT2_ERR_CUDA;
  return status(attention_bwd(static_cast<act_t*>(dqkv), dsum, static_cast<const act_t*>(datt),
                              static_cast<const act_t*>(qkv), static_cast<const act_t*>(att), lse,
                              B, T, C, H, err, static_cast<cudaStream_t>(stream)));
}

int gpt2k_layernorm_fwd(void* stream, void* y, float* mean, float* rstd, const void* x,
                        const float* g, const float* b, int M, int C) {
  if (M < 0 || C < 8 || C > 2048 || C % 8 || !aligned16(x) || !aligned16(y)) return GPT2_ERR_ARG;
  if (M == 0) return GPT2_OK;
  layernorm_fwd(static_cast<act_t*>(y), mean, rstd, static_cast<const act_t*>(x), g, b, M, C,
                static_cast<cudaStream_t>(stream));
  return status(cudaGetLastError());
}

size_t gpt2k_layernorm_bwd_scratch(int C) { return (size_t)kLnBlocks * 3 * (C > 0 ? C : 0); }

int gpt2k_layernorm_bwd(void* stream, void* dx, const void* dy, const void* x, const float* mean,
                        const float* rstd, const float* g, float* dg, float* db, float* dsum,
                        float* partials, int M, int C, int accumulate) {
  if (M < 0 || C < 8 || C > 2048 || C % 8 || !aligned16(x) || !aligned16(dy) || !aligned16(dx) ||
      !partials)
    return GPT2_ERR_ARG;
  if (M == 0) return GPT2_OK;
  layernorm_bwd(static_cast<act_t*>(dx), static_cast<const act_t*>(dy),
                static_cast<const act_t*>(x), mean, rstd, g, dg, db, dsum, partials, M, C,
                accumulate ? 1 : 0, static_cast<cudaStream_t>(stream));
  return status(cudaGetLastError());
}

int gpt2k_classifier(void* stream, void* logits, float* losses, const int* tgt, int M, int V,
                     int Vp, int write_grad) {
  if (M < 0 || V < 1 || Vp < V || Vp % 8 || !aligned16(logits)) return GPT2_ERR_ARG;
  if (M == 0) return GPT2_OK;
  int* err = err_word();
  if (!err) return GPT2_ERR_CUDA;
  classifier(static_cast<act_t*>(logits), losses, tgt, M, V, Vp, write_grad ? 1 : 0, err,
             static_cast<cudaStream_t>(stream));
  return status(cudaGetLastError());
}

int gpt2k_take_error(void) {
  int* err = err_word();
  if (!err) return GPT2_ERR_CUDA;
  int e = 0;
  if (cudaMemcpy(&e, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GPT2_ERR_CUDA;
  cudaMemset(err, 0, sizeof(int));
  return e | noalloc_take_error();
}

}  // extern "C"
