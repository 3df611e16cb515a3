/*
 * gpt2_kernels.h -- kernel-level entry points of the GPT-2 step library.
 *
 * These expose single kernels of the step (the projection GEMM with its
 * fused epilogues, the causal attention forward and backward) so that each
 * can be checked against the CPU oracle and timed on its own.  Operands are
 * device pointers in the library's activation dtype (bf16 in libgpt2.so,
 * fp32 in libgpt2_fp32.so); work is enqueued on `stream` (a cudaStream_t,
 * may be NULL) and is asynchronous.  Return 0 on success, a negative
 * GPT2_ERR_* code (gpt2.h) otherwise.
 */
#ifndef GPT2_B200_KERNELS_H
#define GPT2_B200_KERNELS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogue kinds of gpt2k_gemm. */
#define GPT2K_EPI_STORE 0      /* out = alpha D */
#define GPT2K_EPI_BIAS 1       /* out = alpha D + bias */
#define GPT2K_EPI_BIAS_GELU 2  /* aux = alpha D + bias; out = GELU_tanh(aux) */
#define GPT2K_EPI_BIAS_RESID 3 /* out = resid + alpha D + bias */
#define GPT2K_EPI_DGELU 4      /* out = alpha D * GELU_tanh'(aux) */
#define GPT2K_EPI_F32_ACC 5    /* out32 += alpha D (fp32) */

/* D[m, n] = sum_k A(m, k) B(n, k) for m < M, n < N, k < K, followed by the
 * epilogue.  A(m, k) = A[m lda + k] if a_mn = 0, A[k lda + m] if a_mn = 1;
 * B(n, k) = B[n ldb + k] if b_mn = 0, B[k ldb + n] if b_mn = 1.  This is
 * the projection y = x W^T + b of every GPT-2 layer (forward: a_mn = b_mn =
 * 0), its input gradient (b_mn = 1) and its weight gradient (a_mn = b_mn = 1,
 * EPI_F32_ACC).  Row strides are in elements; in the bf16 build lda and ldb
 * must be multiples of 8 and A, B 16-byte aligned (TMA).  `out`, `resid`,
 * `aux` use the activation dtype with strides ldo, ldr, ldaux; bias and
 * out32 are fp32.  split_ws (may be NULL) is fp32 scratch of split_ws_floats
 * floats that the weight-gradient form may use for a fixed-order split-K
 * reduction.  Supported (a_mn, b_mn, epi) in the bf16 build: (0,0, STORE |
 * BIAS | BIAS_GELU | BIAS_RESID), (0,1, STORE | DGELU), (1,1, F32_ACC),
 * (1,0, STORE). */
int gpt2k_gemm(void* stream, int epi, int M, int N, int K, const void* A, long lda, int a_mn,
               const void* B, long ldb, int b_mn, float alpha, void* out, long ldo, float* out32,
               long ldo32, const float* bias, const void* resid, long ldr, void* aux, long ldaux,
               float* split_ws, size_t split_ws_floats);

/* Causal attention forward over qkv [B*T, 3C] = [q | k | v] (head h in
 * columns h*C/H .. of each part): att [B*T, C], lse [B, H, T] (natural-log
 * log-sum-exp of the scaled scores, fp32). */
int gpt2k_attention_fwd(void* stream, void* att, float* lse, const void* qkv, int B, int T, int C,
                        int H);

/* Its backward: dqkv [B*T, 3C] (overwritten) from datt [B*T, C], the
 * forward's qkv, att and lse; dsum is fp32 scratch of B*H*T floats. */
int gpt2k_attention_bwd(void* stream, void* dqkv, float* dsum, const void* datt, const void* qkv,
                        const void* att, const float* lse, int B, int T, int C, int H);

/* Device error word of the kernel-level calls (bit 2: a bounded wait in a
 * GEMM expired); read and cleared.  Synchronous. */
int gpt2k_take_error(void);

#ifdef __cplusplus
}
#endif

#endif /* GPT2_B200_KERNELS_H */
