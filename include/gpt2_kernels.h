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

/* Test of the bounded waits (no counterpart on the pages): the forward
 * product out[M, N] = A[M, K] B[N, K]^T (store epilogue, row-major, ld = K
 * and N) with CTA 0's TMA producer skipping the load of k-block `kblock` of
 * its first tile, so that the MMA issuer's wait for it runs out after the
 * kernels' wait limit (about 2 s).  The kernel then takes its abort path:
 * the device error word of the kernel-level calls receives bit value 4
 * (read it with gpt2k_take_error), every role leaves its loop, the copies in
 * flight land, TMEM is freed and the kernel returns; `out` holds garbage.
 * The context stays usable.  Never part of the training step. */
int gpt2k_gemm_expiry_test(void* stream, int M, int N, int K, const void* A, const void* B,
                           void* out, int kblock);

/* Whether gpt2k_gemm (and the model's products) run the products with
 * N >= 256 and M > 128 (other than the GELU epilogues, whose pace their
 * epilogue sets) as 256 x 256 tiles over pairs of CTAs on
 * neighbouring SMs (tcgen05 cta_group::2: each CTA stages half of the B
 * tile, halving its shared-memory operand traffic) instead of 128 x 256
 * tiles on single CTAs.  enable = 0 or 1; the default is 1; the fp32
 * validation build has no pairs.  Process-wide, not thread-safe against
 * concurrent launches; returns the previous setting. */
int gpt2k_gemm_set_cta_pairs(int enable);

/* Whether the library's kernels are launched with programmatic stream
 * serialization (programmatic dependent launch): a kernel may then be
 * launched while the kernel before it in the stream is still finishing,
 * its CTAs taking SMs as that kernel's leave and running their set-up
 * (barriers, TMEM allocation) there; each kernel waits
 * (griddepcontrol.wait) for the kernels before it to complete before it
 * touches global memory, so results do not change.  enable = 0 or 1; the
 * default is 1.  Process-wide, applies to launches made after the call
 * (a CUDA graph keeps the setting it was captured with); returns the
 * previous setting. */
int gpt2k_set_programmatic_launch(int enable);

/* Causal attention forward over qkv [B*T, 3C] = [q | k | v] (head h in
 * columns h*C/H .. of each part): att [B*T, C], lse [B, H, T] (natural-log
 * log-sum-exp of the scaled scores, fp32). */
int gpt2k_attention_fwd(void* stream, void* att, float* lse, const void* qkv, int B, int T, int C,
                        int H);

/* Its backward: dqkv [B*T, 3C] (overwritten) from datt [B*T, C], the
 * forward's qkv, att and lse; dsum is 16-byte aligned fp32 scratch of
 * gpt2k_attention_bwd_scratch(B, T, H) floats (per-row softmax statistics:
 * D = rowsum(datt * att) and, for head dim 64, the log-sum-exp beside it,
 * over T rounded up to whole 128-row tiles). */
size_t gpt2k_attention_bwd_scratch(int B, int T, int H);
int gpt2k_attention_bwd(void* stream, void* dqkv, float* dsum, const void* datt, const void* qkv,
                        const void* att, const float* lse, int B, int T, int C, int H);

/* LayerNorm forward over the rows of x [M, C] (first page, layer structure;
 * eps 1e-5, biased variance): y = (x - mean) rstd g + b in the activation
 * dtype, mean and rstd [M] fp32 kept for the backward; g, b fp32 [C].
 * C must be a multiple of 8 and at most 2048; x, y 16-byte aligned. */
int gpt2k_layernorm_fwd(void* stream, void* y, float* mean, float* rstd, const void* x,
                        const float* g, const float* b, int M, int C);

/* Its backward (the chain rule through y): with dxhat = dy g and xhat =
 * (x - mean) rstd, dx = (accumulate ? dx : 0) + rstd (dxhat - mean_c(dxhat)
 * - xhat mean_c(dxhat xhat)); dg += sum_m dy xhat; db += sum_m dy; and, if
 * dsum is not NULL, dsum += sum_m dx as stored (the bias gradient of the
 * projection that produced x's residual).  The column sums add per-block
 * partials in a fixed order (bit-reproducible).  partials is fp32 scratch
 * of gpt2k_layernorm_bwd_scratch(C) floats.  Shape rules as the forward. */
int gpt2k_layernorm_bwd(void* stream, void* dx, const void* dy, const void* x, const float* mean,
                        const float* rstd, const float* g, float* dg, float* db, float* dsum,
                        float* partials, int M, int C, int accumulate);
size_t gpt2k_layernorm_bwd_scratch(int C);

/* Softmax cross-entropy over the rows of logits [M, Vp] (activation dtype),
 * classes 0 .. V-1 (the padded columns V .. Vp-1 are excluded; condensed
 * GPT-2 page, vocabulary padding): losses[m] = logsumexp(z_m[0:V]) -
 * z_m[tgt[m]] (fp32); if write_grad, the logits are overwritten with
 * (softmax - onehot(tgt)) / M for columns < V and 0 for the padding.  A
 * target outside [0, V) is read as 0 and sets error bit value 2.  Vp must
 * be a multiple of 8 and logits 16-byte aligned. */
int gpt2k_classifier(void* stream, void* logits, float* losses, const int* tgt, int M, int V,
                     int Vp, int write_grad);

/* Device error word of the kernel-level calls (bit value 2: a bad target;
 * 4: a bounded wait in a tensor-core kernel expired), ORed with the private
 * error word of gpt2k_gemm_wgrad_noalloc on the current device (calls made
 * with err_dev = NULL); both are read and cleared.  Synchronous. */
int gpt2k_take_error(void);

/* Size, in floats, of the fixed scratch array behind
 * gpt2k_gemm_wgrad_noalloc (16 MiB). */
#define GPT2K_NOALLOC_SCRATCH_FLOATS (4u << 20)

/* The weight-gradient product of gpt2k_gemm (a_mn = b_mn = 1, fp32
 * accumulate: out32[m, n] += alpha * sum_k A[k lda + m] B[k ldb + n]) for
 * callers that cannot give the library device memory.  The pages have no
 * counterpart of this call; it exists for the host side of this library.
 *
 * Who needs it: a caller whose device memory all belongs to its own
 * allocator -- for instance PyTorch's caching allocator, which may already
 * hold nearly all free memory, so that any cudaMalloc made behind its back
 * fails or fragments the pool -- and which therefore cannot hand over a
 * split-K workspace, nor let the library allocate one.
 *
 * What it does instead: the split-K partial sums go to a file-scope device
 * array of GPT2K_NOALLOC_SCRATCH_FLOATS floats.  The call itself makes no
 * cudaMalloc, cudaFree or allocating library routine call.
 *  - Set-up: the first call on a device looks up the array's device address
 *    with that device current.  CUDA loads modules lazily by default, so
 *    that lookup is also when the driver places the 16 MiB array on the
 *    device: the first call needs 16 MiB free.  Make it early -- before the
 *    caller's allocator has taken the memory -- and outside any stream
 *    capture.  From then on the array stays on that device until the
 *    process exits.
 *  - At most max_splits (1..8) K-slices are used; max_splits * M * N must
 *    not exceed GPT2K_NOALLOC_SCRATCH_FLOATS, else GPT2_ERR_ARG is returned
 *    before any work is enqueued.  The result is the same as gpt2k_gemm's
 *    weight-gradient form given a workspace of max_splits * M * N floats.
 *  - Every call on a device shares the one array and leaves its last
 *    partial sums in it; each call writes every partial it later reads.
 *    Calls whose work overlaps on the GPU (other streams, other threads)
 *    race on the array: serialise them.
 *  - err_dev (may be NULL) is a device int that receives bit value 4 if a
 *    bounded wait inside the GEMM expired (the output is then incomplete).
 *    With NULL the bit goes to a private word of the device, which
 *    accumulates until gpt2k_take_error reads and clears it.
 * Operands and strides as for gpt2k_gemm; asynchronous on `stream`. */
int gpt2k_gemm_wgrad_noalloc(void* stream, int M, int N, int K, const void* A, long lda,
                             const void* B, long ldb, float alpha, float* out32, long ldo32,
                             int max_splits, int* err_dev);

#ifdef __cplusplus
}
#endif

#endif /* GPT2_B200_KERNELS_H */
