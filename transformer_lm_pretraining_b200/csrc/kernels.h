// Launch interface of the GPT-2 step kernels (internal to the library).
#pragma once

#include "common.cuh"

namespace gpt2k {

// ------------------------------------------------------------- layout --
// Flat parameter order (one slice per tensor, row-major, y = x W^T + b).
enum Tensor {
  T_WTE, T_WPE, T_LN1G, T_LN1B, T_WQKV, T_BQKV, T_WO, T_BO, T_LN2G, T_LN2B,
  T_WFC, T_BFC, T_WP, T_BP, T_LNFG, T_LNFB, T_COUNT
};

struct Layout {
  int L, H, C, V, Vp, Tmax;
  size_t off[T_COUNT];
  size_t num[T_COUNT];
  size_t total;
};

Layout make_layout(int L, int H, int C, int V, int Vp, int Tmax);
bool tensor_decayed(int t);

// ---------------------------------------------------------------- GEMM --
// D[m, n] = alpha * sum_k A(m, k) B(n, k), then the epilogue.
//   A(m, k) = A[m * lda + k]  (a_mn = 0, "K-major")  or A[k * lda + m] (a_mn = 1)
//   B(n, k) = B[n * ldb + k]  (b_mn = 0)             or B[k * ldb + n] (b_mn = 1)
enum Epi {
  EPI_STORE = 0,       // out = D
  EPI_BIAS = 1,        // out = D + bias[n]
  EPI_BIAS_GELU = 2,   // aux = D + bias[n]; out = gelu(aux)
  EPI_BIAS_RESID = 3,  // out = resid + D + bias[n]
  EPI_DGELU = 4,       // out = D * gelu'(aux)
  EPI_F32_ACC = 5,     // out32 += D
  EPI_F32_STORE = 6,   // out32 = D
};

struct GemmArgs {
  int M, N, K;
  const act_t* A; long lda; int a_mn;
  const act_t* B; long ldb; int b_mn;
  int epi;
  float alpha;
  act_t* out; long ldo;
  float* out32; long ldo32;
  const float* bias;
  const act_t* resid; long ldr;
  act_t* aux; long ldaux;
  // split-K (EPI_F32_ACC only): partial sums go to split_ws, then a
  // fixed-order reduction adds them into out32.  max_splits = 1 disables.
  float* split_ws; size_t split_ws_floats; int max_splits;
  // EPI_F32_ACC: out32 is known to hold zeros.  A split in two may then add
  // both partials straight into out32 (TMA reduce-add, no workspace, no
  // reduction kernel): 0 + a + b is the same float in either order (and the
  // reduction's 0 + (a + b)), so the result stays deterministic.
  int acc_zero;
  // Test of the bounded waits only: n > 0 makes CTA 0's producer skip the
  // load of k-block n - 1 of its first tile, so that the MMA's wait for it
  // expires (error word ERR_TIMEOUT) and the kernel takes its abort path.
  // 0 (the value of a zero-initialised GemmArgs) in every product call.
  int expiry_test;
  // EPI_DGELU (when gemm_colsum_supported()): if set, colsum[s * N + n] =
  // the sum of the stored (bf16) output over rows 32 s .. 32 s + 31 of
  // column n, added in row order; [ceil(M / 32)][N] floats, N even,
  // 16-byte aligned.  The bias gradient of the product whose output gradient
  // this is, without a second pass over it.
  float* colsum;
  // EPI_F32_ACC with A and B MN-major: a second product with the same N and
  // K, out32_2 += alpha * A2^T B2 over M2 rows, launched with this one where
  // the tiles allow (M2 = 0: none).  Its accumulator holds zeros exactly
  // when out32's does (acc_zero).
  int M2;
  const act_t* A2; long lda2;
  const act_t* B2; long ldb2;
  float* out32_2; long ldo32_2;
};
// The second product of a, as a product of its own.
inline GemmArgs gemm_second(const GemmArgs& a) {
  GemmArgs b = a;
  b.M = a.M2; b.M2 = 0;
  b.A = a.A2; b.lda = a.lda2;
  b.B = a.B2; b.ldb = a.ldb2;
  b.out32 = a.out32_2; b.ldo32 = a.ldo32_2;
  return b;
}
bool gemm_colsum_supported();

cudaError_t gemm(const GemmArgs& a, cudaStream_t s, int* err_flag);
// Whether wide products run as 256 x 256 tiles over CTA pairs (default on;
// the fp32 build has no pairs).  Returns the previous setting.
int gemm_set_cta_pairs(int enable);

// ------------------------------------------------------------- encoder --
// x0[m, :] = wte[tok[m], :] + wpe[m % T, :]; saves the (range-checked)
// tokens for the backward pass; bad ids set err bit 1 and read row 0.
void encoder_fwd(act_t* x0, int* tok_saved, const int* tok, const act_t* wte,
                 const act_t* wpe, int B, int T, int C, int V, int* err, cudaStream_t s);

struct EncoderScratch {
  int* keys[2];     // [M] each
  int* vals[2];     // [M] each
  int* hist;        // [256 * ceil(M / 1024)]
  float* partial;   // [M * C]
};
size_t encoder_scratch_bytes(int M, int C);
void encoder_scratch_carve(EncoderScratch* es, void* base, int M, int C);

// dwpe[t, :] += sum_b dx0[b T + t, :];  dwte[v, :] += sum_{m: tok[m] = v} dx0[m, :]
// in ascending m (stable radix sort by token, fixed-chunk partial sums).
void encoder_bwd(float* dwte, float* dwpe, const act_t* dx0, const int* tok_saved,
                 int B, int T, int C, int Vp, const EncoderScratch& es, cudaStream_t s);

// ----------------------------------------------------------- layernorm --
void layernorm_fwd(act_t* y, float* mean, float* rstd, const act_t* x, const float* g,
                   const float* b, int M, int C, cudaStream_t s);
// dres = (accumulate ? dres : 0) + LN backward of dy;  dg, db += column sums
// of dy * xhat and dy; dbias_out (may be null) += column sums of the written
// dres.  Per-block partials in `partials` [kLnBlocks * 3C], reduced in a
// fixed order.
constexpr int kLnBlocks = 592;
// The second stage of a two-stage reduction, described instead of launched:
// dst[j][c] += sum over rows r < nrows of partials[r * nsums * C + j * C + c]
// for j < nsums (dst[j] null: skipped), in the fixed order of `kind`
// (REDUCE_LN: the layernorm backward's; REDUCE_COLSUM: colsum_reduce's), so
// that a deferred reduction gives the same bits as the immediate one.
enum ReduceKind { REDUCE_LN = 0, REDUCE_COLSUM = 1 };
struct ReduceJob {
  float* dst[3];
  const float* partials;
  int nrows, nsums, C, kind;
};
constexpr int kMaxReduceJobs = 64;
struct ReduceJobs {
  int n;
  int group_end[kMaxReduceJobs];  // blocks of jobs 0..k (32 columns per block)
  ReduceJob job[kMaxReduceJobs];
};
// Adds a job to the list (false when the list is full).
bool reduce_jobs_add(ReduceJobs& jobs, const ReduceJob& j);
// Runs every job of the list in one launch and empties it.
void reduce_jobs_run(ReduceJobs& jobs, cudaStream_t s);

// With `defer` set, only the first stage runs and *defer describes the
// second (the partials must then stay untouched until it has run).
void layernorm_bwd(act_t* dres, const act_t* dy, const act_t* x, const float* mean,
                   const float* rstd, const float* g, float* dg, float* db, float* dbias_out,
                   float* partials, int M, int C, int accumulate, cudaStream_t s,
                   ReduceJob* defer = nullptr);

// ------------------------------------------------------------ column sums --
constexpr int kColsumChunks = 192;
// db[n] += sum_m dy[m, n] (fixed order); partials: [kColsumChunks * N] floats
void colsum_acc(float* db, const act_t* dy, int M, int N, float* partials, cudaStream_t s,
                ReduceJob* defer = nullptr);
// db[n] += sum over c < chunks of partials[c * N + n], c ascending (the
// second stage of colsum_acc, for partials a GEMM epilogue wrote)
void colsum_reduce(float* db, const float* partials, int chunks, int N, cudaStream_t s,
                   ReduceJob* defer = nullptr);

// ----------------------------------------------------------- attention --
// qkv [B*T, 3C] = [q | k | v], head h at columns h*hd..; att [B*T, C];
// lse [B, H, T] (natural log).
cudaError_t attention_fwd(act_t* att, float* lse, const act_t* qkv, int B, int T, int C, int H,
                          int* err, cudaStream_t s);
// tcgen05 forward (head dim 64; bf16 build)
bool attention_fwd_tc_supported(int C, int H);
cudaError_t attention_fwd_tc(act_t* att, float* lse, const act_t* qkv, int B, int T, int C, int H,
                             int* err, cudaStream_t s);
// dqkv [B*T, 3C] (overwritten); dsum: fp32 scratch of
// attention_bwd_scratch_floats(B, T, H) floats, 16-byte aligned.
size_t attention_bwd_scratch_floats(int B, int T, int H);
cudaError_t attention_bwd(act_t* dqkv, float* dsum, const act_t* datt, const act_t* qkv,
                          const act_t* att, const float* lse, int B, int T, int C, int H,
                          int* err, cudaStream_t s);
// tcgen05 backward (head dim 64; bf16 build); it forms D = rowsum(dO * O)
// itself, from datt and the forward's output att, and keeps the per-row
// (L log2 e, D) pairs in `scratch` (attention_bwd_tc_scratch_floats floats:
// B*H rows of T rounded up to 128 pairs)
size_t attention_bwd_tc_scratch_floats(int B, int T, int H);
cudaError_t attention_bwd_tc(act_t* dqkv, float* scratch, const act_t* datt, const act_t* qkv,
                             const act_t* att, const float* lse, int B, int T, int C, int H,
                             int* err, cudaStream_t s);

// ---------------------------------------------------------- classifier --
// In place over logits [M, Vp]: per row lse over the first V columns,
// losses[m] = lse - z[tgt[m]], and (write_grad != 0) z <- (softmax(z) -
// onehot(tgt)) / M for columns < V, 0 for the padded columns.  Bad targets
// set err bit 2.
void classifier(act_t* logits, float* losses, const int* tgt, int M, int V, int Vp, int write_grad,
                int* err, cudaStream_t s);
// out[0] = mean of losses[0..M) (fixed-order reduction)
void mean_loss(float* out, const float* losses, int M, cudaStream_t s);

// ------------------------------------------------------------ generation --
// Positions: each of these works at p, or at p + *p_dev when p_dev is given
// (a device position counter, so that one decode step can be captured once
// and replayed as a CUDA graph).
// x[b] = wte[tok[b * ld_tok + p]] + wpe[p] for b < B (bad ids: ERR_TOKEN, read as 0)
void decode_embed(act_t* x, const int* tok, int ld_tok, int p, const int* p_dev, const act_t* wte,
                  const act_t* wpe, int B, int C, int V, int* err, cudaStream_t s);
// att[b] = causal attention of the single query q[b] over the first n
// cached positions kv[b][0..n) ([b][Ttot][2C] rows of [k | v]); C / H <= 128
void decode_attention(act_t* att, const act_t* q, const act_t* kv, int Ttot, int n,
                      const int* p_dev, int B, int C, int H, cudaStream_t s);
// tok[b * ld_tok + p_out] = the next token drawn from the V logits of row
// b (greedy at temperature 0; else top-k tempered softmax at the SplitMix64
// uniform of (seed, p_out * 65536 + b)); logits_out (may be null): rows
// [p_out - out_p0][B][V] fp32
void sample_tokens(int* tok, int ld_tok, int p_out, const int* p_dev, const act_t* logits,
                   long ld_logits, int B, int V, float temperature, int top_k, uint64_t seed,
                   float* logits_out, int out_p0, cudaStream_t s);
// cache[b][p] = kvnew[b] (rows of 2C: [k | v]; cache [b][Ttot][2C])
void kv_append(act_t* cache, const act_t* kvnew, int p, const int* p_dev, int Ttot, int B, int C,
               cudaStream_t s);
// *p_dev += 1
void pos_advance(int* p_dev, cudaStream_t s);

// g = GELU_tanh(u) elementwise (n elements, activation dtype); the same
// function the fc GEMM's epilogue applies to the stored u.
void gelu_fwd(act_t* g, const act_t* u, size_t n, cudaStream_t s);

// ----------------------------------------------------------- optimizer --
void init_params(float* p, const Layout& lay, uint64_t seed, cudaStream_t s);
void f32_to_act(act_t* out, const float* in, size_t n, cudaStream_t s);
void act_to_f32(float* out, const act_t* in, size_t n, cudaStream_t s);

// scalars layout (device floats)
enum Scalar { S_NORM = 0, S_CLIP = 1, S_LOSS = 2, S_LR = 3, S_BC1 = 4, S_BC2 = 5, S_COUNT = 16 };
constexpr int kNormBlocks = 592;
// scalars[S_NORM] = ||g||_2, scalars[S_CLIP] = max_norm / (norm + 1e-6) or 1
void grad_norm_clip(float* scalars, const float* g, size_t n, float max_norm, double* partials,
                    cudaStream_t s);

// scalars[S_NORM] = 0, scalars[S_CLIP] = 1 (no clipping pending)
void reset_clip(float* scalars, cudaStream_t s);

struct AdamArgs {
  float b1, b2, eps, wd;  // the learning rate and bias corrections are device scalars
};

// The optimizer step counter and its learning rate, on the device: t =
// ++*step; scalars[S_LR] = lr, or with `scheduled` the warmup-then-cosine
// schedule lr(t - 1) (sched = {max_lr, min_lr, warmup, max_steps});
// scalars[S_BC1] = 1 - b1^t, scalars[S_BC2] = 1 - b2^t.
void adam_prep(float* scalars, int* step, float lr, bool scheduled, const double* sched, float b1,
               float b2, cudaStream_t s);
// Decay applies to the tensors flagged in `decay_mask` (bit per tensor).
// over the flat parameter range [begin, end) (begin and end - begin multiples
// of 4 unless end is the total)
void adamw(float* p, act_t* pact, const float* g, float* m, float* v, const Layout& lay,
           const AdamArgs& a, const float* scalars, cudaStream_t s, size_t begin, size_t end);
// *out = sum of g[i]^2 over n elements (fixed-order two-stage reduction in double)
void grad_sumsq(double* out, const float* g, size_t n, double* partials, cudaStream_t s);
// scalars[S_NORM] = sqrt(*sumsq), scalars[S_CLIP] as grad_norm_clip
void clip_from_sumsq(float* scalars, const double* sumsq, float max_norm, cudaStream_t s);

// Programmatic dependent launch of every kernel (default on); returns the
// previous setting.
int set_pdl(int enable);

// Process-wide count of kernel launches made by this library.
void note_launch(int n = 1);
long launch_count();

// Error bits in the device error word.
enum ErrBits { ERR_TOKEN = 1, ERR_TARGET = 2, ERR_TIMEOUT = 4 };

// Error bits left by gpt2k_gemm_wgrad_noalloc calls made without an error
// word of their own, on the current device; read and cleared (synchronous).
int noalloc_take_error();

}  // namespace gpt2k
