/*
 * gpt2.h -- C ABI of the B200-native GPT-2 pretraining step.
 *
 * One handle holds one decoder-only GPT-2 (tied token embedding / LM head,
 * learned positions, pre-LayerNorm, causal multi-head attention, 4C tanh-GELU
 * MLP, softmax cross-entropy over a vocabulary padded to a multiple of 64)
 * and its optimiser state.  The step the calls below make up is the one the
 * pages describe: forward, backward (accumulated over micro-batches with the
 * loss divided by the number of micro-batches), global-norm gradient clipping
 * at 1.0, and AdamW with beta = (0.9, 0.95), eps = 1e-8 and weight decay 0.1
 * on 2-D parameters only, driven by a warmup-then-cosine LR schedule
 * ("Let's reproduce GPT-2 (124M)" condensed, sections 1-3; "TinyStories
 * training", the training excerpt).
 *
 * Conventions for every call:
 *  - Pointers named *_dev are device pointers; *_host are host pointers.
 *  - All device work is enqueued on the handle's stream (gpt2_set_stream;
 *    default: the legacy default stream) and is asynchronous, except where a
 *    host out-pointer is given: then the call synchronises the stream.
 *  - Every call that can fail returns a gpt2_status: 0 on success, a
 *    negative GPT2_ERR_* code otherwise; gpt2_last_error() gives the text.
 *  - Memory: the caller owns the device memory it binds with
 *    gpt2_bind_memory (e.g. allocated by PyTorch).  If nothing is bound when
 *    the first call needs memory, the library allocates it with cudaMalloc
 *    and frees it in gpt2_destroy.
 *  - Precision (this library build): parameters, gradients and AdamW moments
 *    are fp32; activations, the GEMM weight copies and the logits are bf16;
 *    LayerNorm statistics, the attention log-sum-exp and every reduction are
 *    fp32.  The validation build (libgpt2_fp32.so) keeps everything in fp32
 *    and uses no tensor cores.
 *  - Determinism: no call uses floating-point atomics; two runs with the
 *    same inputs give bit-identical parameters, gradients and losses.
 */
#ifndef GPT2_B200_H
#define GPT2_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gpt2 gpt2_t;
typedef int gpt2_status;

#define GPT2_OK 0
#define GPT2_ERR_ARG (-1)       /* bad shape or argument */
#define GPT2_ERR_STATE (-2)     /* call out of order or memory not bound */
#define GPT2_ERR_TOKEN (-3)     /* a token or target outside [0, V) */
#define GPT2_ERR_NONFINITE (-4) /* loss or gradient norm is not finite */
#define GPT2_ERR_CUDA (-5)      /* a CUDA runtime error */
#define GPT2_ERR_TIMEOUT (-6)   /* a kernel's bounded wait expired */

/* Build variant: 1 for the bf16 tensor-core build, 0 for the fp32 validation
 * build. */
int gpt2_build_is_bf16(void);

/* Create a model.  L layers, H heads, width C (C % H == 0, C % 8 == 0,
 * head dim C/H in {32, 64, 128}), vocabulary V padded to Vpad (Vpad >= V,
 * Vpad % 64 == 0), context Tmax.  Parameters are initialised on the device
 * at the first gpt2_bind_memory/allocation: N(0, 0.02) for wte (rows < V),
 * wpe, W_qkv and W_fc; N(0, 0.02/sqrt(2L)) for the residual projections W_o
 * and W_p (condensed GPT-2 page, section 1); LayerNorm gains 1; biases, LN
 * betas and the padded wte rows 0.  Normals come from a counter-based
 * SplitMix64 + Box-Muller generator keyed by (seed, tensor, element).
 * Errors: GPT2_ERR_ARG on a bad shape. */
gpt2_status gpt2_create(int L, int H, int C, int V, int Vpad, int Tmax, uint64_t seed,
                        gpt2_t** out);
void gpt2_destroy(gpt2_t* h);

/* Number of parameters in the flat buffer (including the Vpad - V padded
 * wte rows): 12 L C^2 + 13 L C + 2 C + Vpad C + Tmax C. */
size_t gpt2_num_params(const gpt2_t* h);

/* Device bytes for the persistent state (fp32 params, grads, m, v, the bf16
 * weight copy and a few scalars). */
size_t gpt2_state_bytes(const gpt2_t* h);

/* Device bytes of workspace (activations kept for the backward pass, logits,
 * backward scratch) for micro-batches of B sequences of length T. */
size_t gpt2_workspace_bytes(const gpt2_t* h, int B, int T);

/* Bind caller-owned device memory: dev_state (>= gpt2_state_bytes) and
 * dev_work (>= gpt2_workspace_bytes for the largest B,T used later).  Both
 * must be 256-byte aligned.  Binding new state memory re-initialises the
 * parameters from the seed and zeroes grads, moments and the step count.
 * dev_state may be NULL to keep the current state; dev_work may be NULL to
 * keep the current workspace. */
gpt2_status gpt2_bind_memory(gpt2_t* h, void* dev_state, size_t state_bytes, void* dev_work,
                             size_t work_bytes);

/* Activation recompute (the recompute option of the first page's training
 * loop): level 1 keeps no GELU output per layer (one layer's buffer is
 * reused) and the backward recomputes GELU(u) from the stored pre-activation
 * u before the projection's weight gradient; level 0 (the default) keeps
 * them.  Results are bit-identical at both levels (the forward applies GELU
 * to u as stored).  Level 1 shrinks gpt2_workspace_bytes by (L-1) B T 4C
 * activations; set it before sizing and binding the workspace.  Errors:
 * GPT2_ERR_ARG (level not 0 or 1). */
gpt2_status gpt2_set_recompute(gpt2_t* h, int level);

/* Stream (a cudaStream_t) on which every later call enqueues its work. */
gpt2_status gpt2_set_stream(gpt2_t* h, void* cuda_stream);

/* Forward pass over tok_dev [B, T] (int32, row-major, values in [0, V)).
 * With tgt_dev (int32 [B, T]) it also computes the mean softmax
 * cross-entropy over the B*T positions (padded logits excluded) and leaves in
 * the logits buffer the gradient of that mean loss w.r.t. the logits, ready
 * for gpt2_backward.  loss_host (may be NULL) receives the mean loss and
 * makes the call synchronous; tokens are then also validated (GPT2_ERR_TOKEN;
 * out-of-range ids are read as id 0 on the device, never out of bounds).
 * Without targets the logits [B*T, Vpad] stay in the workspace (see
 * gpt2_logits).  Errors: GPT2_ERR_ARG (T > Tmax, workspace too small),
 * GPT2_ERR_STATE (no memory), GPT2_ERR_TOKEN, GPT2_ERR_NONFINITE. */
gpt2_status gpt2_forward(gpt2_t* h, const int32_t* tok_dev, const int32_t* tgt_dev, int B, int T,
                         float* loss_host);

/* Forward-only evaluation (the validation loop of the TinyStories page and
 * the evaluation of the condensed GPT-2 page): the forward of gpt2_forward
 * with targets, giving the same per-position and mean losses, but the
 * logits [B*T, Vpad] are left as computed (no gradient is written into
 * them) and no gpt2_backward may follow (GPT2_ERR_STATE until the next
 * forward with targets).  B*T may be anything up to what the workspace was
 * sized for.  loss_host (may be NULL) receives the mean loss and makes the
 * call synchronous; the perplexity is exp(loss).  Errors as gpt2_forward. */
gpt2_status gpt2_evaluate(gpt2_t* h, const int32_t* tok_dev, const int32_t* tgt_dev, int B, int T,
                          float* loss_host);

/* Autoregressive generation with a key/value cache (the sampling loop of
 * the pages).  tok_dev is a device int32 buffer [B][T_total] whose first
 * T_prompt columns hold the prompts; the call fills columns T_prompt ..
 * T_total-1, one token per position: the forward over the prompts (as
 * gpt2_forward without targets) leaves their keys and values in a cache,
 * then each new position runs one-position layers against it.  Each token
 * is drawn from the logits over the first V classes: temperature 0 takes
 * the argmax (lowest index among equal maxima); otherwise the softmax of
 * logits / temperature over the top_k largest logits (top_k <= 0: all; ties
 * at the k-th value kept) is inverted at the uniform draw u = (SplitMix64
 * output n = position * 65536 + row of `seed`) >> 11, times 2^-53.
 * step_logits (may be NULL) is device fp32 [T_total - T_prompt][B][V] and
 * receives the logits each token was drawn from.  The cache and the
 * one-position buffers are device memory the library allocates and keeps
 * until gpt2_destroy; the forward record afterwards holds the prompts (no
 * gpt2_backward).  With a stream set (gpt2_set_stream) and profiling off,
 * the decode steps after the first replay one captured CUDA graph (the step
 * reads its position from a device counter); the results are the same as
 * with plain launches.  Asynchronous.  Errors: GPT2_ERR_ARG (T_prompt < 1,
 * T_total <= T_prompt or > Tmax, head dim above 128), GPT2_ERR_CUDA. */
gpt2_status gpt2_generate(gpt2_t* h, int32_t* tok_dev, int B, int T_prompt, int T_total,
                          float temperature, int top_k, uint64_t seed, float* step_logits);

/* Mean loss of the last forward with targets, read back to the host
 * (synchronises the stream). */
gpt2_status gpt2_read_loss(gpt2_t* h, float* loss_host);

/* Zero the gradient buffer. */
gpt2_status gpt2_zero_grad(gpt2_t* h);

/* Backward pass of the preceding forward (which must have had targets, at
 * the same B, T): adds d(loss_scale * mean loss)/d(params) into the fp32
 * gradient buffer.  Use loss_scale = 1/n_micro to accumulate n_micro
 * micro-batches (condensed GPT-2 page, section 3).  Errors: GPT2_ERR_STATE
 * (no forward with targets since the last backward). */
gpt2_status gpt2_backward(gpt2_t* h, float loss_scale);

/* Global L2 norm n of all gradients (fixed-order two-stage reduction); when
 * n > max_norm every gradient is to be scaled by max_norm / (n + 1e-6).  The
 * scale is kept on the device and applied inside gpt2_adamw_step.
 * norm_host (may be NULL) receives n and makes the call synchronous; a
 * non-finite n then returns GPT2_ERR_NONFINITE (and AdamW skips the update
 * on the device whatever the caller does). */
gpt2_status gpt2_grad_norm_clip(gpt2_t* h, float max_norm, float* norm_host);

/* One AdamW step on every parameter (t += 1; bias-corrected moments;
 * p -= lr (mhat / (sqrt(vhat) + eps) + wd p) with wd applied to the 2-D
 * tensors wte, wpe, W_qkv, W_o, W_fc, W_p only), using the clip scale of the
 * last gpt2_grad_norm_clip (1 if none since the last step).  Refreshes the
 * bf16 weight copy.  Gradients are left as they are.  The step counter t
 * lives on the device (gpt2_get_state reads it). */
gpt2_status gpt2_adamw_step(gpt2_t* h, float lr, float beta1, float beta2, float eps,
                            float weight_decay);

/* The same step with lr = gpt2_lr(t - 1, max_lr, min_lr, warmup, max_steps)
 * evaluated on the device from its own step counter (after t += 1), so that
 * a captured step (gpt2_step_graph_capture) follows the schedule when it is
 * replayed.  warmup >= 1. */
gpt2_status gpt2_adamw_step_scheduled(gpt2_t* h, double max_lr, double min_lr, long warmup,
                                      long max_steps, float beta1, float beta2, float eps,
                                      float weight_decay);

/* One whole optimizer step captured as a CUDA graph owned by the handle and
 * replayed with gpt2_step_graph_launch, in place of the ~370 separate
 * launches of the eager calls (the graph is uploaded to the device here,
 * on the model's stream): gpt2_zero_grad; for i < n_micro,
 * gpt2_forward(tok_dev + i B T, tgt_dev + i B T, B, T) and
 * gpt2_backward(1 / n_micro); gpt2_grad_norm_clip(max_norm);
 * gpt2_adamw_step_scheduled(...).  tok_dev and tgt_dev (n_micro B T ids
 * each) are read at every replay: write the next step's tokens there before
 * launching it.  Capturing runs no kernel.  Requirements: a stream set with
 * gpt2_set_stream (not the legacy default stream), profiling off, and one
 * eager step of the same B and T run before (first-use set-up of the kernels
 * is not captured).  A new capture replaces the previous graph.
 * gpt2_step_graph_kernels gives the number of kernels one replay runs. */
gpt2_status gpt2_step_graph_capture(gpt2_t* h, const int32_t* tok_dev, const int32_t* tgt_dev,
                                    int B, int T, int n_micro, float max_norm, double max_lr,
                                    double min_lr, long warmup, long max_steps, float beta1,
                                    float beta2, float eps, float weight_decay);
gpt2_status gpt2_step_graph_launch(gpt2_t* h);
long gpt2_step_graph_kernels(const gpt2_t* h);

/* Host-side schedule: lr = max_lr (step+1)/warmup for step < warmup, then a
 * cosine from max_lr at step = warmup to min_lr at step = max_steps, and
 * min_lr after (condensed GPT-2 page, section 3: warmup 715, cosine to 10 %
 * of 6e-4). Pure function. */
double gpt2_lr(long step, double max_lr, double min_lr, long warmup, long max_steps);

/* Host copies of the fp32 flat parameter / gradient buffers
 * (gpt2_num_params floats); synchronous. */
gpt2_status gpt2_get_params(const gpt2_t* h, float* host);
gpt2_status gpt2_set_params(gpt2_t* h, const float* host); /* also refreshes the bf16 copy */
gpt2_status gpt2_get_grads(const gpt2_t* h, float* host);

/* Device pointer to the fp32 gradient buffer itself (gpt2_num_params floats,
 * the layout of gpt2_tensor_info), owned by the model.  For replicas that
 * exchange gradients: after every replica's gpt2_backward calls, a sum
 * all-reduce of this buffer (on the model's stream, or ordered after it)
 * and then gpt2_grad_norm_clip / gpt2_adamw_step on every replica keep the
 * replicas' parameters identical.  Valid until gpt2_destroy or
 * gpt2_bind_memory. */
gpt2_status gpt2_grads_device(gpt2_t* h, float** dev_ptr);

/* Data-parallel building blocks (condensed GPT-2 page, section 3: each GPU
 * runs its own micro-batches and the gradients are averaged before the
 * update; the llm.c page's ZeRO-1 option shards the optimizer state).
 *
 * gpt2_padded_params: length of the device buffers behind
 * gpt2_grads_device / gpt2_params_device, gpt2_num_params rounded up to a
 * multiple of 2048 with zeros, so that R ranks (R a power of two up to 2048)
 * can take equal contiguous shards of them.
 * gpt2_grad_sumsq: sum of the squared gradient elements [begin, end) (a
 * shard; begin a multiple of 4, end <= gpt2_padded_params), as a double at
 * sumsq_dev (device, 8-byte aligned), in a fixed-order two-stage reduction.
 * gpt2_clip_from_sumsq: the global norm n = sqrt(*sumsq_dev) (e.g. the sum of
 * every rank's shard sums) and the clip scale of gpt2_grad_norm_clip from it;
 * norm_host as there.
 * gpt2_adamw_step_range: gpt2_adamw_step on the parameters [begin, end) only
 * (begin and end - begin multiples of 4, unless end is the number of
 * parameters; also advances the step counter), refreshing the bf16 copy of
 * that range only.
 * gpt2_params_device: device pointer to the fp32 parameters (padded length),
 * e.g. for an all-gather of every rank's updated shard.
 * gpt2_refresh_weights: rewrite the bf16 weight copy the GEMMs read from the
 * fp32 parameters (after such an all-gather).
 * gpt2_set_backward_events: n = L + 1 cudaEvent_t handles (or n = 0 to stop)
 * that gpt2_backward records on its stream: event l once layer l's gradients
 * are final (every per-layer tensor slice of layer l), event L after the last
 * kernel (wte, wpe, lnf); a caller can start the gradient exchange of each
 * layer on another stream while the backward of the layers below runs. */
size_t gpt2_padded_params(const gpt2_t* h);
gpt2_status gpt2_grad_sumsq(gpt2_t* h, size_t begin, size_t end, double* sumsq_dev);
gpt2_status gpt2_clip_from_sumsq(gpt2_t* h, const double* sumsq_dev, float max_norm,
                                 float* norm_host);
gpt2_status gpt2_adamw_step_range(gpt2_t* h, float lr, float beta1, float beta2, float eps,
                                  float weight_decay, size_t begin, size_t end);
gpt2_status gpt2_params_device(gpt2_t* h, float** dev_ptr);
gpt2_status gpt2_refresh_weights(gpt2_t* h);
gpt2_status gpt2_set_backward_events(gpt2_t* h, void* const* events, int n);

/* Checkpoint state: params, m, v (each gpt2_num_params floats) and the step
 * counter t.  Any pointer may be NULL to skip that part. Synchronous. */
gpt2_status gpt2_get_state(const gpt2_t* h, float* params, float* m, float* v, long* t);
gpt2_status gpt2_set_state(gpt2_t* h, const float* params, const float* m, const float* v,
                           long t);

/* Tensor i (0..15) of the flat layout: name, 1 or 2 (or 3 for per-layer
 * matrices) dims, shape, offset in floats.  Order: wte[Vpad,C] wpe[Tmax,C]
 * ln1_g[L,C] ln1_b[L,C] w_qkv[L,3C,C] b_qkv[L,3C] w_o[L,C,C] b_o[L,C]
 * ln2_g[L,C] ln2_b[L,C] w_fc[L,4C,C] b_fc[L,4C] w_p[L,C,4C] b_p[L,C]
 * lnf_g[C] lnf_b[C]; matrices are (out, in) row-major, y = x W^T + b. */
gpt2_status gpt2_tensor_info(const gpt2_t* h, int i, const char** name, int* ndim,
                             int64_t shape[3], size_t* offset);

/* Device pointer to the logits of the last forward without targets,
 * [B*T, Vpad] row-major in the activation dtype (bf16 / fp32 build). */
gpt2_status gpt2_logits(const gpt2_t* h, const void** dev_ptr);

/* Per-position losses of the last forward with targets (B*T floats, host). */
gpt2_status gpt2_get_losses(const gpt2_t* h, float* host, size_t n);

/* Copy an activation of the last forward to the host as fp32 (for tests):
 * kind 0 residual input of layer `layer` (layer == L: the final residual),
 * 1 ln1 out, 2 qkv, 3 attention out, 4 residual after attention, 5 ln2 out,
 * 6 fc pre-activation, 7 GELU out, 8 lnf out.  n = number of floats. */
gpt2_status gpt2_read_activation(const gpt2_t* h, int kind, int layer, float* host, size_t n);

/* Text of the last error on this handle ("" if none). */
const char* gpt2_last_error(const gpt2_t* h);

/* Number of kernel launches this library has made in the process so far
 * (all handles); differences across a region count its launches. */
long gpt2_launch_count(void);

/* Per-kernel-family timing with CUDA events on the handle's stream.  Kinds:
 * 0 GEMM, 1 attention forward, 2 attention backward, 3 LayerNorm forward,
 * 4 LayerNorm backward, 5 classifier, 6 encoder (fwd+bwd), 7 bias-gradient
 * column sums, 8 optimiser (norm, clip, AdamW), 9 GELU recompute.
 * gpt2_profile_read synchronises the stream, writes for each kind the summed
 * milliseconds, the number of timed regions and the algorithmic FLOPs (GEMM:
 * 2MNK; attention: causal products), and clears the records.  `kinds` is the
 * length of the arrays (>= 10). */
gpt2_status gpt2_profile_enable(gpt2_t* h, int on);
gpt2_status gpt2_profile_read(gpt2_t* h, double* ms, long* launches, double* flops, int kinds);

#ifdef __cplusplus
}
#endif

#endif /* GPT2_B200_H */
