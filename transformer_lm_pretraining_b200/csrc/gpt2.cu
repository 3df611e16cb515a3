// GPT-2 step engine behind the C ABI of include/gpt2.h: parameter/optimiser
// state layout, activation workspace layout, and the sequence of kernel
// launches for forward, backward, clip and AdamW.

#include <cmath>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/gpt2.h"
#include "kernels.h"

using namespace gpt2k;

namespace {

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// Carves consecutive 256-byte aligned regions out of one allocation.
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t n) {
    T* p = reinterpret_cast<T*>(base ? base + used : nullptr);
    used += align256(n * sizeof(T));
    return p;
  }
};

struct Acts {
  act_t *res, *h1, *qkv, *att, *xmid, *h2, *u, *g, *hf, *logits;
  float *mean1, *rstd1, *lse, *mean2, *rstd2, *meanf, *rstdf, *losses;
  int* tok;
  act_t *dres, *dh, *datt, *dqkv, *dbig;
  float *dsum, *partials, *splitk;
  // partials of the backward's parameter-gradient column reductions, one
  // slice per reduction, so that their second stages run together at the
  // end of the backward (deferred_floats: the arena's size)
  float* deferred;
  size_t deferred_floats;
  void* enc_scratch;
  size_t splitk_floats;
};

// Floats of the deferred-reduction arena: per layer two layernorm backwards
// (kLnBlocks x 3C partials each), the W_fc bias (per-32-row slabs of 4C) and
// the W_qkv bias (kColsumChunks x 3C), plus the final layernorm.
size_t deferred_floats(size_t M, size_t C, size_t L) {
  const size_t ln = (size_t)kLnBlocks * 3 * C;
  const size_t fc = std::max((M + 31) / 32, (size_t)kColsumChunks) * 4 * C;
  return (2 * L + 1) * ln + L * (fc + (size_t)kColsumChunks * 3 * C);
}

constexpr int kMaxSplits = 8;

// Optional per-kernel-family timing with CUDA events on the handle's stream.
enum ProfKind {
  PK_GEMM, PK_ATTN_FWD, PK_ATTN_BWD, PK_LAYERNORM, PK_LN_BWD, PK_CLASSIFIER, PK_ENCODER,
  PK_COLSUM, PK_OPTIMIZER, PK_RECOMPUTE, PK_COUNT
};

struct ProfRec {
  int kind;
  cudaEvent_t a, b;
  double flops;
};

}  // namespace

struct gpt2 {
  Layout lay;
  uint64_t seed = 0;
  cudaStream_t stream = nullptr;
  // state
  void* state = nullptr;
  size_t state_bytes = 0;
  bool own_state = false;
  float *params = nullptr, *grads = nullptr, *m = nullptr, *v = nullptr;
  act_t* pact = nullptr;
  float* scalars = nullptr;
  double* norm_partials = nullptr;
  int* err = nullptr;
  int* dstep = nullptr;  // the optimizer step counter t, on the device
  // workspace
  void* work = nullptr;
  size_t work_bytes = 0;
  bool own_work = false;
  int recompute = 0;  // 1: GELU outputs are not kept; the backward recomputes them
  // generation: key/value cache and one-position scratch (library-owned)
  void* gen = nullptr;
  size_t gen_bytes = 0;
  // forward record
  int B = 0, T = 0;
  bool have_grad_logits = false;
  bool have_logits = false;
  // every gradient is zero (gpt2_zero_grad since the last backward), so the
  // first backward's two-way split weight gradients may add in place
  bool grads_zero = false;
  Acts a{};
  std::string last_error;
  // events recorded after each layer's backward (and the last one after the
  // embedding's), for callers overlapping gradient communication
  std::vector<cudaEvent_t> bwd_events;
  // a captured optimizer step (gpt2_step_graph_capture)
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t graph_exec = nullptr;
  long graph_launches = 0;
  // profiling
  bool prof = false;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<ProfRec> recs;
};

namespace {

gpt2_status fail(gpt2_t* h, gpt2_status code, const std::string& msg) {
  if (h) h->last_error = msg;
  return code;
}

gpt2_status cuda_fail(gpt2_t* h, cudaError_t e, const char* where) {
  return fail(h, GPT2_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

#define GPT2_CUDA(h, call)                                   \
  do {                                                       \
    cudaError_t e_ = (call);                                 \
    if (e_ != cudaSuccess) return cuda_fail(h, e_, #call);   \
  } while (0)

// Parameters per buffer, padded with zeros to a multiple of 2048 so that
// data-parallel ranks (up to 2048 of them, in powers of two) can take equal
// shards of the flat buffers.
size_t padded_params(const Layout& lay) { return (lay.total + 2047) / 2048 * 2048; }

// Layout of the state allocation.
size_t carve_state(const Layout& lay, void* base, gpt2_t* h) {
  Carver c(base);
  const size_t Pp = padded_params(lay);
  float* params = c.take<float>(Pp);
  float* grads = c.take<float>(Pp);
  float* m = c.take<float>(Pp);
  float* v = c.take<float>(Pp);
#if GPT2_ACT_BF16
  act_t* pact = c.take<act_t>(Pp);
#else
  act_t* pact = params;
#endif
  float* scalars = c.take<float>(S_COUNT);
  double* np = c.take<double>(kNormBlocks);
  int* err = c.take<int>(16);
  if (h) {
    h->params = params; h->grads = grads; h->m = m; h->v = v; h->pact = pact;
    h->scalars = scalars; h->norm_partials = np; h->err = err;
    h->dstep = err + 8;
  }
  return c.used;
}

// Layout of the workspace for B x T tokens.
size_t carve_work(const Layout& lay, int B, int T, int recompute, void* base, Acts* a) {
  const size_t M = (size_t)B * T, C = lay.C, L = lay.L, H = lay.H;
  Carver c(base);
  Acts x{};
  x.res = c.take<act_t>((L + 1) * M * C);
  x.h1 = c.take<act_t>(L * M * C);
  x.qkv = c.take<act_t>(L * M * 3 * C);
  x.att = c.take<act_t>(L * M * C);
  x.xmid = c.take<act_t>(L * M * C);
  x.h2 = c.take<act_t>(L * M * C);
  x.u = c.take<act_t>(L * M * 4 * C);
  x.g = c.take<act_t>((recompute ? 1 : L) * M * 4 * C);  // one layer's worth when recomputed
  x.hf = c.take<act_t>(M * C);
  x.logits = c.take<act_t>(M * (size_t)lay.Vp);
  x.mean1 = c.take<float>(L * M);
  x.rstd1 = c.take<float>(L * M);
  x.lse = c.take<float>(L * M * H);
  x.mean2 = c.take<float>(L * M);
  x.rstd2 = c.take<float>(L * M);
  x.meanf = c.take<float>(M);
  x.rstdf = c.take<float>(M);
  x.losses = c.take<float>(M);
  x.tok = c.take<int>(M);
  x.dres = c.take<act_t>(M * C);
  x.dh = c.take<act_t>(M * C);
  x.datt = c.take<act_t>(M * C);
  x.dqkv = c.take<act_t>(M * 3 * C);
  x.dbig = c.take<act_t>(M * 4 * C);
  x.dsum = c.take<float>(attention_bwd_scratch_floats(B, T, (int)H));
  const size_t part = std::max((size_t)kColsumChunks * 4 * C, (size_t)kLnBlocks * 3 * C);
  x.partials = c.take<float>(part);
  x.deferred_floats = deferred_floats(M, C, L);
  x.deferred = c.take<float>(x.deferred_floats);
  x.splitk_floats = (size_t)kMaxSplits * 4 * C * C;
  x.splitk = c.take<float>(x.splitk_floats);
  x.enc_scratch = c.take<char>(encoder_scratch_bytes((int)M, (int)C));
  if (a) *a = x;
  return c.used;
}

gpt2_status check_err_word(gpt2_t* h) {
  int e = 0;
  GPT2_CUDA(h, cudaMemcpyAsync(&e, h->err, sizeof(int), cudaMemcpyDeviceToHost, h->stream));
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  if (e) {
    GPT2_CUDA(h, cudaMemsetAsync(h->err, 0, sizeof(int), h->stream));
    if (e & ERR_TIMEOUT) return fail(h, GPT2_ERR_TIMEOUT, "a kernel's bounded wait expired");
    if (e & ERR_TOKEN) return fail(h, GPT2_ERR_TOKEN, "token id outside [0, V)");
    if (e & ERR_TARGET) return fail(h, GPT2_ERR_TOKEN, "target id outside [0, V)");
  }
  return GPT2_OK;
}

gpt2_status ensure_state(gpt2_t* h) {
  if (h->state) return GPT2_OK;
  const size_t bytes = carve_state(h->lay, nullptr, nullptr);
  void* p = nullptr;
  GPT2_CUDA(h, cudaMalloc(&p, bytes));
  gpt2_status st = gpt2_bind_memory(h, p, bytes, nullptr, 0);
  if (st != GPT2_OK) {
    cudaFree(p);
    return st;
  }
  h->own_state = true;
  return GPT2_OK;
}

gpt2_status ensure_work(gpt2_t* h, int B, int T) {
  const size_t need = carve_work(h->lay, B, T, h->recompute, nullptr, nullptr);
  if (h->work && h->work_bytes >= need) return GPT2_OK;
  if (h->work && !h->own_work)
    return fail(h, GPT2_ERR_ARG, "bound workspace is smaller than gpt2_workspace_bytes(B, T)");
  if (h->own_work) {
    cudaFree(h->work);
    h->work = nullptr;
  }
  void* p = nullptr;
  GPT2_CUDA(h, cudaMalloc(&p, need));
  h->work = p;
  h->work_bytes = need;
  h->own_work = true;
  return GPT2_OK;
}

#define GPT2_TRY(expr)            \
  do {                            \
    gpt2_status st_ = (expr);     \
    if (st_ != GPT2_OK) return st_; \
  } while (0)

cudaEvent_t prof_event(gpt2_t* h) {
  if (!h->ev_pool.empty()) {
    cudaEvent_t e = h->ev_pool.back();
    h->ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Timeline marks: with profiling on, each mark records an event on the
// stream; the time up to the next mark is charged to the mark's kernel
// family (only that family's launches sit between two marks).
void mark(gpt2_t* h, int kind, double flops = 0) {
  if (!h->prof) return;
  cudaEvent_t e = prof_event(h);
  cudaEventRecord(e, h->stream);
  if (!h->recs.empty() && h->recs.back().b == nullptr) h->recs.back().b = e;
  h->recs.push_back({kind, e, nullptr, flops});
}
void mark_end(gpt2_t* h) {
  if (!h->prof || h->recs.empty() || h->recs.back().b != nullptr) return;
  cudaEvent_t e = prof_event(h);
  cudaEventRecord(e, h->stream);
  h->recs.back().b = e;
}

gpt2_status run_gemm(gpt2_t* h, const GemmArgs& ga) {
  mark(h, PK_GEMM, 2.0 * (ga.M + ga.M2) * ga.N * ga.K);
  GPT2_CUDA(h, gemm(ga, h->stream, h->err));
  return GPT2_OK;
}

GemmArgs gemm_args(int M, int N, int K) {
  GemmArgs g{};
  g.M = M; g.N = N; g.K = K;
  g.alpha = 1.f;
  g.max_splits = 1;
  return g;
}

}  // namespace

extern "C" {

int gpt2_build_is_bf16(void) { return GPT2_ACT_BF16; }

gpt2_status gpt2_create(int L, int H, int C, int V, int Vpad, int Tmax, uint64_t seed,
                        gpt2_t** out) {
  if (!out) return GPT2_ERR_ARG;
  *out = nullptr;
  if (L < 1 || H < 1 || C < 8 || V < 1 || Tmax < 1 || C % H || C % 8 || Vpad < V || Vpad % 64 ||
      C > 2048)
    return GPT2_ERR_ARG;
  const int hd = C / H;
#if GPT2_ACT_BF16
  if (hd != 32 && hd != 64 && hd != 128) return GPT2_ERR_ARG;
#else
  if (hd > 128 || hd % 8) return GPT2_ERR_ARG;
#endif
  gpt2_t* h = new gpt2_t();
  h->lay = make_layout(L, H, C, V, Vpad, Tmax);
  h->seed = seed;
  *out = h;
  return GPT2_OK;
}

void gpt2_destroy(gpt2_t* h) {
  if (!h) return;
  if (h->own_state && h->state) cudaFree(h->state);
  if (h->own_work && h->work) cudaFree(h->work);
  if (h->gen) cudaFree(h->gen);
  if (h->graph_exec) cudaGraphExecDestroy(h->graph_exec);
  if (h->graph) cudaGraphDestroy(h->graph);
  std::vector<cudaEvent_t> evs = h->ev_pool;
  for (const ProfRec& r : h->recs) {
    evs.push_back(r.a);
    if (r.b) evs.push_back(r.b);
  }
  std::sort(evs.begin(), evs.end());
  evs.erase(std::unique(evs.begin(), evs.end()), evs.end());
  for (cudaEvent_t e : evs) cudaEventDestroy(e);
  delete h;
}

size_t gpt2_num_params(const gpt2_t* h) { return h ? h->lay.total : 0; }

size_t gpt2_state_bytes(const gpt2_t* h) { return h ? carve_state(h->lay, nullptr, nullptr) : 0; }

size_t gpt2_workspace_bytes(const gpt2_t* h, int B, int T) {
  if (!h || B < 1 || T < 1) return 0;
  return carve_work(h->lay, B, T, h->recompute, nullptr, nullptr);
}

gpt2_status gpt2_bind_memory(gpt2_t* h, void* dev_state, size_t state_bytes, void* dev_work,
                             size_t work_bytes) {
  if (!h) return GPT2_ERR_ARG;
  if (dev_state) {
    if (reinterpret_cast<uintptr_t>(dev_state) & 255)
      return fail(h, GPT2_ERR_ARG, "state memory must be 256-byte aligned");
    if (state_bytes < gpt2_state_bytes(h)) return fail(h, GPT2_ERR_ARG, "state memory too small");
    if (h->own_state && h->state) cudaFree(h->state);
    h->own_state = false;
    h->state = dev_state;
    h->state_bytes = state_bytes;
    const size_t used = carve_state(h->lay, dev_state, h);
    const size_t P = h->lay.total;
    // everything zero (gradients, moments, the zero padding of every buffer,
    // scalars, error word, step counter), then the seeded parameters
    GPT2_CUDA(h, cudaMemsetAsync(dev_state, 0, used, h->stream));
    init_params(h->params, h->lay, h->seed, h->stream);
    GPT2_CUDA(h, cudaGetLastError());
    reset_clip(h->scalars, h->stream);
#if GPT2_ACT_BF16
    f32_to_act(h->pact, h->params, P, h->stream);
    GPT2_CUDA(h, cudaGetLastError());
#endif
    h->have_grad_logits = h->have_logits = false;
  }
  if (dev_work) {
    if (reinterpret_cast<uintptr_t>(dev_work) & 255)
      return fail(h, GPT2_ERR_ARG, "workspace must be 256-byte aligned");
    if (h->own_work && h->work) cudaFree(h->work);
    h->own_work = false;
    h->work = dev_work;
    h->work_bytes = work_bytes;
    h->have_grad_logits = h->have_logits = false;
  }
  return GPT2_OK;
}

gpt2_status gpt2_set_recompute(gpt2_t* h, int level) {
  if (!h || level < 0 || level > 1) return fail(h, GPT2_ERR_ARG, "recompute level is 0 or 1");
  if (level != h->recompute) {
    h->recompute = level;
    h->have_grad_logits = h->have_logits = false;  // the workspace layout changed
  }
  return GPT2_OK;
}

gpt2_status gpt2_set_stream(gpt2_t* h, void* cuda_stream) {
  if (!h) return GPT2_ERR_ARG;
  h->stream = static_cast<cudaStream_t>(cuda_stream);
  return GPT2_OK;
}

namespace {

// The forward pass; `train` leaves dL/dlogits in the logits buffer for the
// backward, otherwise (evaluation) the logits are kept as computed.
gpt2_status forward_impl(gpt2_t* h, const int32_t* tok, const int32_t* tgt, int B, int T,
                         float* loss_host, bool train) {
  if (!h || !tok || B < 1 || T < 1) return fail(h, GPT2_ERR_ARG, "bad forward arguments");
  const Layout& y = h->lay;
  if (T > y.Tmax) return fail(h, GPT2_ERR_ARG, "T > Tmax");
  gpt2_status st = ensure_state(h);
  if (st) return st;
  st = ensure_work(h, B, T);
  if (st) return st;
  Acts& a = h->a;
  carve_work(y, B, T, h->recompute, h->work, &a);
  h->B = B;
  h->T = T;
  const int M = B * T, C = y.C, L = y.L, H = y.H;
  const size_t MC = (size_t)M * C;
  cudaStream_t s = h->stream;
  const float* P = h->params;
  const act_t* W = h->pact;

  mark(h, PK_ENCODER);
  encoder_fwd(a.res, a.tok, tok, W + y.off[T_WTE], W + y.off[T_WPE], B, T, C, y.V, h->err, s);
  for (int l = 0; l < L; ++l) {
    act_t* x = a.res + (size_t)l * MC;
    act_t* h1 = a.h1 + (size_t)l * MC;
    act_t* qkv = a.qkv + (size_t)l * 3 * MC;
    act_t* att = a.att + (size_t)l * MC;
    act_t* xm = a.xmid + (size_t)l * MC;
    act_t* h2 = a.h2 + (size_t)l * MC;
    act_t* u = a.u + (size_t)l * 4 * MC;
    act_t* g = a.g + (h->recompute ? 0 : (size_t)l * 4 * MC);
    mark(h, PK_LAYERNORM);
    layernorm_fwd(h1, a.mean1 + (size_t)l * M, a.rstd1 + (size_t)l * M, x,
                  P + y.off[T_LN1G] + (size_t)l * C, P + y.off[T_LN1B] + (size_t)l * C, M, C, s);
    {  // qkv = h1 W_qkv^T + b_qkv
      GemmArgs ga = gemm_args(M, 3 * C, C);
      ga.A = h1; ga.lda = C;
      ga.B = W + y.off[T_WQKV] + (size_t)l * 3 * C * C; ga.ldb = C;
      ga.epi = EPI_BIAS; ga.bias = P + y.off[T_BQKV] + (size_t)l * 3 * C;
      ga.out = qkv; ga.ldo = 3 * C;
      GPT2_TRY(run_gemm(h, ga));
    }
    mark(h, PK_ATTN_FWD, 4.0 * B * H * (double)T * (T + 1) / 2 * (C / H));
    GPT2_CUDA(h, attention_fwd(att, a.lse + (size_t)l * M * H, qkv, B, T, C, H, h->err, s));
    {  // xmid = x + att W_o^T + b_o
      GemmArgs ga = gemm_args(M, C, C);
      ga.A = att; ga.lda = C;
      ga.B = W + y.off[T_WO] + (size_t)l * C * C; ga.ldb = C;
      ga.epi = EPI_BIAS_RESID; ga.bias = P + y.off[T_BO] + (size_t)l * C;
      ga.resid = x; ga.ldr = C;
      ga.out = xm; ga.ldo = C;
      GPT2_TRY(run_gemm(h, ga));
    }
    mark(h, PK_LAYERNORM);
    layernorm_fwd(h2, a.mean2 + (size_t)l * M, a.rstd2 + (size_t)l * M, xm,
                  P + y.off[T_LN2G] + (size_t)l * C, P + y.off[T_LN2B] + (size_t)l * C, M, C, s);
    {  // u = h2 W_fc^T + b_fc; g = gelu(u)
      GemmArgs ga = gemm_args(M, 4 * C, C);
      ga.A = h2; ga.lda = C;
      ga.B = W + y.off[T_WFC] + (size_t)l * 4 * C * C; ga.ldb = C;
      ga.epi = EPI_BIAS_GELU; ga.bias = P + y.off[T_BFC] + (size_t)l * 4 * C;
      ga.aux = u; ga.ldaux = 4 * C;
      ga.out = g; ga.ldo = 4 * C;
      GPT2_TRY(run_gemm(h, ga));
    }
    {  // x_next = xmid + g W_p^T + b_p
      GemmArgs ga = gemm_args(M, C, 4 * C);
      ga.A = g; ga.lda = 4 * C;
      ga.B = W + y.off[T_WP] + (size_t)l * 4 * C * C; ga.ldb = 4 * C;
      ga.epi = EPI_BIAS_RESID; ga.bias = P + y.off[T_BP] + (size_t)l * C;
      ga.resid = xm; ga.ldr = C;
      ga.out = a.res + (size_t)(l + 1) * MC; ga.ldo = C;
      GPT2_TRY(run_gemm(h, ga));
    }
  }
  mark(h, PK_LAYERNORM);
  layernorm_fwd(a.hf, a.meanf, a.rstdf, a.res + (size_t)L * MC, P + y.off[T_LNFG],
                P + y.off[T_LNFB], M, C, s);
  {  // logits = hf wte^T over all Vpad rows (padded rows are 0)
    GemmArgs ga = gemm_args(M, y.Vp, C);
    ga.A = a.hf; ga.lda = C;
    ga.B = W + y.off[T_WTE]; ga.ldb = C;
    ga.epi = EPI_STORE;
    ga.out = a.logits; ga.ldo = y.Vp;
    GPT2_TRY(run_gemm(h, ga));
  }
  h->have_grad_logits = false;
  h->have_logits = false;
  if (tgt) {
    mark(h, PK_CLASSIFIER);
    classifier(a.logits, a.losses, tgt, M, y.V, y.Vp, train ? 1 : 0, h->err, s);
    mean_loss(h->scalars + S_LOSS, a.losses, M, s);
    h->have_grad_logits = train;
    h->have_logits = !train;
  } else {
    h->have_logits = true;
  }
  mark_end(h);
  GPT2_CUDA(h, cudaGetLastError());
  if (loss_host) {
    GPT2_CUDA(h, cudaMemcpyAsync(loss_host, h->scalars + S_LOSS, sizeof(float),
                                 cudaMemcpyDeviceToHost, s));
    st = check_err_word(h);
    if (st) return st;
    if (tgt && !std::isfinite(*loss_host)) return fail(h, GPT2_ERR_NONFINITE, "loss is not finite");
  }
  return GPT2_OK;
}

}  // namespace

gpt2_status gpt2_forward(gpt2_t* h, const int32_t* tok, const int32_t* tgt, int B, int T,
                         float* loss_host) {
  return forward_impl(h, tok, tgt, B, T, loss_host, true);
}

gpt2_status gpt2_evaluate(gpt2_t* h, const int32_t* tok, const int32_t* tgt, int B, int T,
                          float* loss_host) {
  if (!tgt) return fail(h, GPT2_ERR_ARG, "evaluation needs targets");
  return forward_impl(h, tok, tgt, B, T, loss_host, false);
}

namespace {

// Generation buffers: the key/value cache [L][B][Ttot][2C] and the
// one-position activations of a decode step.
constexpr int kGenSplits = 16;  // K splits of a one-position product at most
struct GenBufs {
  act_t *cache, *x0, *x1, *hb, *q, *kvnew, *att, *xm, *u, *g, *logits;
  float *mean, *rstd;
  float* splitws;  // split-K partials of the one-position products
  int* prompt;
  int* pos;  // the decode position (device counter)
};

size_t carve_gen(const Layout& y, int B, int Tp, int Ttot, void* base, GenBufs* out) {
  const size_t C = y.C;
  Carver c(base);
  GenBufs g{};
  g.cache = c.take<act_t>((size_t)y.L * B * Ttot * 2 * C);
  g.x0 = c.take<act_t>(B * C);
  g.x1 = c.take<act_t>(B * C);
  g.hb = c.take<act_t>(B * C);
  g.q = c.take<act_t>(B * C);
  g.kvnew = c.take<act_t>(B * 2 * C);
  g.att = c.take<act_t>(B * C);
  g.xm = c.take<act_t>(B * C);
  g.u = c.take<act_t>(B * 4 * C);
  g.g = c.take<act_t>(B * 4 * C);
  g.logits = c.take<act_t>((size_t)B * y.Vp);
  g.mean = c.take<float>(B);
  g.rstd = c.take<float>(B);
  g.splitws = c.take<float>((size_t)kGenSplits * B * 4 * C);
  g.prompt = c.take<int>((size_t)B * Tp);
  g.pos = c.take<int>(1);
  if (out) *out = g;
  return c.used;
}

}  // namespace

gpt2_status gpt2_generate(gpt2_t* h, int32_t* tok, int B, int Tp, int Ttot, float temperature,
                          int top_k, uint64_t seed, float* step_logits) {
  if (!h || !tok || B < 1 || Tp < 1 || Ttot <= Tp) return fail(h, GPT2_ERR_ARG, "bad generate arguments");
  const Layout& y = h->lay;
  if (Ttot > y.Tmax) return fail(h, GPT2_ERR_ARG, "T_total > Tmax");
  if (y.C / y.H > 128) return fail(h, GPT2_ERR_ARG, "generation supports head dims up to 128");
  gpt2_status st = ensure_state(h);
  if (st) return st;
  const size_t need = carve_gen(y, B, Tp, Ttot, nullptr, nullptr);
  if (h->gen_bytes < need) {
    if (h->gen) cudaFree(h->gen);
    h->gen = nullptr;
    h->gen_bytes = 0;
    GPT2_CUDA(h, cudaMalloc(&h->gen, need));
    h->gen_bytes = need;
  }
  GenBufs gb;
  carve_gen(y, B, Tp, Ttot, h->gen, &gb);
  cudaStream_t s = h->stream;
  const int C = y.C, L = y.L, H = y.H;
  const float* P = h->params;
  const act_t* W = h->pact;
  // prefill: the training forward over the prompt (contiguous copy), then
  // its keys and values into the cache
  GPT2_CUDA(h, cudaMemcpy2DAsync(gb.prompt, (size_t)Tp * sizeof(int), tok, (size_t)Ttot * sizeof(int),
                                 (size_t)Tp * sizeof(int), B, cudaMemcpyDeviceToDevice, s));
  st = forward_impl(h, gb.prompt, nullptr, B, Tp, nullptr, true);
  if (st) return st;
  const Acts& a = h->a;
  const size_t MCp = (size_t)B * Tp * C;
  for (int l = 0; l < L; ++l)
    for (int b = 0; b < B; ++b)
      GPT2_CUDA(h, cudaMemcpy2DAsync(gb.cache + ((size_t)l * B + b) * Ttot * 2 * C, 2 * C * sizeof(act_t),
                                     a.qkv + (size_t)l * 3 * MCp + (size_t)b * Tp * 3 * C + C,
                                     3 * C * sizeof(act_t), 2 * C * sizeof(act_t), Tp,
                                     cudaMemcpyDeviceToDevice, s));
  sample_tokens(tok, Ttot, Tp, nullptr, a.logits + (size_t)(Tp - 1) * y.Vp, (long)Tp * y.Vp, B, y.V,
                temperature, top_k, seed, step_logits, Tp, s);
  // decode: the step at position p takes token p and yields token p + 1.
  // It works at the device position counter gb.pos, so that the same launch
  // sequence serves every position: the first step runs as plain launches
  // (first use of its kernels), the rest replay it captured as a CUDA graph.
  const int p_first = Tp;
  GPT2_CUDA(h, cudaMemcpyAsync(gb.pos, &p_first, sizeof(int), cudaMemcpyHostToDevice, s));
  // the one-position products split K across the SMs (see gemm)
  auto split = [&](GemmArgs& ga) {
    ga.split_ws = gb.splitws;
    ga.split_ws_floats = (size_t)kGenSplits * B * 4 * C;
    ga.max_splits = kGenSplits;
  };
  auto step = [&]() -> gpt2_status {
    decode_embed(gb.x0, tok, Ttot, 0, gb.pos, W + y.off[T_WTE], W + y.off[T_WPE], B, C, y.V,
                 h->err, s);
    act_t* x = gb.x0;
    act_t* xn = gb.x1;
    for (int l = 0; l < L; ++l) {
      act_t* kv = gb.cache + (size_t)l * B * Ttot * 2 * C;
      layernorm_fwd(gb.hb, gb.mean, gb.rstd, x, P + y.off[T_LN1G] + (size_t)l * C,
                    P + y.off[T_LN1B] + (size_t)l * C, B, C, s);
      {  // q = h W_q^T + b_q
        GemmArgs ga = gemm_args(B, C, C);
        ga.A = gb.hb; ga.lda = C;
        ga.B = W + y.off[T_WQKV] + (size_t)l * 3 * C * C; ga.ldb = C;
        ga.epi = EPI_BIAS; ga.bias = P + y.off[T_BQKV] + (size_t)l * 3 * C;
        ga.out = gb.q; ga.ldo = C;
        split(ga);
        GPT2_TRY(run_gemm(h, ga));
      }
      {  // [k | v] of the position, then into the cache at it
        GemmArgs ga = gemm_args(B, 2 * C, C);
        ga.A = gb.hb; ga.lda = C;
        ga.B = W + y.off[T_WQKV] + (size_t)l * 3 * C * C + (size_t)C * C; ga.ldb = C;
        ga.epi = EPI_BIAS; ga.bias = P + y.off[T_BQKV] + (size_t)l * 3 * C + C;
        ga.out = gb.kvnew; ga.ldo = 2 * C;
        split(ga);
        GPT2_TRY(run_gemm(h, ga));
      }
      kv_append(kv, gb.kvnew, 0, gb.pos, Ttot, B, C, s);
      decode_attention(gb.att, gb.q, kv, Ttot, 1, gb.pos, B, C, H, s);  // n = position + 1
      {  // xm = x + att W_o^T + b_o
        GemmArgs ga = gemm_args(B, C, C);
        ga.A = gb.att; ga.lda = C;
        ga.B = W + y.off[T_WO] + (size_t)l * C * C; ga.ldb = C;
        ga.epi = EPI_BIAS_RESID; ga.bias = P + y.off[T_BO] + (size_t)l * C;
        ga.resid = x; ga.ldr = C;
        ga.out = gb.xm; ga.ldo = C;
        split(ga);
        GPT2_TRY(run_gemm(h, ga));
      }
      layernorm_fwd(gb.hb, gb.mean, gb.rstd, gb.xm, P + y.off[T_LN2G] + (size_t)l * C,
                    P + y.off[T_LN2B] + (size_t)l * C, B, C, s);
      {  // u = h W_fc^T + b_fc; g = gelu(u)
        GemmArgs ga = gemm_args(B, 4 * C, C);
        ga.A = gb.hb; ga.lda = C;
        ga.B = W + y.off[T_WFC] + (size_t)l * 4 * C * C; ga.ldb = C;
        ga.epi = EPI_BIAS_GELU; ga.bias = P + y.off[T_BFC] + (size_t)l * 4 * C;
        ga.aux = gb.u; ga.ldaux = 4 * C;
        ga.out = gb.g; ga.ldo = 4 * C;
        split(ga);
        GPT2_TRY(run_gemm(h, ga));
      }
      {  // x_next = xm + g W_p^T + b_p
        GemmArgs ga = gemm_args(B, C, 4 * C);
        ga.A = gb.g; ga.lda = 4 * C;
        ga.B = W + y.off[T_WP] + (size_t)l * 4 * C * C; ga.ldb = 4 * C;
        ga.epi = EPI_BIAS_RESID; ga.bias = P + y.off[T_BP] + (size_t)l * C;
        ga.resid = gb.xm; ga.ldr = C;
        ga.out = xn; ga.ldo = C;
        split(ga);
        GPT2_TRY(run_gemm(h, ga));
      }
      std::swap(x, xn);
    }
    layernorm_fwd(gb.hb, gb.mean, gb.rstd, x, P + y.off[T_LNFG], P + y.off[T_LNFB], B, C, s);
    {  // logits of the position
      GemmArgs ga = gemm_args(B, y.Vp, C);
      ga.A = gb.hb; ga.lda = C;
      ga.B = W + y.off[T_WTE]; ga.ldb = C;
      ga.epi = EPI_STORE;
      ga.out = gb.logits; ga.ldo = y.Vp;
      GPT2_TRY(run_gemm(h, ga));
    }
    sample_tokens(tok, Ttot, 1, gb.pos, gb.logits, y.Vp, B, y.V, temperature, top_k, seed,
                  step_logits, Tp, s);  // token position + 1
    pos_advance(gb.pos, s);
    return GPT2_OK;
  };
  const int nsteps = Ttot - 1 - Tp;
  if (nsteps > 0) {
    st = step();
    if (st) return st;
  }
  if (nsteps > 1) {
    if (h->stream && !h->prof) {  // capture needs a stream of its own; profiling marks stay eager
      GPT2_CUDA(h, cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal));
      st = step();
      cudaGraph_t g = nullptr;
      const cudaError_t ec = cudaStreamEndCapture(s, &g);
      if (st) {
        if (g) cudaGraphDestroy(g);
        return st;
      }
      if (ec != cudaSuccess) return cuda_fail(h, ec, "cudaStreamEndCapture (decode step)");
      cudaGraphExec_t ex = nullptr;
      const cudaError_t ei = cudaGraphInstantiate(&ex, g, 0);
      cudaGraphDestroy(g);
      if (ei != cudaSuccess) return cuda_fail(h, ei, "cudaGraphInstantiate (decode step)");
      cudaError_t el = cudaSuccess;
      for (int i = 1; i < nsteps && el == cudaSuccess; ++i) el = cudaGraphLaunch(ex, s);
      cudaGraphExecDestroy(ex);  // freed once its launches complete
      if (el != cudaSuccess) return cuda_fail(h, el, "cudaGraphLaunch (decode step)");
    } else {
      for (int i = 1; i < nsteps; ++i) {
        st = step();
        if (st) return st;
      }
    }
  }
  h->have_logits = h->have_grad_logits = false;  // the forward record now holds the prompt only
  GPT2_CUDA(h, cudaGetLastError());
  return GPT2_OK;
}

gpt2_status gpt2_read_loss(gpt2_t* h, float* loss_host) {
  if (!h || !loss_host || !h->scalars) return GPT2_ERR_ARG;
  GPT2_CUDA(h, cudaMemcpyAsync(loss_host, h->scalars + S_LOSS, sizeof(float),
                               cudaMemcpyDeviceToHost, h->stream));
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  return GPT2_OK;
}

gpt2_status gpt2_zero_grad(gpt2_t* h) {
  if (!h) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  GPT2_CUDA(h, cudaMemsetAsync(h->grads, 0, h->lay.total * sizeof(float), h->stream));
  h->grads_zero = true;
  return GPT2_OK;
}

gpt2_status gpt2_backward(gpt2_t* h, float loss_scale) {
  if (!h) return GPT2_ERR_ARG;
  if (!h->have_grad_logits)
    return fail(h, GPT2_ERR_STATE, "backward needs a preceding forward with targets");
  const int acc_zero = h->grads_zero ? 1 : 0;
  h->grads_zero = false;
  const Layout& y = h->lay;
  Acts& a = h->a;
  const int B = h->B, T = h->T, M = B * T, C = y.C, L = y.L, H = y.H;
  const size_t MC = (size_t)M * C;
  cudaStream_t s = h->stream;
  const float* P = h->params;
  const act_t* W = h->pact;
  float* G = h->grads;
  EncoderScratch es;
  encoder_scratch_carve(&es, a.enc_scratch, M, C);
  // Without per-layer gradient events (no overlapped data-parallel
  // reduction), the second stages of the parameter-gradient column
  // reductions (layernorm gamma and beta, the biases) wait until the end of
  // the backward and run in one grouped launch, off the path from layer to
  // layer; each reduction keeps its partials in a slice of its own.
  const bool defer = h->bwd_events.empty() && a.deferred != nullptr;
  ReduceJobs jobs;
  jobs.n = 0;
  ReduceJob job;
  size_t dused = 0;
  auto slice = [&](size_t n, float* immediate) {
    if (!defer) return immediate;
    float* p = a.deferred + dused;
    dused += n;
    return p;
  };
  auto queue = [&]() {
    if (!defer) return;
    if (!reduce_jobs_add(jobs, job)) {  // the list is full: run it first
      reduce_jobs_run(jobs, s);
      reduce_jobs_add(jobs, job);
    }
  };
  const size_t ln_part = (size_t)kLnBlocks * 3 * C;
  ReduceJob* dj = defer ? &job : nullptr;

  {  // dhf = scale * dz wte  (dz: the logits buffer)
    GemmArgs ga = gemm_args(M, C, y.Vp);
    ga.A = a.logits; ga.lda = y.Vp;
    ga.B = W + y.off[T_WTE]; ga.ldb = C; ga.b_mn = 1;
    ga.epi = EPI_STORE; ga.alpha = loss_scale;
    ga.out = a.dh; ga.ldo = C;
    GPT2_TRY(run_gemm(h, ga));
  }
  {  // dwte += scale * dz^T hf
    GemmArgs ga = gemm_args(y.Vp, C, M);
    ga.A = a.logits; ga.lda = y.Vp; ga.a_mn = 1;
    ga.B = a.hf; ga.ldb = C; ga.b_mn = 1;
    ga.epi = EPI_F32_ACC; ga.alpha = loss_scale;
    ga.out32 = G + y.off[T_WTE]; ga.ldo32 = C;
    ga.split_ws = a.splitk; ga.split_ws_floats = a.splitk_floats; ga.max_splits = kMaxSplits;
    ga.acc_zero = acc_zero;
    GPT2_TRY(run_gemm(h, ga));
  }
  mark(h, PK_LN_BWD);
  // dres = d x_L; its column sum is the bias gradient of the last W_p
  layernorm_bwd(a.dres, a.dh, a.res + (size_t)L * MC, a.meanf, a.rstdf, P + y.off[T_LNFG],
                G + y.off[T_LNFG], G + y.off[T_LNFB], G + y.off[T_BP] + (size_t)(L - 1) * C,
                slice(ln_part, a.partials), M, C, 0, s, dj);
  queue();

  for (int l = L - 1; l >= 0; --l) {
    const act_t* x = a.res + (size_t)l * MC;
    const act_t* h1 = a.h1 + (size_t)l * MC;
    const act_t* qkv = a.qkv + (size_t)l * 3 * MC;
    const act_t* att = a.att + (size_t)l * MC;
    const act_t* xm = a.xmid + (size_t)l * MC;
    const act_t* h2 = a.h2 + (size_t)l * MC;
    const act_t* u = a.u + (size_t)l * 4 * MC;
    const act_t* g = a.g + (h->recompute ? 0 : (size_t)l * 4 * MC);
    // ---- MLP: x_next = xm + gelu(h2 Wfc^T + bfc) Wp^T + bp
    {  // du = (dres Wp) * gelu'(u)
      GemmArgs ga = gemm_args(M, 4 * C, C);
      ga.A = a.dres; ga.lda = C;
      ga.B = W + y.off[T_WP] + (size_t)l * 4 * C * C; ga.ldb = 4 * C; ga.b_mn = 1;
      ga.epi = EPI_DGELU; ga.aux = const_cast<act_t*>(u); ga.ldaux = 4 * C;
      ga.out = a.dbig; ga.ldo = 4 * C;
      // the bias gradient of W_fc: per-32-row column sums of du from the
      // epilogue (into the split-K workspace, free until dWp below), or a
      // pass over du while it is still in L2
      const int slabs = (M + 31) / 32;
      const bool fused =
          gemm_colsum_supported() && (defer || (size_t)slabs * 4 * C <= a.splitk_floats);
      float* part = slice(std::max((size_t)slabs, (size_t)kColsumChunks) * 4 * C,
                          fused ? a.splitk : a.partials);
      if (fused) ga.colsum = part;
      GPT2_TRY(run_gemm(h, ga));
      mark(h, PK_COLSUM);
      if (fused) colsum_reduce(G + y.off[T_BFC] + (size_t)l * 4 * C, part, slabs, 4 * C, s, dj);
      else colsum_acc(G + y.off[T_BFC] + (size_t)l * 4 * C, a.dbig, M, 4 * C, part, s, dj);
      queue();
    }
    if (h->recompute) {  // g = gelu(u), as the forward's epilogue computed it
      mark(h, PK_RECOMPUTE);
      gelu_fwd(const_cast<act_t*>(g), u, 4 * MC, s);
    }
    {  // dWp += dres^T g
      GemmArgs ga = gemm_args(C, 4 * C, M);
      ga.A = a.dres; ga.lda = C; ga.a_mn = 1;
      ga.B = g; ga.ldb = 4 * C; ga.b_mn = 1;
      ga.epi = EPI_F32_ACC;
      ga.out32 = G + y.off[T_WP] + (size_t)l * 4 * C * C; ga.ldo32 = 4 * C;
      ga.split_ws = a.splitk; ga.split_ws_floats = a.splitk_floats; ga.max_splits = kMaxSplits;
      ga.acc_zero = acc_zero;
      GPT2_TRY(run_gemm(h, ga));
    }
    {  // dh = du Wfc
      GemmArgs ga = gemm_args(M, C, 4 * C);
      ga.A = a.dbig; ga.lda = 4 * C;
      ga.B = W + y.off[T_WFC] + (size_t)l * 4 * C * C; ga.ldb = C; ga.b_mn = 1;
      ga.epi = EPI_STORE;
      ga.out = a.dh; ga.ldo = C;
      GPT2_TRY(run_gemm(h, ga));
    }
    {  // dWfc += du^T h2
      GemmArgs ga = gemm_args(4 * C, C, M);
      ga.A = a.dbig; ga.lda = 4 * C; ga.a_mn = 1;
      ga.B = h2; ga.ldb = C; ga.b_mn = 1;
      ga.epi = EPI_F32_ACC;
      ga.out32 = G + y.off[T_WFC] + (size_t)l * 4 * C * C; ga.ldo32 = C;
      ga.split_ws = a.splitk; ga.split_ws_floats = a.splitk_floats; ga.max_splits = kMaxSplits;
      ga.acc_zero = acc_zero;
      GPT2_TRY(run_gemm(h, ga));
    }
    mark(h, PK_LN_BWD);
    // dres = d x_mid; its column sum is the bias gradient of W_o
    layernorm_bwd(a.dres, a.dh, xm, a.mean2 + (size_t)l * M, a.rstd2 + (size_t)l * M,
                  P + y.off[T_LN2G] + (size_t)l * C, G + y.off[T_LN2G] + (size_t)l * C,
                  G + y.off[T_LN2B] + (size_t)l * C, G + y.off[T_BO] + (size_t)l * C,
                  slice(ln_part, a.partials), M, C, 1, s, dj);
    queue();
    // ---- attention: xm = x + att Wo^T + bo
    {  // datt = dres Wo
      GemmArgs ga = gemm_args(M, C, C);
      ga.A = a.dres; ga.lda = C;
      ga.B = W + y.off[T_WO] + (size_t)l * C * C; ga.ldb = C; ga.b_mn = 1;
      ga.epi = EPI_STORE;
      ga.out = a.datt; ga.ldo = C;
      GPT2_TRY(run_gemm(h, ga));
    }
    mark(h, PK_ATTN_BWD, 10.0 * B * H * (double)T * (T + 1) / 2 * (C / H));
    GPT2_CUDA(h, attention_bwd(a.dqkv, a.dsum, a.datt, qkv, att, a.lse + (size_t)l * M * H, B, T,
                               C, H, h->err, s));
    // the bias gradient of W_qkv while dqkv is still in L2
    mark(h, PK_COLSUM);
    colsum_acc(G + y.off[T_BQKV] + (size_t)l * 3 * C, a.dqkv, M, 3 * C,
               slice((size_t)kColsumChunks * 3 * C, a.partials), s, dj);
    queue();
    {  // dh = dqkv Wqkv
      GemmArgs ga = gemm_args(M, C, 3 * C);
      ga.A = a.dqkv; ga.lda = 3 * C;
      ga.B = W + y.off[T_WQKV] + (size_t)l * 3 * C * C; ga.ldb = C; ga.b_mn = 1;
      ga.epi = EPI_STORE;
      ga.out = a.dh; ga.ldo = C;
      GPT2_TRY(run_gemm(h, ga));
    }
    {  // dWqkv += dqkv^T h1, and in the same launch dWo += dres^T att (dres
       // still holds the gradient at x_mid): W_qkv's units alone would leave
       // CTA pairs idle (54 for 74 at GPT-2 124M), W_o's fill them
      GemmArgs ga = gemm_args(3 * C, C, M);
      ga.A = a.dqkv; ga.lda = 3 * C; ga.a_mn = 1;
      ga.B = h1; ga.ldb = C; ga.b_mn = 1;
      ga.epi = EPI_F32_ACC;
      ga.out32 = G + y.off[T_WQKV] + (size_t)l * 3 * C * C; ga.ldo32 = C;
      ga.M2 = C;
      ga.A2 = a.dres; ga.lda2 = C;
      ga.B2 = att; ga.ldb2 = C;
      ga.out32_2 = G + y.off[T_WO] + (size_t)l * C * C; ga.ldo32_2 = C;
      ga.split_ws = a.splitk; ga.split_ws_floats = a.splitk_floats; ga.max_splits = kMaxSplits;
      ga.acc_zero = acc_zero;
      GPT2_TRY(run_gemm(h, ga));
    }
    mark(h, PK_LN_BWD);
    // dres = d x_l = gradient at the output of layer l-1: bias of its W_p
    layernorm_bwd(a.dres, a.dh, x, a.mean1 + (size_t)l * M, a.rstd1 + (size_t)l * M,
                  P + y.off[T_LN1G] + (size_t)l * C, G + y.off[T_LN1G] + (size_t)l * C,
                  G + y.off[T_LN1B] + (size_t)l * C,
                  l > 0 ? G + y.off[T_BP] + (size_t)(l - 1) * C : nullptr,
                  slice(ln_part, a.partials), M, C, 1, s, dj);
    queue();
    if (!h->bwd_events.empty()) GPT2_CUDA(h, cudaEventRecord(h->bwd_events[l], s));
  }
  if (defer) {
    mark(h, PK_COLSUM);
    reduce_jobs_run(jobs, s);
  }
  mark(h, PK_ENCODER);
  encoder_bwd(G + y.off[T_WTE], G + y.off[T_WPE], a.dres, a.tok, B, T, C, y.Vp, es, s);
  mark_end(h);
  if (!h->bwd_events.empty()) GPT2_CUDA(h, cudaEventRecord(h->bwd_events[L], s));
  GPT2_CUDA(h, cudaGetLastError());
  h->have_grad_logits = false;
  return GPT2_OK;
}

gpt2_status gpt2_grad_norm_clip(gpt2_t* h, float max_norm, float* norm_host) {
  if (!h) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  mark(h, PK_OPTIMIZER);
  grad_norm_clip(h->scalars, h->grads, h->lay.total, max_norm, h->norm_partials, h->stream);
  mark_end(h);
  GPT2_CUDA(h, cudaGetLastError());
  if (norm_host) {
    GPT2_CUDA(h, cudaMemcpyAsync(norm_host, h->scalars + S_NORM, sizeof(float),
                                 cudaMemcpyDeviceToHost, h->stream));
    st = check_err_word(h);
    if (st) return st;
    if (!std::isfinite(*norm_host))
      return fail(h, GPT2_ERR_NONFINITE, "gradient norm is not finite");
  }
  return GPT2_OK;
}

}  // extern "C"

namespace {

// One AdamW step: the device step counter advances, the step's learning
// rate (given, or from the schedule on the device) and bias corrections
// land in device scalars, then the fused update runs.
gpt2_status adamw_impl(gpt2_t* h, float lr, const double* sched, float beta1, float beta2,
                       float eps, float weight_decay, size_t begin = 0, size_t end = (size_t)-1) {
  if (!h) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  if (end > h->lay.total) end = h->lay.total;
  AdamArgs a;
  a.b1 = beta1; a.b2 = beta2; a.eps = eps; a.wd = weight_decay;
  mark(h, PK_OPTIMIZER);
  adam_prep(h->scalars, h->dstep, lr, sched != nullptr, sched, beta1, beta2, h->stream);
  adamw(h->params, h->pact, h->grads, h->m, h->v, h->lay, a, h->scalars, h->stream, begin, end);
  GPT2_CUDA(h, cudaGetLastError());
  reset_clip(h->scalars, h->stream);  // the clip scale applies to one step only
  mark_end(h);
  GPT2_CUDA(h, cudaGetLastError());
  return GPT2_OK;
}

}  // namespace

extern "C" {

gpt2_status gpt2_adamw_step(gpt2_t* h, float lr, float beta1, float beta2, float eps,
                            float weight_decay) {
  return adamw_impl(h, lr, nullptr, beta1, beta2, eps, weight_decay);
}

gpt2_status gpt2_adamw_step_scheduled(gpt2_t* h, double max_lr, double min_lr, long warmup,
                                      long max_steps, float beta1, float beta2, float eps,
                                      float weight_decay) {
  if (warmup < 1 || max_steps < 0) return fail(h, GPT2_ERR_ARG, "bad schedule");
  const double sched[4] = {max_lr, min_lr, (double)warmup, (double)max_steps};
  return adamw_impl(h, 0.f, sched, beta1, beta2, eps, weight_decay);
}

gpt2_status gpt2_adamw_step_range(gpt2_t* h, float lr, float beta1, float beta2, float eps,
                                  float weight_decay, size_t begin, size_t end) {
  if (!h || begin > end || (begin & 3) || (end < h->lay.total && ((end - begin) & 3)))
    return fail(h, GPT2_ERR_ARG, "AdamW range: begin and length must be multiples of 4");
  return adamw_impl(h, lr, nullptr, beta1, beta2, eps, weight_decay, begin, end);
}

size_t gpt2_padded_params(const gpt2_t* h) { return h ? padded_params(h->lay) : 0; }

gpt2_status gpt2_grad_sumsq(gpt2_t* h, size_t begin, size_t end, double* sumsq_dev) {
  if (!h || !sumsq_dev || begin > end) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  if (end > padded_params(h->lay)) return fail(h, GPT2_ERR_ARG, "range past the padded buffer");
  if ((begin & 3) || (reinterpret_cast<uintptr_t>(sumsq_dev) & 7))
    return fail(h, GPT2_ERR_ARG, "begin must be a multiple of 4, sumsq_dev 8-byte aligned");
  mark(h, PK_OPTIMIZER);
  grad_sumsq(sumsq_dev, h->grads + begin, end - begin, h->norm_partials, h->stream);
  mark_end(h);
  GPT2_CUDA(h, cudaGetLastError());
  return GPT2_OK;
}

gpt2_status gpt2_clip_from_sumsq(gpt2_t* h, const double* sumsq_dev, float max_norm,
                                 float* norm_host) {
  if (!h || !sumsq_dev) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  clip_from_sumsq(h->scalars, sumsq_dev, max_norm, h->stream);
  GPT2_CUDA(h, cudaGetLastError());
  if (norm_host) {
    GPT2_CUDA(h, cudaMemcpyAsync(norm_host, h->scalars + S_NORM, sizeof(float),
                                 cudaMemcpyDeviceToHost, h->stream));
    st = check_err_word(h);
    if (st) return st;
    if (!std::isfinite(*norm_host))
      return fail(h, GPT2_ERR_NONFINITE, "gradient norm is not finite");
  }
  return GPT2_OK;
}

gpt2_status gpt2_params_device(gpt2_t* h, float** dev_ptr) {
  if (!h || !dev_ptr) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  *dev_ptr = h->params;
  return GPT2_OK;
}

gpt2_status gpt2_refresh_weights(gpt2_t* h) {
  if (!h) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
#if GPT2_ACT_BF16
  f32_to_act(h->pact, h->params, h->lay.total, h->stream);
  GPT2_CUDA(h, cudaGetLastError());
#endif
  return GPT2_OK;
}

gpt2_status gpt2_set_backward_events(gpt2_t* h, void* const* events, int n) {
  if (!h || n < 0 || (n > 0 && !events)) return GPT2_ERR_ARG;
  if (n && n != h->lay.L + 1) return fail(h, GPT2_ERR_ARG, "backward events: n must be L + 1 or 0");
  h->bwd_events.clear();
  for (int i = 0; i < n; ++i) h->bwd_events.push_back(static_cast<cudaEvent_t>(events[i]));
  return GPT2_OK;
}

gpt2_status gpt2_step_graph_capture(gpt2_t* h, const int32_t* tok_dev, const int32_t* tgt_dev,
                                    int B, int T, int n_micro, float max_norm, double max_lr,
                                    double min_lr, long warmup, long max_steps, float beta1,
                                    float beta2, float eps, float weight_decay) {
  if (!h || !tok_dev || !tgt_dev || B < 1 || T < 1 || n_micro < 1 || warmup < 1)
    return fail(h, GPT2_ERR_ARG, "bad step-graph arguments");
  if (!h->stream) return fail(h, GPT2_ERR_STATE, "capturing needs a stream set by gpt2_set_stream");
  if (h->prof) return fail(h, GPT2_ERR_STATE, "capturing with profiling on");
  if (!h->bwd_events.empty()) return fail(h, GPT2_ERR_STATE, "capturing with backward events set");
  if (T > h->lay.Tmax) return fail(h, GPT2_ERR_ARG, "T > Tmax");
  gpt2_status st = ensure_state(h);
  if (st) return st;
  st = ensure_work(h, B, T);  // no allocation may happen while capturing
  if (st) return st;
  if (h->graph_exec) cudaGraphExecDestroy(h->graph_exec);
  if (h->graph) cudaGraphDestroy(h->graph);
  h->graph_exec = nullptr;
  h->graph = nullptr;
  const long n0 = launch_count();
  GPT2_CUDA(h, cudaStreamBeginCapture(h->stream, cudaStreamCaptureModeThreadLocal));
  const size_t M = (size_t)B * T;
  st = gpt2_zero_grad(h);
  for (int i = 0; i < n_micro && !st; ++i) {
    st = forward_impl(h, tok_dev + i * M, tgt_dev + i * M, B, T, nullptr, true);
    if (!st) st = gpt2_backward(h, 1.0f / (float)n_micro);
  }
  if (!st) st = gpt2_grad_norm_clip(h, max_norm, nullptr);
  if (!st)
    st = gpt2_adamw_step_scheduled(h, max_lr, min_lr, warmup, max_steps, beta1, beta2, eps,
                                   weight_decay);
  cudaGraph_t g = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(h->stream, &g);
  if (st) {
    if (g) cudaGraphDestroy(g);
    return st;
  }
  if (ec != cudaSuccess) return cuda_fail(h, ec, "cudaStreamEndCapture");
  cudaGraphExec_t ex = nullptr;
  const cudaError_t ei = cudaGraphInstantiate(&ex, g, 0);
  if (ei != cudaSuccess) {
    cudaGraphDestroy(g);
    return cuda_fail(h, ei, "cudaGraphInstantiate");
  }
  h->graph = g;
  h->graph_exec = ex;
  h->graph_launches = launch_count() - n0;
  // the one-time upload of the graph to the device, here rather than in the
  // first replay
  GPT2_CUDA(h, cudaGraphUpload(ex, h->stream));
  return GPT2_OK;
}

gpt2_status gpt2_step_graph_launch(gpt2_t* h) {
  if (!h) return GPT2_ERR_ARG;
  if (!h->graph_exec) return fail(h, GPT2_ERR_STATE, "no captured step");
  GPT2_CUDA(h, cudaGraphLaunch(h->graph_exec, h->stream));
  return GPT2_OK;
}

long gpt2_step_graph_kernels(const gpt2_t* h) { return h ? h->graph_launches : 0; }

double gpt2_lr(long step, double max_lr, double min_lr, long warmup, long max_steps) {
  if (step < warmup) return max_lr * (double)(step + 1) / (double)warmup;
  if (step > max_steps || max_steps <= warmup) return min_lr;
  const double ratio = (double)(step - warmup) / (double)(max_steps - warmup);
  return min_lr + 0.5 * (1.0 + std::cos(M_PI * ratio)) * (max_lr - min_lr);
}

gpt2_status gpt2_get_params(const gpt2_t* hc, float* host) {
  gpt2_t* h = const_cast<gpt2_t*>(hc);
  if (!h || !host) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  GPT2_CUDA(h, cudaMemcpyAsync(host, h->params, h->lay.total * 4, cudaMemcpyDeviceToHost, h->stream));
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  return GPT2_OK;
}

gpt2_status gpt2_set_params(gpt2_t* h, const float* host) {
  if (!h || !host) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  GPT2_CUDA(h, cudaMemcpyAsync(h->params, host, h->lay.total * 4, cudaMemcpyHostToDevice, h->stream));
#if GPT2_ACT_BF16
  f32_to_act(h->pact, h->params, h->lay.total, h->stream);
  GPT2_CUDA(h, cudaGetLastError());
#endif
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  return GPT2_OK;
}

gpt2_status gpt2_get_grads(const gpt2_t* hc, float* host) {
  gpt2_t* h = const_cast<gpt2_t*>(hc);
  if (!h || !host) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  GPT2_CUDA(h, cudaMemcpyAsync(host, h->grads, h->lay.total * 4, cudaMemcpyDeviceToHost, h->stream));
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  return GPT2_OK;
}

gpt2_status gpt2_grads_device(gpt2_t* h, float** dev_ptr) {
  if (!h || !dev_ptr) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  *dev_ptr = h->grads;
  return GPT2_OK;
}

gpt2_status gpt2_get_state(const gpt2_t* hc, float* params, float* m, float* v, long* t) {
  gpt2_t* h = const_cast<gpt2_t*>(hc);
  if (!h) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  const size_t n = h->lay.total * 4;
  if (params) GPT2_CUDA(h, cudaMemcpyAsync(params, h->params, n, cudaMemcpyDeviceToHost, h->stream));
  if (m) GPT2_CUDA(h, cudaMemcpyAsync(m, h->m, n, cudaMemcpyDeviceToHost, h->stream));
  if (v) GPT2_CUDA(h, cudaMemcpyAsync(v, h->v, n, cudaMemcpyDeviceToHost, h->stream));
  int ti = 0;
  GPT2_CUDA(h, cudaMemcpyAsync(&ti, h->dstep, sizeof(int), cudaMemcpyDeviceToHost, h->stream));
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  if (t) *t = ti;
  return GPT2_OK;
}

gpt2_status gpt2_set_state(gpt2_t* h, const float* params, const float* m, const float* v, long t) {
  if (!h || t < 0 || t > 0x7fffffffL) return GPT2_ERR_ARG;
  gpt2_status st = ensure_state(h);
  if (st) return st;
  const size_t n = h->lay.total * 4;
  if (params) {
    GPT2_CUDA(h, cudaMemcpyAsync(h->params, params, n, cudaMemcpyHostToDevice, h->stream));
#if GPT2_ACT_BF16
    f32_to_act(h->pact, h->params, h->lay.total, h->stream);
    GPT2_CUDA(h, cudaGetLastError());
#endif
  }
  if (m) GPT2_CUDA(h, cudaMemcpyAsync(h->m, m, n, cudaMemcpyHostToDevice, h->stream));
  if (v) GPT2_CUDA(h, cudaMemcpyAsync(h->v, v, n, cudaMemcpyHostToDevice, h->stream));
  const int ti = (int)t;
  GPT2_CUDA(h, cudaMemcpyAsync(h->dstep, &ti, sizeof(int), cudaMemcpyHostToDevice, h->stream));
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  return GPT2_OK;
}

gpt2_status gpt2_tensor_info(const gpt2_t* h, int i, const char** name, int* ndim,
                             int64_t shape[3], size_t* offset) {
  static const char* names[T_COUNT] = {"wte", "wpe", "ln1_g", "ln1_b", "w_qkv", "b_qkv",
                                       "w_o", "b_o", "ln2_g", "ln2_b", "w_fc", "b_fc",
                                       "w_p", "b_p", "lnf_g", "lnf_b"};
  if (!h || i < 0 || i >= T_COUNT) return GPT2_ERR_ARG;
  const Layout& y = h->lay;
  int64_t sh[3] = {0, 0, 0};
  int nd = 0;
  const int64_t L = y.L, C = y.C;
  switch (i) {
    case T_WTE: nd = 2; sh[0] = y.Vp; sh[1] = C; break;
    case T_WPE: nd = 2; sh[0] = y.Tmax; sh[1] = C; break;
    case T_WQKV: nd = 3; sh[0] = L; sh[1] = 3 * C; sh[2] = C; break;
    case T_BQKV: nd = 2; sh[0] = L; sh[1] = 3 * C; break;
    case T_WO: nd = 3; sh[0] = L; sh[1] = C; sh[2] = C; break;
    case T_WFC: nd = 3; sh[0] = L; sh[1] = 4 * C; sh[2] = C; break;
    case T_BFC: nd = 2; sh[0] = L; sh[1] = 4 * C; break;
    case T_WP: nd = 3; sh[0] = L; sh[1] = C; sh[2] = 4 * C; break;
    case T_LNFG: case T_LNFB: nd = 1; sh[0] = C; break;
    default: nd = 2; sh[0] = L; sh[1] = C; break;
  }
  if (name) *name = names[i];
  if (ndim) *ndim = nd;
  if (shape) for (int k = 0; k < 3; ++k) shape[k] = sh[k];
  if (offset) *offset = y.off[i];
  return GPT2_OK;
}

gpt2_status gpt2_logits(const gpt2_t* h, const void** dev_ptr) {
  if (!h || !dev_ptr) return GPT2_ERR_ARG;
  if (!h->have_logits) return GPT2_ERR_STATE;
  *dev_ptr = h->a.logits;
  return GPT2_OK;
}

gpt2_status gpt2_get_losses(const gpt2_t* hc, float* host, size_t n) {
  gpt2_t* h = const_cast<gpt2_t*>(hc);
  if (!h || !host || !h->work) return GPT2_ERR_ARG;
  if (n > (size_t)h->B * h->T) return fail(h, GPT2_ERR_ARG, "n > B*T");
  GPT2_CUDA(h, cudaMemcpyAsync(host, h->a.losses, n * 4, cudaMemcpyDeviceToHost, h->stream));
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  return GPT2_OK;
}

gpt2_status gpt2_read_activation(const gpt2_t* hc, int kind, int layer, float* host, size_t n) {
  gpt2_t* h = const_cast<gpt2_t*>(hc);
  if (!h || !host || !h->work) return GPT2_ERR_ARG;
  const Layout& y = h->lay;
  const size_t M = (size_t)h->B * h->T, C = y.C;
  const Acts& a = h->a;
  const act_t* src = nullptr;
  size_t cnt = 0;
  if (layer < 0 || layer > y.L || (kind != 0 && kind != 8 && layer == y.L)) return GPT2_ERR_ARG;
  switch (kind) {
    case 0: src = a.res + layer * M * C; cnt = M * C; break;
    case 1: src = a.h1 + layer * M * C; cnt = M * C; break;
    case 2: src = a.qkv + layer * 3 * M * C; cnt = 3 * M * C; break;
    case 3: src = a.att + layer * M * C; cnt = M * C; break;
    case 4: src = a.xmid + layer * M * C; cnt = M * C; break;
    case 5: src = a.h2 + layer * M * C; cnt = M * C; break;
    case 6: src = a.u + layer * 4 * M * C; cnt = 4 * M * C; break;
    case 7:
      if (h->recompute) return fail(h, GPT2_ERR_STATE, "GELU outputs are not kept (recompute)");
      src = a.g + layer * 4 * M * C;
      cnt = 4 * M * C;
      break;
    case 8: src = a.hf; cnt = M * C; break;
    default: return GPT2_ERR_ARG;
  }
  if (n != cnt) return fail(h, GPT2_ERR_ARG, "n does not match the activation size");
#if GPT2_ACT_BF16
  std::vector<uint16_t> tmp(cnt);
  GPT2_CUDA(h, cudaMemcpyAsync(tmp.data(), src, cnt * 2, cudaMemcpyDeviceToHost, h->stream));
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  for (size_t i = 0; i < cnt; ++i) {
    const uint32_t bits = (uint32_t)tmp[i] << 16;
    std::memcpy(host + i, &bits, 4);
  }
#else
  GPT2_CUDA(h, cudaMemcpyAsync(host, src, cnt * 4, cudaMemcpyDeviceToHost, h->stream));
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
#endif
  return GPT2_OK;
}

const char* gpt2_last_error(const gpt2_t* h) { return h ? h->last_error.c_str() : "null handle"; }

long gpt2_launch_count(void) { return launch_count(); }

gpt2_status gpt2_profile_enable(gpt2_t* h, int on) {
  if (!h) return GPT2_ERR_ARG;
  h->prof = on != 0;
  return GPT2_OK;
}

gpt2_status gpt2_profile_read(gpt2_t* h, double* ms, long* launches, double* flops, int kinds) {
  if (!h || kinds < PK_COUNT) return GPT2_ERR_ARG;
  for (int k = 0; k < kinds; ++k) {
    if (ms) ms[k] = 0;
    if (launches) launches[k] = 0;
    if (flops) flops[k] = 0;
  }
  mark_end(h);
  GPT2_CUDA(h, cudaStreamSynchronize(h->stream));
  std::vector<cudaEvent_t> used;
  for (const ProfRec& r : h->recs) {
    if (r.b) {
      float t = 0.f;
      GPT2_CUDA(h, cudaEventElapsedTime(&t, r.a, r.b));
      if (ms) ms[r.kind] += t;
      if (launches) launches[r.kind] += 1;
      if (flops) flops[r.kind] += r.flops;
      used.push_back(r.b);
    }
    used.push_back(r.a);
  }
  std::sort(used.begin(), used.end());
  used.erase(std::unique(used.begin(), used.end()), used.end());
  h->ev_pool.insert(h->ev_pool.end(), used.begin(), used.end());
  h->recs.clear();
  return GPT2_OK;
}

}  // extern "C"
