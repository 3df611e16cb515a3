// GPT-2 pretraining step: plain CPU oracle.
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct CPU
// statement of one GPT-2 pretraining step (forward, backward, global-norm
// clip, AdamW, LR schedule, parameter init).  Only the test suite, the smoke
// check and the benchmark's CPU-baseline leg may load it.  It shares no code,
// header, table or helper with the CUDA library, and the CUDA library never
// calls it.
//
// What it follows (page: section):
//  * Model: "Let's reproduce GPT-2 (124M)" condensed (sotaaz.com),
//    section 1 -- GPT-2 small as a plain module, token embedding tied to the
//    output layer, N(0, 0.02) init with the projections that are added to
//    the residual stream scaled by 1/sqrt(2 * n_layer).
//  * GELU: same page, "nanoGPT's GELU differs from GPT-2" -- GPT-2 uses the
//    tanh approximation, 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).
//  * Vocabulary padding: same page, section 2 (the last speed-up step pads
//    the vocabulary); padded logits are excluded from the softmax.
//  * Optimiser: same page, section 3 -- AdamW beta = (0.9, 0.95),
//    eps = 1e-8, gradients clipped to global norm 1.0, linear warmup then
//    cosine decay to 10 % of the maximum LR, weight decay 0.1 on 2-D
//    parameters (matmul weights and embeddings) only, and gradient
//    accumulation with the loss divided by the number of micro-batches.
//  * The same recipe at small scale: "TinyStories training" (lameproof.com),
//    the training excerpt (lr 1e-3, warmup 200, wd 0.1, clip 1.0, bf16).
//
// Readings where the pages are silent (each also listed in the design notes):
//  LayerNorm eps = 1e-5 with the biased (1/C) variance; attention scale
//  1/sqrt(head_dim), strictly causal, no dropout; no LM-head bias; padded
//  rows of wte start at 0; loss is the mean over all B*T positions; AdamW is
//  decoupled (p -= lr * (mhat / (sqrt(vhat) + eps) + wd * p)) with step t
//  counted from 1; clip scales by max_norm / (norm + 1e-6) only when
//  norm > max_norm; warmup uses (step + 1) / warmup.
//
// Every computation is written as plain loops in the order of the
// definitions.  Loops carry `omp parallel for` only over independent output
// elements, so a -fopenmp build gives results bit-identical to the
// single-threaded build (each output's reduction order is unchanged).

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <vector>
#include <algorithm>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------- layout --
// Flat parameter order (one slice per tensor, row-major, y = x W^T + b):
//  0 wte[Vp,C] 1 wpe[Tmax,C] 2 ln1_g[L,C] 3 ln1_b[L,C] 4 w_qkv[L,3C,C]
//  5 b_qkv[L,3C] 6 w_o[L,C,C] 7 b_o[L,C] 8 ln2_g[L,C] 9 ln2_b[L,C]
//  10 w_fc[L,4C,C] 11 b_fc[L,4C] 12 w_p[L,C,4C] 13 b_p[L,C] 14 lnf_g[C]
//  15 lnf_b[C]
enum { WTE, WPE, LN1G, LN1B, WQKV, BQKV, WO, BO, LN2G, LN2B, WFC, BFC, WP, BP,
       LNFG, LNFB, NT };

struct Cfg {
  int L, H, C, V, Vp, Tmax;
  size_t off[NT];
  size_t num[NT];
  size_t total;
};

Cfg make_cfg(int L, int H, int C, int V, int Vp, int Tmax) {
  Cfg g;
  g.L = L; g.H = H; g.C = C; g.V = V; g.Vp = Vp; g.Tmax = Tmax;
  const size_t l = (size_t)L, c = (size_t)C;
  g.num[WTE] = (size_t)Vp * c;
  g.num[WPE] = (size_t)Tmax * c;
  g.num[LN1G] = l * c;      g.num[LN1B] = l * c;
  g.num[WQKV] = l * 3 * c * c; g.num[BQKV] = l * 3 * c;
  g.num[WO] = l * c * c;    g.num[BO] = l * c;
  g.num[LN2G] = l * c;      g.num[LN2B] = l * c;
  g.num[WFC] = l * 4 * c * c; g.num[BFC] = l * 4 * c;
  g.num[WP] = l * 4 * c * c;  g.num[BP] = l * c;
  g.num[LNFG] = c;          g.num[LNFB] = c;
  size_t o = 0;
  for (int i = 0; i < NT; ++i) { g.off[i] = o; o += g.num[i]; }
  g.total = o;
  return g;
}

// 2-D tensors (matmul weights and embeddings) are weight-decayed.
bool is_decayed(int tensor) {
  return tensor == WTE || tensor == WPE || tensor == WQKV || tensor == WO ||
         tensor == WFC || tensor == WP;
}

// ------------------------------------------------------------ init RNG --
// SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014): the n-th output of a generator seeded with s is
// mix(s + n * GAMMA).  Tensor tau draws from the generator seeded with the
// (tau+1)-th output of the master generator seeded with `seed`; element i
// uses that generator's outputs 2i+1 and 2i+2 for one Box-Muller normal
// (Box & Muller 1958, cosine branch), computed in double, rounded once.
const uint64_t GAMMA = 0x9E3779B97F4A7C15ull;

uint64_t sm_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t sm_output(uint64_t seed, uint64_t n) { return sm_mix(seed + n * GAMMA); }

double std_normal(uint64_t tensor_seed, uint64_t i) {
  const uint64_t r1 = sm_output(tensor_seed, 2 * i + 1);
  const uint64_t r2 = sm_output(tensor_seed, 2 * i + 2);
  const double u1 = (double)((r1 >> 11) + 1) * 0x1.0p-53;  // (0, 1]
  const double u2 = (double)(r2 >> 11) * 0x1.0p-53;        // [0, 1)
  return std::sqrt(-2.0 * std::log(u1)) * std::cos(2.0 * M_PI * u2);
}

template <class R>
void init_params(const Cfg& g, uint64_t seed, R* p) {
  std::fill(p, p + g.total, R(0));
  const double sd = 0.02;
  const double sd_res = 0.02 / std::sqrt(2.0 * g.L);
  for (int t = 0; t < NT; ++t) {
    const uint64_t ts = sm_output(seed, (uint64_t)t + 1);
    R* dst = p + g.off[t];
    size_t count = g.num[t];
    double s = 0.0;
    switch (t) {
      case WTE: count = (size_t)g.V * g.C; s = sd; break;  // pad rows stay 0
      case WPE: case WQKV: case WFC: s = sd; break;
      case WO: case WP: s = sd_res; break;
      case LN1G: case LN2G: case LNFG:
        for (size_t i = 0; i < count; ++i) dst[i] = R(1);
        continue;
      default: continue;  // biases and LN betas: 0
    }
    for (size_t i = 0; i < count; ++i)
      dst[i] = (R)(float)(s * std_normal(ts, i));
  }
}

// ------------------------------------------------------------ primitives --
template <class R> R gelu_tanh(R x) {
  const R k = std::sqrt(R(2) / R(M_PI));
  return R(0.5) * x * (R(1) + std::tanh(k * (x + R(0.044715) * x * x * x)));
}

template <class R> R gelu_tanh_grad(R x) {
  const R k = std::sqrt(R(2) / R(M_PI));
  const R inner = k * (x + R(0.044715) * x * x * x);
  const R th = std::tanh(inner);
  const R dinner = k * (R(1) + R(3) * R(0.044715) * x * x);
  return R(0.5) * (R(1) + th) + R(0.5) * x * (R(1) - th * th) * dinner;
}

template <class R> R gelu_erf(R x) {
  return R(0.5) * x * (R(1) + std::erf(x / std::sqrt(R(2))));
}

const double LN_EPS = 1e-5;

// y = (x - mean) * rstd * g + b, biased variance.
template <class R>
void layernorm_fwd(const R* x, const R* g, const R* b, R* y, R* mean, R* rstd,
                   int M, int C) {
#pragma omp parallel for
  for (int m = 0; m < M; ++m) {
    const R* xr = x + (size_t)m * C;
    R s = 0;
    for (int c = 0; c < C; ++c) s += xr[c];
    const R mu = s / C;
    R v = 0;
    for (int c = 0; c < C; ++c) v += (xr[c] - mu) * (xr[c] - mu);
    v /= C;
    const R rs = R(1) / std::sqrt(v + R(LN_EPS));
    R* yr = y + (size_t)m * C;
    for (int c = 0; c < C; ++c) yr[c] = (xr[c] - mu) * rs * g[c] + b[c];
    mean[m] = mu;
    rstd[m] = rs;
  }
}

// dx += rstd * (dxhat - mean(dxhat) - xhat * mean(dxhat * xhat)),
// dxhat = dy * g;  dg += sum_m dy * xhat;  db += sum_m dy.
template <class R>
void layernorm_bwd(const R* x, const R* g, const R* mean, const R* rstd,
                   const R* dy, R* dx, R* dg, R* db, int M, int C) {
#pragma omp parallel for
  for (int m = 0; m < M; ++m) {
    const R* xr = x + (size_t)m * C;
    const R* dyr = dy + (size_t)m * C;
    R a = 0, bsum = 0;
    for (int c = 0; c < C; ++c) {
      const R xh = (xr[c] - mean[m]) * rstd[m];
      const R dxh = dyr[c] * g[c];
      a += dxh;
      bsum += dxh * xh;
    }
    a /= C;
    bsum /= C;
    R* dxr = dx + (size_t)m * C;
    for (int c = 0; c < C; ++c) {
      const R xh = (xr[c] - mean[m]) * rstd[m];
      const R dxh = dyr[c] * g[c];
      dxr[c] += rstd[m] * (dxh - a - xh * bsum);
    }
  }
#pragma omp parallel for
  for (int c = 0; c < C; ++c) {
    R sg = 0, sb = 0;
    for (int m = 0; m < M; ++m) {
      const R xh = (x[(size_t)m * C + c] - mean[m]) * rstd[m];
      sg += dy[(size_t)m * C + c] * xh;
      sb += dy[(size_t)m * C + c];
    }
    dg[c] += sg;
    db[c] += sb;
  }
}

// y[m,n] = sum_k x[m,k] W[n,k] (+ b[n])
template <class R>
void linear_fwd(const R* x, const R* W, const R* b, R* y, int M, int K, int N) {
#pragma omp parallel for
  for (int m = 0; m < M; ++m) {
    const R* xr = x + (size_t)m * K;
    for (int n = 0; n < N; ++n) {
      const R* wr = W + (size_t)n * K;
      R s = 0;
      for (int k = 0; k < K; ++k) s += xr[k] * wr[k];
      y[(size_t)m * N + n] = b ? s + b[n] : s;
    }
  }
}

// dx[m,k] += sum_n dy[m,n] W[n,k];  dW[n,k] += sum_m dy[m,n] x[m,k];
// db[n] += sum_m dy[m,n]  (dx, db may be null)
template <class R>
void linear_bwd(const R* x, const R* W, const R* dy, R* dx, R* dW, R* db,
                int M, int K, int N) {
  if (dx) {
#pragma omp parallel for
    for (int m = 0; m < M; ++m) {
      R* dxr = dx + (size_t)m * K;
      std::vector<R> acc(K, R(0));
      for (int n = 0; n < N; ++n) {
        const R d = dy[(size_t)m * N + n];
        const R* wr = W + (size_t)n * K;
        for (int k = 0; k < K; ++k) acc[k] += d * wr[k];
      }
      for (int k = 0; k < K; ++k) dxr[k] += acc[k];
    }
  }
#pragma omp parallel for
  for (int n = 0; n < N; ++n) {
    std::vector<R> acc(K, R(0));
    R sb = 0;
    for (int m = 0; m < M; ++m) {
      const R d = dy[(size_t)m * N + n];
      const R* xr = x + (size_t)m * K;
      for (int k = 0; k < K; ++k) acc[k] += d * xr[k];
      sb += d;
    }
    R* dwr = dW + (size_t)n * K;
    for (int k = 0; k < K; ++k) dwr[k] += acc[k];
    if (db) db[n] += sb;
  }
}

// Causal multi-head attention over qkv[M, 3C] = [q | k | v]; head h uses
// columns h*hd .. h*hd+hd-1 of each part.  y[m, h*hd + d].
template <class R>
void attention_fwd(const R* qkv, R* y, int B, int T, int C, int H) {
  const int hd = C / H;
  const R scale = R(1) / std::sqrt(R(hd));
#pragma omp parallel for collapse(2)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      std::vector<R> s(T);
      for (int i = 0; i < T; ++i) {
        const R* q = qkv + ((size_t)b * T + i) * 3 * C + h * hd;
        R mx = -INFINITY;
        for (int j = 0; j <= i; ++j) {
          const R* k = qkv + ((size_t)b * T + j) * 3 * C + C + h * hd;
          R d = 0;
          for (int e = 0; e < hd; ++e) d += q[e] * k[e];
          s[j] = d * scale;
          mx = std::max(mx, s[j]);
        }
        R z = 0;
        for (int j = 0; j <= i; ++j) { s[j] = std::exp(s[j] - mx); z += s[j]; }
        R* yr = y + ((size_t)b * T + i) * C + h * hd;
        for (int e = 0; e < hd; ++e) yr[e] = 0;
        for (int j = 0; j <= i; ++j) {
          const R p = s[j] / z;
          const R* v = qkv + ((size_t)b * T + j) * 3 * C + 2 * C + h * hd;
          for (int e = 0; e < hd; ++e) yr[e] += p * v[e];
        }
      }
    }
}

// Backward of attention_fwd: recomputes each softmax row.
// dq_i = scale sum_j ds_ij k_j, dk_j = scale sum_i ds_ij q_i,
// dv_j = sum_i p_ij dy_i, ds_ij = p_ij (dp_ij - sum_l p_il dp_il),
// dp_ij = dy_i . v_j.   dqkv is overwritten.
template <class R>
void attention_bwd(const R* qkv, const R* dy, R* dqkv, int B, int T, int C,
                   int H) {
  const int hd = C / H;
  const R scale = R(1) / std::sqrt(R(hd));
  std::fill(dqkv, dqkv + (size_t)B * T * 3 * C, R(0));
#pragma omp parallel for collapse(2)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      std::vector<R> p(T), dp(T);
      for (int i = 0; i < T; ++i) {
        const R* q = qkv + ((size_t)b * T + i) * 3 * C + h * hd;
        const R* dyi = dy + ((size_t)b * T + i) * C + h * hd;
        R mx = -INFINITY;
        for (int j = 0; j <= i; ++j) {
          const R* k = qkv + ((size_t)b * T + j) * 3 * C + C + h * hd;
          R d = 0;
          for (int e = 0; e < hd; ++e) d += q[e] * k[e];
          p[j] = d * scale;
          mx = std::max(mx, p[j]);
        }
        R z = 0;
        for (int j = 0; j <= i; ++j) { p[j] = std::exp(p[j] - mx); z += p[j]; }
        for (int j = 0; j <= i; ++j) p[j] /= z;
        R dsum = 0;
        for (int j = 0; j <= i; ++j) {
          const R* v = qkv + ((size_t)b * T + j) * 3 * C + 2 * C + h * hd;
          R d = 0;
          for (int e = 0; e < hd; ++e) d += dyi[e] * v[e];
          dp[j] = d;
          dsum += p[j] * d;
        }
        R* dq = dqkv + ((size_t)b * T + i) * 3 * C + h * hd;
        for (int j = 0; j <= i; ++j) {
          const R ds = p[j] * (dp[j] - dsum);
          const R* k = qkv + ((size_t)b * T + j) * 3 * C + C + h * hd;
          R* dk = dqkv + ((size_t)b * T + j) * 3 * C + C + h * hd;
          R* dv = dqkv + ((size_t)b * T + j) * 3 * C + 2 * C + h * hd;
          for (int e = 0; e < hd; ++e) {
            dq[e] += scale * ds * k[e];
            dk[e] += scale * ds * q[e];
            dv[e] += p[j] * dyi[e];
          }
        }
      }
    }
}

// ----------------------------------------------------------------- model --
// log sum_v exp(z[v]) over the first V logits of a row (max-shifted).
template <class R>
R row_lse(const R* z, int V) {
  R mx = -INFINITY;
  for (int v = 0; v < V; ++v) mx = std::max(mx, z[v]);
  R s = 0;
  for (int v = 0; v < V; ++v) s += std::exp(z[v] - mx);
  return mx + std::log(s);
}

// Softmax cross-entropy of M rows of V logits: losses[m] = lse_m - z[tgt[m]]
// and, when dz is given, dz = (softmax - onehot(tgt)) * scale / M.
template <class R>
void softmax_xent(const R* z, int M, int V, const int* tgt, R scale, R* losses, R* dz) {
  for (int m = 0; m < M; ++m) {
    const R* zr = z + (size_t)m * V;
    const R lse = row_lse(zr, V);
    if (losses) losses[m] = lse - zr[tgt[m]];
    if (!dz) continue;
    for (int v = 0; v < V; ++v) {
      R d = std::exp(zr[v] - lse);
      if (v == tgt[m]) d -= R(1);
      dz[(size_t)m * V + v] = d * scale / R(M);
    }
  }
}

// The next token from one row of V logits (generation loop of the pages).
// temperature 0: the argmax (lowest index among equal maxima).  Otherwise
// the softmax of z / temperature over the top_k largest logits (top_k <= 0
// or >= V: all of them; logits equal to the k-th largest are kept), and the
// token is the smallest v at which the cumulative probability exceeds u
// (u uniform in [0, 1), a draw the caller passes in).
template <class R>
int sample_token(const R* z, int V, R temperature, int top_k, double u) {
  int best = 0;
  for (int v = 1; v < V; ++v)
    if (z[v] > z[best]) best = v;
  if (temperature <= R(0)) return best;
  R thr = -INFINITY;
  if (top_k > 0 && top_k < V) {
    std::vector<R> sorted(z, z + V);
    std::nth_element(sorted.begin(), sorted.begin() + (top_k - 1), sorted.end(), std::greater<R>());
    thr = sorted[top_k - 1];
  }
  const R mx = z[best];
  R total = 0;
  for (int v = 0; v < V; ++v)
    if (z[v] >= thr) total += std::exp((z[v] - mx) / temperature);
  const R target = R(u) * total;
  R cum = 0;
  int last = best;
  for (int v = 0; v < V; ++v) {
    if (z[v] < thr) continue;
    cum += std::exp((z[v] - mx) / temperature);
    last = v;
    if (cum > target) return v;
  }
  return last;
}

template <class R>
struct Model {
  Cfg g;
  int B = 0, T = 0;
  // activations kept for the backward pass
  std::vector<R> x0;                         // encoder output [M,C]
  std::vector<std::vector<R>> xin, h1, m1, r1, qkv, att, xmid, h2, m2, r2, u, ge;
  std::vector<R> xL, hf, mf, rf, logits;     // logits [M,V]
  std::vector<R> lossv;                      // per position [M]
  const int* tok = nullptr;
  const int* tgt = nullptr;

  explicit Model(const Cfg& c) : g(c) {}

  const R* P(const R* p, int t, int l, size_t per) const {
    return p + g.off[t] + (size_t)l * per;
  }

  // Returns the mean loss when tgt != null (else 0).
  R forward(const R* p, const int* tok_, const int* tgt_, int B_, int T_) {
    B = B_; T = T_; tok = tok_; tgt = tgt_;
    const int C = g.C, L = g.L, M = B * T, V = g.V;
    const size_t MC = (size_t)M * C;
    x0.assign(MC, 0);
    for (int b = 0; b < B; ++b)
      for (int t = 0; t < T; ++t) {
        const int m = b * T + t;
        const R* we = p + g.off[WTE] + (size_t)tok[m] * C;
        const R* pe = p + g.off[WPE] + (size_t)t * C;
        for (int c = 0; c < C; ++c) x0[(size_t)m * C + c] = we[c] + pe[c];
      }
    auto rs = [&](std::vector<std::vector<R>>& v, size_t n) {
      v.assign(L, std::vector<R>(n));
    };
    rs(xin, MC); rs(h1, MC); rs(m1, M); rs(r1, M); rs(qkv, 3 * MC);
    rs(att, MC); rs(xmid, MC); rs(h2, MC); rs(m2, M); rs(r2, M);
    rs(u, 4 * MC); rs(ge, 4 * MC);
    const std::vector<R>* x = &x0;
    std::vector<R> tmp(MC), tmp4(4 * MC);
    for (int l = 0; l < L; ++l) {
      xin[l] = *x;
      layernorm_fwd(xin[l].data(), P(p, LN1G, l, C), P(p, LN1B, l, C),
                    h1[l].data(), m1[l].data(), r1[l].data(), M, C);
      linear_fwd(h1[l].data(), P(p, WQKV, l, (size_t)3 * C * C),
                 P(p, BQKV, l, 3 * C), qkv[l].data(), M, C, 3 * C);
      attention_fwd(qkv[l].data(), att[l].data(), B, T, C, g.H);
      linear_fwd(att[l].data(), P(p, WO, l, (size_t)C * C), P(p, BO, l, C),
                 tmp.data(), M, C, C);
      for (size_t i = 0; i < MC; ++i) xmid[l][i] = xin[l][i] + tmp[i];
      layernorm_fwd(xmid[l].data(), P(p, LN2G, l, C), P(p, LN2B, l, C),
                    h2[l].data(), m2[l].data(), r2[l].data(), M, C);
      linear_fwd(h2[l].data(), P(p, WFC, l, (size_t)4 * C * C),
                 P(p, BFC, l, 4 * C), u[l].data(), M, C, 4 * C);
      for (size_t i = 0; i < 4 * MC; ++i) ge[l][i] = gelu_tanh(u[l][i]);
      linear_fwd(ge[l].data(), P(p, WP, l, (size_t)4 * C * C), P(p, BP, l, C),
                 tmp.data(), M, 4 * C, C);
      if (l + 1 < L) {
        // next layer input; stored as xin[l+1] at the top of the loop
        for (size_t i = 0; i < MC; ++i) tmp[i] = xmid[l][i] + tmp[i];
        xL = tmp;
        x = &xL;
      } else {
        xL.resize(MC);
        for (size_t i = 0; i < MC; ++i) xL[i] = xmid[l][i] + tmp[i];
      }
    }
    if (L == 0) xL = x0;
    hf.resize(MC); mf.resize(M); rf.resize(M);
    layernorm_fwd(xL.data(), p + g.off[LNFG], p + g.off[LNFB], hf.data(),
                  mf.data(), rf.data(), M, C);
    // tied head over the real vocabulary only (padded columns are masked)
    logits.resize((size_t)M * V);
    linear_fwd(hf.data(), p + g.off[WTE], (const R*)nullptr, logits.data(), M,
               C, V);
    if (!tgt) return 0;
    lossv.resize(M);
    softmax_xent(logits.data(), M, V, tgt, R(1), lossv.data(), (R*)nullptr);
    R total = 0;
    for (int m = 0; m < M; ++m) total += lossv[m];
    return total / M;
  }

  // Accumulates d(loss_scale * mean loss)/dparam into grad.
  void backward(const R* p, R* grad, R loss_scale) {
    const int C = g.C, L = g.L, M = B * T, V = g.V;
    const size_t MC = (size_t)M * C;
    // softmax cross-entropy: dz = (softmax - onehot) * scale / M
    std::vector<R> dz((size_t)M * V);
    softmax_xent(logits.data(), M, V, tgt, loss_scale, (R*)nullptr, dz.data());
    std::vector<R> dhf(MC, 0), dx(MC, 0);
    linear_bwd(hf.data(), p + g.off[WTE], dz.data(), dhf.data(),
               grad + g.off[WTE], (R*)nullptr, M, C, V);
    layernorm_bwd(xL.data(), p + g.off[LNFG], mf.data(), rf.data(), dhf.data(),
                  dx.data(), grad + g.off[LNFG], grad + g.off[LNFB], M, C);
    std::vector<R> dge(4 * MC), du(4 * MC), dh(MC), datt(MC), dqkv(3 * MC);
    for (int l = L - 1; l >= 0; --l) {
      // x_out = xmid + gelu(h2 Wfc^T + bfc) Wp^T + bp
      std::fill(dge.begin(), dge.end(), R(0));
      linear_bwd(ge[l].data(), P(p, WP, l, (size_t)4 * C * C), dx.data(),
                 dge.data(), (R*)(grad + g.off[WP] + (size_t)l * 4 * C * C),
                 grad + g.off[BP] + (size_t)l * C, M, 4 * C, C);
      for (size_t i = 0; i < 4 * MC; ++i) du[i] = dge[i] * gelu_tanh_grad(u[l][i]);
      std::fill(dh.begin(), dh.end(), R(0));
      linear_bwd(h2[l].data(), P(p, WFC, l, (size_t)4 * C * C), du.data(),
                 dh.data(), grad + g.off[WFC] + (size_t)l * 4 * C * C,
                 grad + g.off[BFC] + (size_t)l * 4 * C, M, C, 4 * C);
      // dx now holds d xmid (residual path) + LN2 backward
      layernorm_bwd(xmid[l].data(), P(p, LN2G, l, C), m2[l].data(),
                    r2[l].data(), dh.data(), dx.data(),
                    grad + g.off[LN2G] + (size_t)l * C,
                    grad + g.off[LN2B] + (size_t)l * C, M, C);
      // xmid = xin + att Wo^T + bo
      std::fill(datt.begin(), datt.end(), R(0));
      linear_bwd(att[l].data(), P(p, WO, l, (size_t)C * C), dx.data(),
                 datt.data(), grad + g.off[WO] + (size_t)l * C * C,
                 grad + g.off[BO] + (size_t)l * C, M, C, C);
      attention_bwd(qkv[l].data(), datt.data(), dqkv.data(), B, T, C, g.H);
      std::fill(dh.begin(), dh.end(), R(0));
      linear_bwd(h1[l].data(), P(p, WQKV, l, (size_t)3 * C * C), dqkv.data(),
                 dh.data(), grad + g.off[WQKV] + (size_t)l * 3 * C * C,
                 grad + g.off[BQKV] + (size_t)l * 3 * C, M, C, 3 * C);
      layernorm_bwd(xin[l].data(), P(p, LN1G, l, C), m1[l].data(),
                    r1[l].data(), dh.data(), dx.data(),
                    grad + g.off[LN1G] + (size_t)l * C,
                    grad + g.off[LN1B] + (size_t)l * C, M, C);
    }
    // encoder: dwte[tok[m]] += dx0[m]; dwpe[t] += dx0[m], ascending m
    for (int m = 0; m < M; ++m) {
      const int t = m % T;
      R* gw = grad + g.off[WTE] + (size_t)tok[m] * C;
      R* gp = grad + g.off[WPE] + (size_t)t * C;
      for (int c = 0; c < C; ++c) {
        gw[c] += dx[(size_t)m * C + c];
        gp[c] += dx[(size_t)m * C + c];
      }
    }
  }
};

template <class R>
R grad_norm(const R* gr, size_t n) {
  R s = 0;
  for (size_t i = 0; i < n; ++i) s += gr[i] * gr[i];
  return std::sqrt(s);
}

// Returns the pre-clip norm; scales by max_norm / (norm + 1e-6) when
// norm > max_norm.
template <class R>
R clip(R* gr, size_t n, R max_norm) {
  const R nrm = grad_norm(gr, n);
  if (nrm > max_norm) {
    const R c = max_norm / (nrm + R(1e-6));
    for (size_t i = 0; i < n; ++i) gr[i] *= c;
  }
  return nrm;
}

template <class R>
void adamw(const Cfg& g, R* p, const R* gr, R* m, R* v, long t, R lr, R b1,
           R b2, R eps, R wd) {
  const R bc1 = R(1) - std::pow(b1, (R)t);
  const R bc2 = R(1) - std::pow(b2, (R)t);
  for (int tn = 0; tn < NT; ++tn) {
    const R w = is_decayed(tn) ? wd : R(0);
    for (size_t i = g.off[tn]; i < g.off[tn] + g.num[tn]; ++i) {
      m[i] = b1 * m[i] + (R(1) - b1) * gr[i];
      v[i] = b2 * v[i] + (R(1) - b2) * gr[i] * gr[i];
      const R mh = m[i] / bc1;
      const R vh = v[i] / bc2;
      p[i] -= lr * (mh / (std::sqrt(vh) + eps) + w * p[i]);
    }
  }
}

template <class R>
R forward_only(const Cfg& g, const R* p, const int* tok, const int* tgt, int B,
               int T, R* losses, R* logits) {
  Model<R> mod(g);
  const R loss = mod.forward(p, tok, tgt, B, T);
  const int M = B * T;
  if (losses && tgt) std::copy(mod.lossv.begin(), mod.lossv.end(), losses);
  if (logits) std::copy(mod.logits.begin(), mod.logits.begin() + (size_t)M * g.V, logits);
  return loss;
}

template <class R>
R forward_backward(const Cfg& g, const R* p, const int* tok, const int* tgt,
                   int B, int T, R loss_scale, R* grad, R* losses) {
  Model<R> mod(g);
  const R loss = mod.forward(p, tok, tgt, B, T);
  mod.backward(p, grad, loss_scale);
  if (losses) std::copy(mod.lossv.begin(), mod.lossv.end(), losses);
  return loss;
}

}  // namespace

// ------------------------------------------------------------------ C API --
extern "C" {

size_t orc_num_params(int L, int C, int V, int Vp, int Tmax) {
  return make_cfg(L, 1, C, V, Vp, Tmax).total;
}

// Offsets and sizes of the 16 tensors in the flat order; decayed flag.
int orc_tensor_slice(int L, int C, int V, int Vp, int Tmax, int i,
                     size_t* off, size_t* num, int* decayed) {
  if (i < 0 || i >= NT) return -1;
  const Cfg g = make_cfg(L, 1, C, V, Vp, Tmax);
  *off = g.off[i];
  *num = g.num[i];
  *decayed = is_decayed(i) ? 1 : 0;
  return 0;
}

double orc_std_normal(uint64_t seed, int tensor, uint64_t i) {
  return std_normal(sm_output(seed, (uint64_t)tensor + 1), i);
}

uint64_t orc_splitmix64(uint64_t seed, uint64_t n) { return sm_output(seed, n); }

#define ORC_DEFINE(R, SFX)                                                     \
  void orc_init_##SFX(int L, int H, int C, int V, int Vp, int Tmax,            \
                      uint64_t seed, R* p) {                                   \
    init_params<R>(make_cfg(L, H, C, V, Vp, Tmax), seed, p);                   \
  }                                                                            \
  R orc_forward_##SFX(int L, int H, int C, int V, int Vp, int Tmax,            \
                      const R* p, const int* tok, const int* tgt, int B,       \
                      int T, R* losses, R* logits) {                           \
    return forward_only<R>(make_cfg(L, H, C, V, Vp, Tmax), p, tok, tgt, B, T,  \
                           losses, logits);                                    \
  }                                                                            \
  R orc_forward_backward_##SFX(int L, int H, int C, int V, int Vp, int Tmax,   \
                               const R* p, const int* tok, const int* tgt,     \
                               int B, int T, R loss_scale, R* grad,            \
                               R* losses) {                                    \
    return forward_backward<R>(make_cfg(L, H, C, V, Vp, Tmax), p, tok, tgt, B, \
                               T, loss_scale, grad, losses);                   \
  }                                                                            \
  R orc_grad_norm_##SFX(const R* gr, size_t n) { return grad_norm<R>(gr, n); } \
  R orc_clip_##SFX(R* gr, size_t n, R max_norm) {                              \
    return clip<R>(gr, n, max_norm);                                           \
  }                                                                            \
  void orc_adamw_##SFX(int L, int C, int V, int Vp, int Tmax, R* p,            \
                       const R* gr, R* m, R* v, long t, R lr, R b1, R b2,      \
                       R eps, R wd) {                                          \
    adamw<R>(make_cfg(L, 1, C, V, Vp, Tmax), p, gr, m, v, t, lr, b1, b2, eps,  \
             wd);                                                              \
  }                                                                            \
  R orc_gelu_tanh_##SFX(R x) { return gelu_tanh<R>(x); }                       \
  R orc_gelu_tanh_grad_##SFX(R x) { return gelu_tanh_grad<R>(x); }             \
  R orc_gelu_erf_##SFX(R x) { return gelu_erf<R>(x); }                         \
  void orc_gelu_tanh_vec_##SFX(const R* x, R* y, size_t n, int grad) {         \
    for (size_t i = 0; i < n; ++i)                                             \
      y[i] = grad ? gelu_tanh_grad<R>(x[i]) : gelu_tanh<R>(x[i]);              \
  }                                                                            \
  void orc_layernorm_fwd_##SFX(const R* x, const R* g, const R* b, R* y,       \
                               R* mean, R* rstd, int M, int C) {               \
    layernorm_fwd<R>(x, g, b, y, mean, rstd, M, C);                            \
  }                                                                            \
  void orc_layernorm_bwd_##SFX(const R* x, const R* g, const R* mean,         \
                               const R* rstd, const R* dy, R* dx, R* dg, R* db, \
                               int M, int C) {                                 \
    layernorm_bwd<R>(x, g, mean, rstd, dy, dx, dg, db, M, C);                  \
  }                                                                            \
  void orc_softmax_xent_##SFX(const R* z, int M, int V, const int* tgt,        \
                              R scale, R* losses, R* dz) {                     \
    softmax_xent<R>(z, M, V, tgt, scale, losses, dz);                          \
  }                                                                            \
  int orc_sample_token_##SFX(const R* z, int V, R temperature, int top_k,     \
                             double u) {                                       \
    return sample_token<R>(z, V, temperature, top_k, u);                       \
  }                                                                            \
  void orc_attention_fwd_##SFX(const R* qkv, R* y, int B, int T, int C,        \
                               int H) {                                        \
    attention_fwd<R>(qkv, y, B, T, C, H);                                      \
  }                                                                            \
  void orc_attention_bwd_##SFX(const R* qkv, const R* dy, R* dqkv, int B,      \
                               int T, int C, int H) {                          \
    attention_bwd<R>(qkv, dy, dqkv, B, T, C, H);                               \
  }                                                                            \
  void orc_linear_fwd_##SFX(const R* x, const R* W, const R* b, R* y, int M,   \
                            int K, int N) {                                    \
    linear_fwd<R>(x, W, b, y, M, K, N);                                        \
  }

ORC_DEFINE(double, f64)
ORC_DEFINE(float, f32)

// Warmup-then-cosine schedule: lr(s) = max (s+1)/W for s < W; for
// W <= s <= S, min + 0.5 (1 + cos(pi (s-W)/(S-W))) (max - min); min after S.
double orc_lr(long step, double max_lr, double min_lr, long warmup,
              long max_steps) {
  if (step < warmup) return max_lr * (double)(step + 1) / (double)warmup;
  if (step > max_steps || max_steps <= warmup) return min_lr;
  const double ratio = (double)(step - warmup) / (double)(max_steps - warmup);
  const double coeff = 0.5 * (1.0 + std::cos(M_PI * ratio));
  return min_lr + coeff * (max_lr - min_lr);
}

int orc_openmp_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
