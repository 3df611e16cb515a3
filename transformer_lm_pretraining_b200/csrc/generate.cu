// Kernels of autoregressive generation with a key/value cache: the
// embedding of one position per sequence, single-query causal attention over
// the cached keys and values, and the next-token sampler.

#include <climits>

#include "kernels.h"

namespace gpt2k {

namespace {

constexpr int kSampleThreads = 1024;

// The position a kernel works at: p, plus *p_dev when p_dev is given (the
// position counter of a decode step replayed from a CUDA graph).
__device__ __forceinline__ int at_pos(int p, const int* p_dev) { return p_dev ? p + *p_dev : p; }

// x[b] = wte[tok[b * ld_tok + p]] + wpe[p]; ids outside [0, V) read as 0 and
// set ERR_TOKEN.
__global__ void decode_embed_kernel(act_t* __restrict__ x, const int* __restrict__ tok, int ld_tok,
                                    int p0, const int* __restrict__ p_dev,
                                    const act_t* __restrict__ wte, const act_t* __restrict__ wpe,
                                    int C, int V, int* err) {
  pdl_start();
  const int b = blockIdx.x;
  const int p = at_pos(p0, p_dev);
  int t = tok[(size_t)b * ld_tok + p];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) atomicOr(err, ERR_TOKEN);
    t = 0;
  }
  for (int c = threadIdx.x * 8; c < C; c += blockDim.x * 8) {
    float a[8], w[8];
    load8(wte + (size_t)t * C + c, a);
    load8(wpe + (size_t)p * C + c, w);
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] += w[i];
    store8(x + (size_t)b * C + c, a);
  }
}

// One block of kDecodeThreads per (head, sequence): the query q[b, head]
// against the n cached keys of that sequence: scores in shared memory,
// softmax in fp32, then the value average (the threads split the keys into
// kDecodeThreads / hd parts per output dimension, added in part order).
// kv rows: [b][Ttot][2C] = [k | v].
constexpr int kDecodeThreads = 256;
__global__ void __launch_bounds__(kDecodeThreads)
    decode_attention_kernel(act_t* __restrict__ att, const act_t* __restrict__ q,
                            const act_t* __restrict__ kv, int Ttot, int n0,
                            const int* __restrict__ p_dev, int C, int H, float scale) {
  pdl_start();
  const int n = at_pos(n0, p_dev);
  extern __shared__ float sc[];  // [n] scores, then [128 / hd][hd] partial outputs
  __shared__ float red[kDecodeThreads / 32], qv[256];
  const int h = blockIdx.x, b = blockIdx.y, hd = C / H;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int d = tid; d < hd; d += blockDim.x) qv[d] = to_f(q[(size_t)b * C + h * hd + d]);
  __syncthreads();
  const act_t* kb = kv + (size_t)b * Ttot * 2 * C + (size_t)h * hd;
  float mx = -INFINITY;
  for (int k = tid; k < n; k += blockDim.x) {
    const act_t* kr = kb + (size_t)k * 2 * C;
    float s = 0.f;
    for (int d = 0; d < hd; d += 8) {
      float kk[8];
      load8(kr + d, kk);
#pragma unroll
      for (int i = 0; i < 8; ++i) s = fmaf(qv[d + i], kk[i], s);
    }
    s *= scale;
    sc[k] = s;
    mx = fmaxf(mx, s);
  }
  mx = warp_max(mx);
  if (lane == 0) red[w] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int i = 1; i < kDecodeThreads / 32; ++i) mx = fmaxf(mx, red[i]);
  __syncthreads();
  float sum = 0.f;
  for (int k = tid; k < n; k += blockDim.x) {
    const float e = __expf(sc[k] - mx);
    sc[k] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  if (lane == 0) red[w] = sum;
  __syncthreads();
  sum = red[0];
#pragma unroll
  for (int i = 1; i < kDecodeThreads / 32; ++i) sum += red[i];
  // output dimension d = tid % hd, key part = tid / hd
  float* part = sc + n;
  const int d = tid % hd, half = tid / hd, halves = blockDim.x / hd;
  if (half < halves) {
    float o = 0.f;
    for (int k = half; k < n; k += halves)
      o = fmaf(sc[k], to_f(kb[(size_t)k * 2 * C + C + d]), o);
    part[half * hd + d] = o;
  }
  __syncthreads();
  if (tid < hd) {
    float o = 0.f;
    for (int hh = 0; hh < halves; ++hh) o += part[hh * hd + tid];
    att[(size_t)b * C + h * hd + tid] = from_f<act_t>(o / sum);
  }
}

// Order-preserving map of a float to an unsigned integer.
__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float block_max_f(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_max(v);
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kSampleThreads / 32; ++i) r = fmaxf(r, red[i]);
  __syncthreads();
  return r;
}
__device__ __forceinline__ float block_sum_f(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_sum(v);
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kSampleThreads / 32; ++i) r += red[i];
  __syncthreads();
  return r;
}
__device__ __forceinline__ int block_min_i(int v, int* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) red[w] = v;
  __syncthreads();
  int r = red[0];
  for (int i = 1; i < kSampleThreads / 32; ++i) r = min(r, red[i]);
  __syncthreads();
  return r;
}

// One block per sequence b: the next token from the row of V logits at
// logits + b * ld_logits, written to tok[b * ld_tok + p_out].  The row is
// staged in shared memory (coalesced); thread t owns the contiguous run of
// columns [t c, t c + c), c = ceil(V / kSampleThreads).  Temperature 0: the
// argmax (lowest index among equal maxima).  Otherwise the softmax of z /
// temperature over the top_k largest logits (ties at the k-th value kept):
// the k-th largest order-preserving key is found by a radix select, a byte at
// a time from the top (integer counts in shared memory), then the runs' sums
// of exp((z - max) / T) are scanned in thread order and the run where the
// cumulative mass first exceeds u * total is walked, u = SplitMix64(seed,
// p_out * 65536 + b) (top 53 bits).  logits_out (may be null) receives the
// row as fp32.  Dynamic shared memory: V activations.
__global__ void __launch_bounds__(kSampleThreads, 1)
    sample_kernel(int* __restrict__ tok, int ld_tok, int p_out0, const int* __restrict__ p_dev,
                  const act_t* __restrict__ logits, long ld_logits, int V, float temperature,
                  int top_k, uint64_t seed, float* __restrict__ logits_out, int out_p0) {
  pdl_start();
  extern __shared__ __align__(16) uint8_t sample_smem[];
  act_t* zs = reinterpret_cast<act_t*>(sample_smem);
  __shared__ float redf[kSampleThreads / 32];
  __shared__ int redi[kSampleThreads / 32];
  __shared__ float scan[kSampleThreads];
  __shared__ int hist[256];
  __shared__ uint32_t sel[2];  // the selected key prefix and the count still to take
  const int p_out = at_pos(p_out0, p_dev);
  if (logits_out) logits_out += (size_t)(p_out - out_p0) * gridDim.x * V;
  const int b = blockIdx.x, tid = threadIdx.x;
  const act_t* z = logits + (size_t)b * ld_logits;
  float mx = -INFINITY;
  for (int v = tid; v < V; v += kSampleThreads) {
    const act_t x = z[v];
    zs[v] = x;
    mx = fmaxf(mx, to_f(x));
    if (logits_out) logits_out[(size_t)b * V + v] = to_f(x);
  }
  mx = block_max_f(mx, redf);  // (its barrier also publishes zs)
  const int chunk = (V + kSampleThreads - 1) / kSampleThreads;
  const int v0 = min(V, tid * chunk), v1 = min(V, v0 + chunk);
  int chosen;
  if (temperature <= 0.f) {
    int first = INT_MAX;
    for (int v = v1 - 1; v >= v0; --v)
      if (to_f(zs[v]) == mx) first = v;
    chosen = block_min_i(first, redi);
  } else {
    // keep z >= the k-th largest value: radix select of the k-th largest key
    uint32_t thr = 0;
    if (top_k > 0 && top_k < V) {
      if (tid == 0) {
        sel[0] = 0u;
        sel[1] = (uint32_t)top_k;
      }
      for (int shift = 24; shift >= 0; shift -= 8) {
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        const uint32_t prefix = sel[0];
        const uint32_t hi_mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
        for (int v = v0; v < v1; ++v) {
          const uint32_t key = ord_key(to_f(zs[v]));
          if ((key & hi_mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
        }
        __syncthreads();
        if (tid == 0) {  // the bin holding the k-th largest, from the top
          uint32_t need = sel[1];
          int bin = 255;
          for (; bin > 0; --bin) {
            const uint32_t c = (uint32_t)hist[bin];
            if (c >= need) break;
            need -= c;
          }
          sel[0] = prefix | ((uint32_t)bin << shift);
          sel[1] = need;
        }
        __syncthreads();
      }
      thr = sel[0];
    }
    const float inv_t = 1.0f / temperature;
    float s = 0.f;
    for (int v = v0; v < v1; ++v) {
      const float zv = to_f(zs[v]);
      if (ord_key(zv) >= thr) s += __expf((zv - mx) * inv_t);
    }
    // exclusive scan of the runs' sums in thread order
    scan[tid] = s;
    __syncthreads();
    if (tid == 0) {
      float acc = 0.f;
      for (int i = 0; i < kSampleThreads; ++i) {
        const float x = scan[i];
        scan[i] = acc;
        acc += x;
      }
      redf[0] = acc;
    }
    __syncthreads();
    const float total = redf[0];
    const double u = (double)(sm64_out(seed, (uint64_t)p_out * 65536u + (uint64_t)b) >> 11) *
                     1.1102230246251565e-16;  // 2^-53
    const float target = (float)u * total;
    int found = INT_MAX, last = -1;
    float cum = scan[tid];
    for (int v = v0; v < v1; ++v) {
      const float zv = to_f(zs[v]);
      if (ord_key(zv) < thr) continue;
      cum += __expf((zv - mx) * inv_t);
      last = v;
      if (cum > target && found == INT_MAX) found = v;
    }
    chosen = block_min_i(found, redi);
    if (chosen == INT_MAX) chosen = -block_min_i(-last, redi);  // rounding: the last kept token
  }
  if (tid == 0) tok[(size_t)b * ld_tok + p_out] = chosen;
}

// cache[b][p] = kvnew[b] (2C values per row; cache rows [b][Ttot][2C])
__global__ void kv_append_kernel(act_t* __restrict__ cache, const act_t* __restrict__ kvnew,
                                 const int* __restrict__ p_dev, int p0, int Ttot, int C2) {
  pdl_start();
  const int b = blockIdx.x, p = at_pos(p0, p_dev);
  for (int c = threadIdx.x; c < C2; c += blockDim.x)
    cache[((size_t)b * Ttot + p) * C2 + c] = kvnew[(size_t)b * C2 + c];
}

__global__ void pos_advance_kernel(int* p_dev) {
  pdl_start();
  if (threadIdx.x == 0) *p_dev += 1;
}

}  // namespace

void decode_embed(act_t* x, const int* tok, int ld_tok, int p, const int* p_dev, const act_t* wte,
                  const act_t* wpe, int B, int C, int V, int* err, cudaStream_t s) {
  launch_kernel(decode_embed_kernel, B, 128, 0, s, x, tok, ld_tok, p, p_dev, wte, wpe, C, V, err);
  note_launch();
}

void decode_attention(act_t* att, const act_t* q, const act_t* kv, int Ttot, int n,
                      const int* p_dev, int B, int C, int H, cudaStream_t s) {
  const int hd = C / H;  // <= 128 (checked by the caller)
  const size_t smem = ((size_t)(p_dev ? Ttot : n) + kDecodeThreads) * sizeof(float);
  launch_kernel(decode_attention_kernel, dim3(H, B), kDecodeThreads, smem, s, att, q, kv, Ttot, n,
                p_dev, C, H,
                1.0f / sqrtf((float)hd));
  note_launch();
}

void sample_tokens(int* tok, int ld_tok, int p_out, const int* p_dev, const act_t* logits,
                   long ld_logits, int B, int V, float temperature, int top_k, uint64_t seed,
                   float* logits_out, int out_p0, cudaStream_t s) {
  const size_t smem = (size_t)V * sizeof(act_t);
  static size_t smem_set = 0;
  if (smem > 48 * 1024 && smem > smem_set) {
    cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    smem_set = smem;
  }
  launch_kernel(sample_kernel, B, kSampleThreads, smem, s, tok, ld_tok, p_out, p_dev, logits,
                ld_logits, V, temperature, top_k, seed, logits_out, out_p0);
  note_launch();
}

void kv_append(act_t* cache, const act_t* kvnew, int p, const int* p_dev, int Ttot, int B, int C,
               cudaStream_t s) {
  launch_kernel(kv_append_kernel, B, 128, 0, s, cache, kvnew, p_dev, p, Ttot, 2 * C);
  note_launch();
}

void pos_advance(int* p_dev, cudaStream_t s) {
  launch_kernel(pos_advance_kernel, 1, 32, 0, s, p_dev);
  note_launch();
}

}  // namespace gpt2k
