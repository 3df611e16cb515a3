// Token + position embedding (wte[tok] + wpe[t]) and its deterministic
// backward.
//
// Backward without floating-point atomics: the positions are stably sorted
// by token id (LSD radix sort, 8-bit digits, ranks from warp match masks so
// that equal ids keep ascending position order), each fixed chunk of 64
// sorted positions sums its runs of equal ids in order, and one block per
// distinct id adds its chunk partials in chunk order into dwte.  The
// summation order therefore depends only on the token sequence.

#include <algorithm>

#include "kernels.h"

namespace gpt2k {

namespace {

constexpr int kSortTile = 1024;
constexpr int kChunk = 64;

__global__ void encoder_fwd_kernel(act_t* __restrict__ x0, int* __restrict__ tok_saved,
                                   const int* __restrict__ tok, const act_t* __restrict__ wte,
                                   const act_t* __restrict__ wpe, int M, int T, int C, int V,
                                   int* err) {
  pdl_start();
  const int m = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (m >= M) return;
  const int lane = threadIdx.x & 31;
  int id = tok[m];
  if (id < 0 || id >= V) {
    if (lane == 0) atomicOr(err, ERR_TOKEN);
    id = 0;
  }
  if (lane == 0) tok_saved[m] = id;
  const act_t* we = wte + (size_t)id * C;
  const act_t* pe = wpe + (size_t)(m % T) * C;
  act_t* o = x0 + (size_t)m * C;
  for (int c = lane * 8; c < C; c += 256) {
    float a[8], b[8];
    load8(we + c, a);
    load8(pe + c, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] += b[i];
    store8(o + c, a);
  }
}

// dwpe[t, c] += sum over b (ascending) of dx0[b T + t, c]
__global__ void wpe_bwd_kernel(float* __restrict__ dwpe, const act_t* __restrict__ dx0, int B,
                               int T, int C) {
  pdl_start();
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)T * C) return;
  const int t = (int)(i / C), c = (int)(i % C);
  float s = 0.f;
  for (int b = 0; b < B; ++b) s += to_f(dx0[((size_t)b * T + t) * C + c]);
  dwpe[i] += s;
}

__global__ void iota_kernel(int* keys_out, int* vals_out, const int* keys_in, int M) {
  pdl_start();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < M) {
    keys_out[i] = keys_in[i];
    vals_out[i] = i;
  }
}

// hist[d * ntiles + tile] = number of keys in the tile whose digit is d
__global__ void radix_hist_kernel(int* __restrict__ hist, const int* __restrict__ keys, int M,
                                  int shift, int ntiles) {
  pdl_start();
  __shared__ int h[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int i = blockIdx.x * kSortTile + threadIdx.x;
  if (i < M) atomicAdd(&h[(keys[i] >> shift) & 255], 1);
  __syncthreads();
  for (int d = threadIdx.x; d < 256; d += blockDim.x) hist[d * ntiles + blockIdx.x] = h[d];
}

// In-place exclusive scan of n ints by one block of 1024 threads.
__global__ void exclusive_scan_kernel(int* data, int n) {
  pdl_start();
  __shared__ int part[1024];
  const int per = (n + 1023) / 1024;
  const int b = threadIdx.x * per;
  int s = 0;
  for (int i = 0; i < per; ++i)
    if (b + i < n) s += data[b + i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int run = threadIdx.x ? part[threadIdx.x - 1] : 0;
  for (int i = 0; i < per; ++i)
    if (b + i < n) {
      const int v = data[b + i];
      data[b + i] = run;
      run += v;
    }
}

// Stable scatter of one tile (one key per thread, in position order).
__global__ void __launch_bounds__(kSortTile)
    radix_scatter_kernel(int* __restrict__ keys_out, int* __restrict__ vals_out,
                         const int* __restrict__ keys_in, const int* __restrict__ vals_in,
                         const int* __restrict__ offsets, int M, int shift, int ntiles) {
  pdl_start();
  __shared__ int cnt[32][257];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 32 * 257; i += blockDim.x) (&cnt[0][0])[i] = 0;
  __syncthreads();
  const int i = blockIdx.x * kSortTile + threadIdx.x;
  const bool valid = i < M;
  const int key = valid ? keys_in[i] : 0;
  const int d = valid ? ((key >> shift) & 255) : 256;
  const unsigned peers = __match_any_sync(0xffffffffu, d);
  const unsigned lower = peers & ((1u << lane) - 1u);
  const int rank = __popc(lower);
  if (lower == 0) cnt[warp][d] = __popc(peers);  // lowest lane of each group
  __syncthreads();
  if (threadIdx.x < 256) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = cnt[w][threadIdx.x];
      cnt[w][threadIdx.x] = run;
      run += c;
    }
  }
  __syncthreads();
  if (valid) {
    const int pos = offsets[d * ntiles + blockIdx.x] + cnt[warp][d] + rank;
    keys_out[pos] = key;
    vals_out[pos] = vals_in[i];
  }
}

// For each chunk of kChunk sorted positions: the sum of each run of equal
// ids inside the chunk, in sorted order, stored at the run's first position.
__global__ void chunk_partial_kernel(float* __restrict__ partial, const act_t* __restrict__ dx0,
                                     const int* __restrict__ skeys, const int* __restrict__ svals,
                                     int M, int C) {
  pdl_start();
  __shared__ int k_s[kChunk], v_s[kChunk];
  const int base = blockIdx.x * kChunk;
  const int n = min(kChunk, M - base);
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    k_s[i] = skeys[base + i];
    v_s[i] = svals[base + i];
  }
  __syncthreads();
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 2;
  if (c >= C) return;
  float s0 = 0.f, s1 = 0.f;
  int start = 0;
  for (int i = 0; i < n; ++i) {
    if (i > 0 && k_s[i] != k_s[i - 1]) {
      float* o = partial + (size_t)(base + start) * C + c;
      o[0] = s0;
      o[1] = s1;
      s0 = s1 = 0.f;
      start = i;
    }
    const act_t* r = dx0 + (size_t)v_s[i] * C + c;
    s0 += to_f(r[0]);
    s1 += to_f(r[1]);
  }
  float* o = partial + (size_t)(base + start) * C + c;
  o[0] = s0;
  o[1] = s1;
}

// One block per sorted position; blocks at the start of a run of equal ids
// add the run's chunk partials (in chunk order) into dwte[id].  VEC: four
// columns per thread as float4 (C % 4 == 0 and 16-byte aligned rows), so a
// block issues its whole row at once.
template <bool VEC>
__global__ void segment_sum_kernel(float* __restrict__ dwte, const float* __restrict__ partial,
                                   const int* __restrict__ skeys, int M, int C) {
  pdl_start();
  const int s = blockIdx.x;
  const int key = skeys[s];
  if (s > 0 && skeys[s - 1] == key) return;
  const int j0 = (s / kChunk + 1) * kChunk;  // the first position of the next chunk
  if (VEC) {
    const int C4 = C / 4;
    for (int c = threadIdx.x; c < C4; c += blockDim.x) {
      float4 acc = reinterpret_cast<const float4*>(partial + (size_t)s * C)[c];
      for (int j = j0; j < M && skeys[j] == key; j += kChunk) {
        const float4 p = reinterpret_cast<const float4*>(partial + (size_t)j * C)[c];
        acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
      }
      float4* d = reinterpret_cast<float4*>(dwte + (size_t)key * C) + c;
      float4 o = *d;
      o.x += acc.x; o.y += acc.y; o.z += acc.z; o.w += acc.w;
      *d = o;
    }
  } else {
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      float acc = partial[(size_t)s * C + c];
      for (int j = j0; j < M && skeys[j] == key; j += kChunk) acc += partial[(size_t)j * C + c];
      dwte[(size_t)key * C + c] += acc;
    }
  }
}

}  // namespace

void encoder_fwd(act_t* x0, int* tok_saved, const int* tok, const act_t* wte, const act_t* wpe,
                 int B, int T, int C, int V, int* err, cudaStream_t s) {
  const int M = B * T;
  const int warps = 8;
  launch_kernel(encoder_fwd_kernel, (M + warps - 1) / warps, warps * 32, 0, s, x0, tok_saved, tok, wte, wpe,
                                                                      M, T, C, V, err);
  note_launch();
}

static size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

size_t encoder_scratch_bytes(int M, int C) {
  const int ntiles = (M + kSortTile - 1) / kSortTile;
  return 4 * align256((size_t)M * 4) + align256((size_t)256 * ntiles * 4) +
         align256((size_t)M * C * 4);
}

void encoder_scratch_carve(EncoderScratch* es, void* base, int M, int C) {
  const int ntiles = (M + kSortTile - 1) / kSortTile;
  char* p = static_cast<char*>(base);
  es->keys[0] = reinterpret_cast<int*>(p); p += align256((size_t)M * 4);
  es->keys[1] = reinterpret_cast<int*>(p); p += align256((size_t)M * 4);
  es->vals[0] = reinterpret_cast<int*>(p); p += align256((size_t)M * 4);
  es->vals[1] = reinterpret_cast<int*>(p); p += align256((size_t)M * 4);
  es->hist = reinterpret_cast<int*>(p); p += align256((size_t)256 * ntiles * 4);
  es->partial = reinterpret_cast<float*>(p);
}

void encoder_bwd(float* dwte, float* dwpe, const act_t* dx0, const int* tok_saved, int B, int T,
                 int C, int Vp, const EncoderScratch& es, cudaStream_t s) {
  const int M = B * T;
  launch_kernel(wpe_bwd_kernel, (int)(((size_t)T * C + 255) / 256), 256, 0, s, dwpe, dx0, B, T, C);
  // stable sort of (token, position) by token
  const int ntiles = (M + kSortTile - 1) / kSortTile;
  launch_kernel(iota_kernel, (M + 255) / 256, 256, 0, s, es.keys[0], es.vals[0], tok_saved, M);
  int bits = 0;
  while ((1 << bits) < Vp) ++bits;
  int cur = 0;
  for (int shift = 0; shift < bits; shift += 8) {
    launch_kernel(radix_hist_kernel, ntiles, kSortTile, 0, s, es.hist, es.keys[cur], M, shift, ntiles);
    launch_kernel(exclusive_scan_kernel, 1, 1024, 0, s, es.hist, 256 * ntiles);
    launch_kernel(radix_scatter_kernel, ntiles, kSortTile, 0, s, es.keys[cur ^ 1], es.vals[cur ^ 1],
                                                      es.keys[cur], es.vals[cur], es.hist, M,
                                                      shift, ntiles);
    cur ^= 1;
    note_launch(3);
  }
  const int nchunks = (M + kChunk - 1) / kChunk;
  dim3 g1(nchunks, (C / 2 + 127) / 128);
  launch_kernel(chunk_partial_kernel, g1, 128, 0, s, es.partial, dx0, es.keys[cur], es.vals[cur], M, C);
  if (C % 4 == 0 && !(reinterpret_cast<uintptr_t>(dwte) & 15) &&
      !(reinterpret_cast<uintptr_t>(es.partial) & 15)) {
    const int threads = std::min(256, (C / 4 + 31) / 32 * 32);
    launch_kernel(segment_sum_kernel<true>, M, threads, 0, s, dwte, es.partial, es.keys[cur], M, C);
  } else {
    launch_kernel(segment_sum_kernel<false>, M, 128, 0, s, dwte, es.partial, es.keys[cur], M, C);
  }
  note_launch(4);
}

}  // namespace gpt2k
