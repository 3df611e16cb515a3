// Causal flash-attention forward on the sm_100a tensor cores (head dim 64).
//
// One CTA per (query tile of 128 rows, batch, head), heaviest tiles first;
// 10 warps:
//   warp 0     TMA: the Q tile once, then K/V tiles of 128 keys into a
//              3-stage shared-memory ring (128-byte swizzle, zero fill past
//              the sequence);
//   warp 1     TMEM owner and MMA issuer: S_j = Q K_j^T (M=128, N=128,
//              K=64) into one of two TMEM buffers, and O_j = P_j V_j
//              (M=128, N=64, K=128; V read MN-major straight from its tile)
//              into one of two more;
//   warps 2-9  softmax: two threads per query row (warps w and w+4 share a
//              TMEM lane quarter), each owning 64 of the 128 key columns and
//              32 of the 64 output dimensions.  They read S_j from TMEM,
//              agree on the running row max through shared memory, write
//              P_j = 2^(S_j log2e/sqrt(d) - m) as bf16 into a swizzled tile
//              (the next MMA's A operand), and fold O_{j-1} into fp32 row
//              accumulators held in registers with the pending rescale
//              factor.  S_{j+1} and O_{j-1} are computed by the tensor core
//              while tile j's softmax runs.
// T x T is never materialised.  The output row is normalised by the
// running sum; the natural-log log-sum-exp of each row is stored for the
// backward pass.  Every wait is bounded (error word ERR_TIMEOUT).

#include <cuda.h>
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <tuple>

#include "attention_tc.cuh"

namespace gpt2k {

namespace {

using namespace tc;
using attn::kHD;
using attn::kBox;

constexpr int kTileQ = attn::kTile;
constexpr int kTileK = attn::kTile;
constexpr int kKVStages = 3;
constexpr int kSoftmaxThreads = attn::kComputeThreads;
constexpr int kThreadsAttn = 64 + kSoftmaxThreads;
constexpr uint32_t kTmemCols = 512;  // S: 2 x 128, O: 2 x 64
constexpr int kAux = 4096;           // barriers + cross-thread row scratch

constexpr size_t attn_smem_bytes() {
  // Q, K ring, V ring, P double buffer (two 64-key boxes each), aux
  return 1024 + kBox + 2 * (size_t)kKVStages * kBox + 2 * 2 * (size_t)kBox + kAux;
}

__device__ __forceinline__ void sm_bar() { named_bar<1, kSoftmaxThreads>(); }
__device__ __forceinline__ bool sm_bar_and(bool pred) {
  return named_bar_and<1, kSoftmaxThreads>(pred);
}

__global__ void __launch_bounds__(kThreadsAttn, 1)
    flash_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQKV, __nv_bfloat16* __restrict__ att,
                        float* __restrict__ lse, int T, int C, int H, float sl2, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kBox;                      // [kKVStages][kBox]
  uint8_t* sV = sK + kKVStages * kBox;          // [kKVStages][kBox]
  uint8_t* sP = sV + kKVStages * kBox;          // [2][2 boxes]
  uint8_t* aux = sP + 4 * kBox;
  uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
  const uint32_t q_full = smem_u32(bars + 0);
  const uint32_t kv_full0 = smem_u32(bars + 1);                  // [3]
  const uint32_t kv_empty0 = smem_u32(bars + 1 + kKVStages);     // [3]
  const uint32_t s_full0 = smem_u32(bars + 1 + 2 * kKVStages);   // [2]
  const uint32_t s_empty0 = s_full0 + 16;                        // [2]
  const uint32_t p_full0 = s_full0 + 32;                         // [2]
  const uint32_t p_empty0 = s_full0 + 48;                        // [2]
  const uint32_t o_full0 = s_full0 + 64;                         // [2]
  const uint32_t o_empty0 = s_full0 + 80;                        // [2]
  const uint32_t drain = s_full0 + 96;                           // abort path only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1 + 2 * kKVStages + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red_max = reinterpret_cast<float*>(aux + 512);   // [2 parity][2 halves][128 rows]
  float* red_l = red_max + 2 * 2 * kTileQ;                // [2 halves][128 rows]

  const int qb = gridDim.x - 1 - blockIdx.x;  // heaviest query tiles first
  const int b = blockIdx.y / H, h = blockIdx.y % H;
  const int q0 = qb * kTileQ;
  const int nkv = qb + 1;  // causal: key tiles 0 .. qb
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full0 + 8 * i, 1);
      mbar_init(s_empty0 + 8 * i, kSoftmaxThreads);
      mbar_init(p_full0 + 8 * i, kSoftmaxThreads);
      mbar_init(p_empty0 + 8 * i, 1);
      mbar_init(o_full0 + 8 * i, 1);
      mbar_init(o_empty0 + 8 * i, kSoftmaxThreads);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA --
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQKV)) : "memory");
      mbar_expect_tx(q_full, kBox);
      tma_load_3d(smem_u32(sQ), &tmQKV, q_full, h * kHD, q0, b);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;
      for (int j = 0; j < nkv; ++j) {
        if (!mbar_wait(kv_empty0 + 8 * stage, phase ^ 1u, abort_flag, err)) break;
        const uint32_t fb = kv_full0 + 8 * stage;
        mbar_expect_tx(fb, 2 * kBox);
        tma_load_3d(smem_u32(sK + stage * kBox), &tmQKV, fb, C + h * kHD, j * kTileK, b);
        tma_load_3d(smem_u32(sV + stage * kBox), &tmQKV, fb, 2 * C + h * kHD, j * kTileK, b);
        issued |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == kKVStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // every copy issued lands before the shared memory is released (the
      // MMA warp has already waited for all of them unless it gave up)
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(q_full, 0) && global_ns() - t0 < kWaitLimitNs) {
      }
      for (int s2 = 0; s2 < kKVStages; ++s2) {
        if (!(issued & (1u << s2))) continue;
        while (!mbar_try_wait(kv_full0 + 8 * s2, (last_parity >> s2) & 1u) &&
               global_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA --
      constexpr uint32_t idS = attn::idesc(kTileK, false);
      constexpr uint32_t idO = attn::idesc(kHD, true);
      bool ok = mbar_wait(q_full, 0, abort_flag, err);
      tc_fence_after();
      const uint32_t q_base = smem_u32(sQ);
      // S_j: stage j % 3, S buffer j % 2
      auto issue_s = [&](int j) -> bool {
        const int st = j % kKVStages, sb = j & 1;
        if (!mbar_wait(kv_full0 + 8 * st, (uint32_t)(j / kKVStages) & 1u, abort_flag, err)) return false;
        if (!mbar_wait(s_empty0 + 8 * sb, ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(sK + st * kBox);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)
          tc_mma(tmem + (uint32_t)(sb * kTileK), desc_kmajor(q_base, k), desc_kmajor(k_base, k), idS,
                 k > 0 ? 1u : 0u);
        tc_commit(s_full0 + 8 * sb);
        return true;
      };
      // O_j = P_j V_j: P buffer j % 2, V stage j % 3, O buffer j % 2
      auto issue_o = [&](int j) -> bool {
        const int st = j % kKVStages, pb = j & 1;
        if (!mbar_wait(p_full0 + 8 * pb, (uint32_t)(j >> 1) & 1u, abort_flag, err)) return false;
        if (!mbar_wait(o_empty0 + 8 * pb, ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t p_base = smem_u32(sP + pb * 2 * kBox);
        const uint32_t v_base = smem_u32(sV + st * kBox);
#pragma unroll
        for (int k = 0; k < kTileK / 16; ++k)
          tc_mma(tmem + 2u * kTileK + (uint32_t)(pb * kHD),
                 desc_kmajor(p_base + (uint32_t)((k >> 2) * kBox), k & 3), desc_mnmajor(v_base, k), idO,
                 k > 0 ? 1u : 0u);
        tc_commit(o_full0 + 8 * pb);
        tc_commit(p_empty0 + 8 * pb);
        tc_commit(kv_empty0 + 8 * st);  // K_j and V_j are no longer read
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 1; j <= nkv && ok; ++j) {
        if (j < nkv) ok = issue_s(j);
        if (ok) ok = issue_o(j - 1);
      }
      if (!ok) {  // let issued MMAs finish before TMEM is released
        tc_commit(drain);
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(drain, 0) && global_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // -------------------------------------------------------- softmax --
    const int qw = warp & 3;           // TMEM lane quarter
    const int half = (warp - 2) >> 2;  // 0: key columns 0-63 / dims 0-31; 1: 64-127 / 32-63
    const int r = qw * 32 + lane;
    const int qi = q0 + r;  // query index in the sequence
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    float o[kHD / 2];
#pragma unroll
    for (int i = 0; i < kHD / 2; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f, a_pend = 1.f;
    bool ok = true;
    for (int j = 0; j <= nkv && ok; ++j) {
      float a_new = 1.f;
      if (j < nkv) {
        const int sb = j & 1;
        ok = sm_bar_and(mbar_wait(s_full0 + 8 * sb, (uint32_t)(j >> 1) & 1u, abort_flag, err));
        if (!ok) break;
        tc_fence_after();
        float s[64];
        {
          uint32_t rr[64];
          const uint32_t col = (uint32_t)(sb * kTileK + 64 * half);
          tc_ld32(lane_base + col, rr);
          tc_ld32(lane_base + col + 32, rr + 32);
          tc_wait_ld();
          tc_fence_before();
          mbar_arrive(s_empty0 + 8 * sb);
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(rr[c]);
        }
        const int key0 = j * kTileK + 64 * half;
        if (j == qb) {  // diagonal tile: keys after the query (and past T) are masked
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (key0 + c > qi || key0 + c >= T) s[c] = -INFINITY;
        }
        // row max over this thread's 64 columns (8 independent chains),
        // then with the partner thread's half through shared memory
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
        for (int c = 8; c < 64; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
        float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        float* rm = red_max + (j & 1) * 2 * kTileQ;
        rm[half * kTileQ + r] = mx;
        sm_bar();
        mx = fmaxf(mx, rm[(half ^ 1) * kTileQ + r]) * sl2;  // scaled (log2 units)
        const float mnew = fmaxf(m, mx);
        a_new = (mnew == -INFINITY) ? 1.f : fast_exp2(m - mnew);
        const float mref = (mnew == -INFINITY) ? 0.f : mnew;
        float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          s[c] = fast_exp2(fmaf(s[c], sl2, -mref));
          sum8[c & 7] += s[c];
        }
        l = l * a_new + (((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) +
                         ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7])));
        m = mnew;
        // P_j (this half's 64 keys = one 128-byte-swizzled box)
        const int pb = j & 1;
        ok = sm_bar_and(mbar_wait(p_empty0 + 8 * pb, ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag, err));
        if (!ok) break;
        uint8_t* pt = sP + (pb * 2 + half) * kBox;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8)
          store8(reinterpret_cast<__nv_bfloat16*>(pt + swz(r, c8)), s + 8 * c8);
        fence_async_smem();
        mbar_arrive(p_full0 + 8 * pb);
      }
      if (j >= 1) {  // fold O_{j-1} (computed with the max of tile j-1)
        const int ob = (j - 1) & 1;
        ok = sm_bar_and(mbar_wait(o_full0 + 8 * ob, (uint32_t)((j - 1) >> 1) & 1u, abort_flag, err));
        if (!ok) break;
        tc_fence_after();
        uint32_t rr[32];
        tc_ld32(lane_base + 2u * kTileK + (uint32_t)(ob * kHD + 32 * half), rr);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(o_empty0 + 8 * ob);
#pragma unroll
        for (int i = 0; i < kHD / 2; ++i) o[i] = o[i] * a_pend + __uint_as_float(rr[i]);
      }
      a_pend = a_new;
    }
    // row sum = the two halves' partial sums
    red_l[half * kTileQ + r] = l;
    sm_bar();
    l += red_l[(half ^ 1) * kTileQ + r];
    if (ok && qi < T) {
      const float inv = 1.f / l;
      __nv_bfloat16* dst = att + ((size_t)b * T + qi) * C + (size_t)h * kHD + 32 * half;
#pragma unroll
      for (int i = 0; i < kHD / 2; i += 8) {
        float t[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) t[k] = o[i + k] * inv;
        store8(dst + i, t);
      }
      if (half == 0) lse[((size_t)b * H + h) * T + qi] = (m + log2f(l)) * 0.6931471805599453f;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

}  // namespace

namespace attn {

cudaError_t seq_map(CUtensorMap* tm, const void* base, int B, int T, int cols) {
  using Key = std::tuple<const void*, int, int, int>;
  static std::map<Key, CUtensorMap> cache;
  static std::mutex mu;
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  const Key key{base, B, T, cols};
  std::lock_guard<std::mutex> g(mu);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *tm = it->second;
    return cudaSuccess;
  }
  if (!enc) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return cudaErrorNotSupported;
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)T * cols * 2};
  cuuint32_t box[3] = {64u, 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  if (enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (cache.size() > 1024) cache.clear();
  cache[key] = *tm;
  return cudaSuccess;
}

}  // namespace attn

bool attention_fwd_tc_supported(int C, int H) {
  return C / H == kHD && (C * 2) % 16 == 0;
}

cudaError_t attention_fwd_tc(act_t* att, float* lse, const act_t* qkv, int B, int T, int C, int H,
                             int* err, cudaStream_t s) {
  if (!attention_fwd_tc_supported(C, H) || (reinterpret_cast<uintptr_t>(qkv) & 15))
    return cudaErrorInvalidValue;
  CUtensorMap tm;
  cudaError_t e = attn::seq_map(&tm, qkv, B, T, 3 * C);
  if (e != cudaSuccess) return e;
  constexpr size_t smem = attn_smem_bytes();
  static_assert(smem <= 232448, "shared memory budget");
  static bool attr = false;
  if (!attr) {
    e = cudaFuncSetAttribute(flash_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const float sl2 = 1.4426950408889634f / sqrtf((float)kHD);
  dim3 grid((T + kTileQ - 1) / kTileQ, B * H);
  flash_fwd_tc_kernel<<<grid, kThreadsAttn, smem, s>>>(tm, att, lse, T, C, H, sl2, err);
  note_launch();
  return cudaGetLastError();
}

}  // namespace gpt2k
