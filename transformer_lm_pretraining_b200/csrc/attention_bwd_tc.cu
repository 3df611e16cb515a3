// Causal flash-attention backward on the sm_100a tensor cores (head dim 64),
// deterministic: no atomics, each gradient tile is owned by one CTA.
//
// Given the forward's log-sum-exp L (natural log) and D = rowsum(dO * O):
//   P = exp(Q K^T / sqrt(d) - L),  dP = dO V^T,  dS = P * (dP - D)
//   dV = P^T dO,  dK = dS^T Q / sqrt(d),  dQ = dS K / sqrt(d)
//
// Two kernels, both 10 warps (TMA, MMA, 8 compute warps = two threads per
// 128-row tile row, each owning 64 of the 128 columns):
//   dK/dV: one CTA per 128-key tile; streams the query tiles i >= j.  The
//          tensor core computes S^T = K Q^T and dP^T = V dO^T into TMEM;
//          the compute warps turn them into P^T and dS^T (bf16, swizzled
//          shared-memory tiles); the tensor core then accumulates
//          dV += P^T dO and dK += dS^T Q in TMEM (dO and Q read MN-major
//          straight from their tiles).
//   dQ:    one CTA per 128-query tile; streams the key tiles j <= i:
//          S = Q K^T and dP = dO V^T into TMEM, dS into shared memory,
//          dQ += dS K in TMEM (K read MN-major).
// Every wait is bounded (error word ERR_TIMEOUT).

#include "attention_tc.cuh"

namespace gpt2k {

namespace {

using namespace tc;
using attn::kBox;
using attn::kHD;
using attn::kTile;

constexpr int kCT = attn::kComputeThreads;
constexpr int kThreadsBwd = 64 + kCT;
constexpr uint32_t kTmemCols = 512;
constexpr int kAux = 1024;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ bool cbar_and(bool p) { return named_bar_and<1, kCT>(p); }

__device__ __forceinline__ void tmem_alloc(uint32_t* slot) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(kTmemCols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base),
               "r"(kTmemCols));
}

// Bounded wait for copies issued to `bar` (latest fill parity `par`).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t par, uint64_t t0) {
  while (!mbar_try_wait(bar, par) && global_ns() - t0 < kWaitLimitNs) {
  }
}

// ------------------------------------------------------------------ dK/dV --
constexpr int kQStages = 2;
constexpr size_t dkdv_smem_bytes() {
  // K, V, [Q, dO] x stages, P^T and dS^T tiles (two boxes each), per-column
  // L and D of two query tiles, aux
  return 1024 + 2 * (size_t)kBox + 2 * (size_t)kQStages * kBox + 4 * (size_t)kBox +
         4 * kTile * sizeof(float) + kAux;
}

__global__ void __launch_bounds__(kThreadsBwd, 1)
    flash_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                             const __grid_constant__ CUtensorMap tmDO, const float* __restrict__ lse,
                             const float* __restrict__ dsum, __nv_bfloat16* __restrict__ dqkv, int T,
                             int C, int H, float sl2, float scale, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + kBox;
  uint8_t* sQ = sV + kBox;                // [kQStages]
  uint8_t* sDO = sQ + kQStages * kBox;    // [kQStages]
  uint8_t* sPT = sDO + kQStages * kBox;   // 2 boxes (query columns 0-63, 64-127)
  uint8_t* sDST = sPT + 2 * kBox;         // 2 boxes
  float* col_lse = reinterpret_cast<float*>(sDST + 2 * kBox);  // [2 tiles][L 128, D 128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(col_lse + 4 * kTile);
  const uint32_t kv_full = smem_u32(bars + 0);
  const uint32_t qd_full0 = smem_u32(bars + 1);   // [2]
  const uint32_t qd_empty0 = smem_u32(bars + 3);  // [2]
  const uint32_t sd_full = smem_u32(bars + 5);
  const uint32_t sd_empty = smem_u32(bars + 6);
  const uint32_t pd_full = smem_u32(bars + 7);
  const uint32_t pd_empty = smem_u32(bars + 8);
  const uint32_t acc_full = smem_u32(bars + 9);
  const uint32_t drain = smem_u32(bars + 10);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int nq = gridDim.x;
  const int j = blockIdx.x;  // key tile; tile 0 (most query tiles) starts first
  const int n = nq - j;      // query tiles i = j .. nq-1
  const int b = blockIdx.y / H, h = blockIdx.y % H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(qd_full0 + 8 * s, 1);
      mbar_init(qd_empty0 + 8 * s, 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(sd_empty, kCT);
    mbar_init(pd_full, kCT);
    mbar_init(pd_empty, 1);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA --
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQKV)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmDO)) : "memory");
      mbar_expect_tx(kv_full, 2 * kBox);
      tma_load_3d(smem_u32(sK), &tmQKV, kv_full, C + h * kHD, j * kTile, b);
      tma_load_3d(smem_u32(sV), &tmQKV, kv_full, 2 * C + h * kHD, j * kTile, b);
      uint32_t issued = 0, last_par = 0;
      for (int t = 0; t < n; ++t) {
        const int st = t & 1, i = j + t;
        const uint32_t par = (uint32_t)(t >> 1) & 1u;
        if (!mbar_wait(qd_empty0 + 8 * st, par ^ 1u, abort_flag, err)) break;
        const uint32_t fb = qd_full0 + 8 * st;
        mbar_expect_tx(fb, 2 * kBox);
        tma_load_3d(smem_u32(sQ + st * kBox), &tmQKV, fb, h * kHD, i * kTile, b);
        tma_load_3d(smem_u32(sDO + st * kBox), &tmDO, fb, h * kHD, i * kTile, b);
        issued |= 1u << st;
        last_par = (last_par & ~(1u << st)) | (par << st);
      }
      const uint64_t t0 = global_ns();
      drain_wait(kv_full, 0, t0);
      for (int s = 0; s < kQStages; ++s)
        if (issued & (1u << s)) drain_wait(qd_full0 + 8 * s, (last_par >> s) & 1u, t0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA --
      constexpr uint32_t idS = attn::idesc(kTile, false);
      constexpr uint32_t idA = attn::idesc(kHD, true);
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      bool ok = mbar_wait(kv_full, 0, abort_flag, err);
      auto issue_sd = [&](int t) -> bool {
        const int st = t & 1;
        if (!mbar_wait(qd_full0 + 8 * st, (uint32_t)(t >> 1) & 1u, abort_flag, err)) return false;
        if (!mbar_wait(sd_empty, ((uint32_t)t & 1u) ^ 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + st * kBox), do_base = smem_u32(sDO + st * kBox);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)  // S^T = K Q^T
          tc_mma(tmem, desc_kmajor(k_base, k), desc_kmajor(q_base, k), idS, k > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)  // dP^T = V dO^T
          tc_mma(tmem + kTile, desc_kmajor(v_base, k), desc_kmajor(do_base, k), idS, k > 0 ? 1u : 0u);
        tc_commit(sd_full);
        return true;
      };
      auto issue_acc = [&](int t) -> bool {
        const int st = t & 1;
        if (!mbar_wait(pd_full, (uint32_t)t & 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + st * kBox), do_base = smem_u32(sDO + st * kBox);
        const uint32_t pt = smem_u32(sPT), dst = smem_u32(sDST);
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k)  // dV += P^T dO
          tc_mma(tmem + 2 * kTile, desc_kmajor(pt + (uint32_t)((k >> 2) * kBox), k & 3),
                 desc_mnmajor(do_base, k), idA, (t > 0 || k > 0) ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k)  // dK += dS^T Q
          tc_mma(tmem + 2 * kTile + kHD, desc_kmajor(dst + (uint32_t)((k >> 2) * kBox), k & 3),
                 desc_mnmajor(q_base, k), idA, (t > 0 || k > 0) ? 1u : 0u);
        tc_commit(pd_empty);
        tc_commit(qd_empty0 + 8 * st);
        return true;
      };
      if (ok) ok = issue_sd(0);
      for (int t = 1; t <= n && ok; ++t) {
        if (t < n) ok = issue_sd(t);
        if (ok) ok = issue_acc(t - 1);
      }
      tc_commit(ok ? acc_full : drain);
      if (!ok) drain_wait(drain, 0, global_ns());
    }
  } else {
    // -------------------------------------------------------- compute --
    const int qw = warp & 3, half = (warp - 2) >> 2;
    const int r = qw * 32 + lane;
    const int kj = j * kTile + r;  // this thread's key row
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const float* lse_bh = lse + ((size_t)b * H + h) * T;
    const float* d_bh = dsum + ((size_t)b * H + h) * T;
    const int ct = threadIdx.x - 64;  // 0 .. 255
    bool ok = true;
    for (int t = 0; t < n && ok; ++t) {
      const int qc0 = (j + t) * kTile + 64 * half;  // first query column of this half
      // this tile's per-column L (log2 units) and D into shared memory,
      // loaded while the tensor core computes S^T and dP^T
      float* cl = col_lse + (t & 1) * 2 * kTile;
      {
        const int q = (j + t) * kTile + (ct & (kTile - 1));
        const float v = q < T ? (ct < kTile ? lse_bh[q] * kLog2e : d_bh[q]) : 0.f;
        cl[ct] = v;  // [0, 128): L, [128, 256): D
      }
      ok = cbar_and(mbar_wait(sd_full, (uint32_t)t & 1u, abort_flag, err));
      if (!ok) break;
      ok = cbar_and(mbar_wait(pd_empty, ((uint32_t)t & 1u) ^ 1u, abort_flag, err));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {  // 32 query columns at a time
        uint32_t rs[32], rp[32];
        const uint32_t col = (uint32_t)(64 * half + 32 * ch);
        tc_ld32(lane_base + col, rs);
        tc_ld32(lane_base + kTile + col, rp);
        float pv[32], dv[32];
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 a = *reinterpret_cast<const float4*>(cl + col + c);
          const float4 d = *reinterpret_cast<const float4*>(cl + kTile + col + c);
          pv[c] = a.x; pv[c + 1] = a.y; pv[c + 2] = a.z; pv[c + 3] = a.w;
          dv[c] = d.x; dv[c + 1] = d.y; dv[c + 2] = d.z; dv[c + 3] = d.w;
        }
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int q = qc0 + 32 * ch + c;
          float p = fast_exp2(fmaf(__uint_as_float(rs[c]), sl2, -pv[c]));
          if (q < kj || q >= T) p = 0.f;  // causal (only bites when i == j) and padding
          pv[c] = p;
          dv[c] = p * (__uint_as_float(rp[c]) - dv[c]);
        }
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          const int chunk = 4 * ch + c8;  // 16-byte chunk within this half's 128-byte row
          store8(reinterpret_cast<__nv_bfloat16*>(sPT + half * kBox + swz(r, chunk)), pv + 8 * c8);
          store8(reinterpret_cast<__nv_bfloat16*>(sDST + half * kBox + swz(r, chunk)), dv + 8 * c8);
        }
      }
      tc_fence_before();
      mbar_arrive(sd_empty);
      fence_async_smem();
      mbar_arrive(pd_full);
    }
    if (ok) ok = cbar_and(mbar_wait(acc_full, 0, abort_flag, err));
    if (ok) {
      tc_fence_after();
      uint32_t rv[32], rk[32];
      tc_ld32(lane_base + 2 * kTile + 32 * half, rv);
      tc_ld32(lane_base + 2 * kTile + kHD + 32 * half, rk);
      tc_wait_ld();
      if (kj < T) {
        __nv_bfloat16* row = dqkv + ((size_t)b * T + kj) * 3 * C + (size_t)h * kHD + 32 * half;
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float a[8], d[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            a[k] = __uint_as_float(rk[i + k]) * scale;
            d[k] = __uint_as_float(rv[i + k]);
          }
          store8(row + C + i, a);
          store8(row + 2 * C + i, d);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem);
}

// --------------------------------------------------------------------- dQ --
constexpr int kKVStages = 3;
constexpr size_t dq_smem_bytes() {
  // Q, dO, [K, V] x stages, dS double buffer (two boxes each), aux
  return 1024 + 2 * (size_t)kBox + 2 * (size_t)kKVStages * kBox + 4 * (size_t)kBox + kAux;
}

__global__ void __launch_bounds__(kThreadsBwd, 1)
    flash_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                           const __grid_constant__ CUtensorMap tmDO, const float* __restrict__ lse,
                           const float* __restrict__ dsum, __nv_bfloat16* __restrict__ dqkv, int T,
                           int C, int H, float sl2, float scale, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = sQ + kBox;
  uint8_t* sK = sDO + kBox;                // [kKVStages]
  uint8_t* sV = sK + kKVStages * kBox;     // [kKVStages]
  uint8_t* sDS = sV + kKVStages * kBox;    // [2 buffers][2 boxes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sDS + 4 * kBox);
  const uint32_t qd_full = smem_u32(bars + 0);
  const uint32_t kv_full0 = smem_u32(bars + 1);              // [3]
  const uint32_t kv_empty0 = smem_u32(bars + 1 + kKVStages); // [3]
  const uint32_t sd_full = smem_u32(bars + 7);
  const uint32_t sd_empty = smem_u32(bars + 8);
  const uint32_t ds_full0 = smem_u32(bars + 9);              // [2]
  const uint32_t ds_empty0 = smem_u32(bars + 11);            // [2]
  const uint32_t acc_full = smem_u32(bars + 13);
  const uint32_t drain = smem_u32(bars + 14);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int qb = gridDim.x - 1 - blockIdx.x;  // heaviest query tiles first
  const int n = qb + 1;                        // key tiles 0 .. qb
  const int b = blockIdx.y / H, h = blockIdx.y % H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(sd_empty, kCT);
    for (int s = 0; s < 2; ++s) {
      mbar_init(ds_full0 + 8 * s, kCT);
      mbar_init(ds_empty0 + 8 * s, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA --
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQKV)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmDO)) : "memory");
      mbar_expect_tx(qd_full, 2 * kBox);
      tma_load_3d(smem_u32(sQ), &tmQKV, qd_full, h * kHD, qb * kTile, b);
      tma_load_3d(smem_u32(sDO), &tmDO, qd_full, h * kHD, qb * kTile, b);
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      for (int jj = 0; jj < n; ++jj) {
        if (!mbar_wait(kv_empty0 + 8 * stage, phase ^ 1u, abort_flag, err)) break;
        const uint32_t fb = kv_full0 + 8 * stage;
        mbar_expect_tx(fb, 2 * kBox);
        tma_load_3d(smem_u32(sK + stage * kBox), &tmQKV, fb, C + h * kHD, jj * kTile, b);
        tma_load_3d(smem_u32(sV + stage * kBox), &tmQKV, fb, 2 * C + h * kHD, jj * kTile, b);
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kKVStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      const uint64_t t0 = global_ns();
      drain_wait(qd_full, 0, t0);
      for (int s = 0; s < kKVStages; ++s)
        if (issued & (1u << s)) drain_wait(kv_full0 + 8 * s, (last_par >> s) & 1u, t0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA --
      constexpr uint32_t idS = attn::idesc(kTile, false);
      constexpr uint32_t idQ = attn::idesc(kHD, true);
      const uint32_t q_base = smem_u32(sQ), do_base = smem_u32(sDO);
      bool ok = mbar_wait(qd_full, 0, abort_flag, err);
      auto issue_sd = [&](int jj) -> bool {
        const int st = jj % kKVStages;
        if (!mbar_wait(kv_full0 + 8 * st, (uint32_t)(jj / kKVStages) & 1u, abort_flag, err)) return false;
        if (!mbar_wait(sd_empty, ((uint32_t)jj & 1u) ^ 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(sK + st * kBox), v_base = smem_u32(sV + st * kBox);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)  // S = Q K^T
          tc_mma(tmem, desc_kmajor(q_base, k), desc_kmajor(k_base, k), idS, k > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)  // dP = dO V^T
          tc_mma(tmem + kTile, desc_kmajor(do_base, k), desc_kmajor(v_base, k), idS, k > 0 ? 1u : 0u);
        tc_commit(sd_full);
        return true;
      };
      auto issue_dq = [&](int jj) -> bool {
        const int st = jj % kKVStages, db = jj & 1;
        if (!mbar_wait(ds_full0 + 8 * db, (uint32_t)(jj >> 1) & 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t ds = smem_u32(sDS + db * 2 * kBox), k_base = smem_u32(sK + st * kBox);
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k)  // dQ += dS K
          tc_mma(tmem + 2 * kTile, desc_kmajor(ds + (uint32_t)((k >> 2) * kBox), k & 3),
                 desc_mnmajor(k_base, k), idQ, (jj > 0 || k > 0) ? 1u : 0u);
        tc_commit(ds_empty0 + 8 * db);
        tc_commit(kv_empty0 + 8 * st);
        return true;
      };
      if (ok) ok = issue_sd(0);
      for (int jj = 1; jj <= n && ok; ++jj) {
        if (jj < n) ok = issue_sd(jj);
        if (ok) ok = issue_dq(jj - 1);
      }
      tc_commit(ok ? acc_full : drain);
      if (!ok) drain_wait(drain, 0, global_ns());
    }
  } else {
    // -------------------------------------------------------- compute --
    const int qw = warp & 3, half = (warp - 2) >> 2;
    const int r = qw * 32 + lane;
    const int qi = qb * kTile + r;  // this thread's query row
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const size_t bh = (size_t)b * H + h;
    const float lse2 = qi < T ? lse[bh * T + qi] * kLog2e : 0.f;
    const float drow = qi < T ? dsum[bh * T + qi] : 0.f;
    bool ok = true;
    for (int jj = 0; jj < n && ok; ++jj) {
      const int db = jj & 1;
      const int key0 = jj * kTile + 64 * half;
      ok = cbar_and(mbar_wait(sd_full, (uint32_t)jj & 1u, abort_flag, err));
      if (!ok) break;
      ok = cbar_and(mbar_wait(ds_empty0 + 8 * db, ((uint32_t)(jj >> 1) & 1u) ^ 1u, abort_flag, err));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {  // 32 key columns at a time
        uint32_t rs[32], rp[32];
        const uint32_t col = (uint32_t)(64 * half + 32 * ch);
        tc_ld32(lane_base + col, rs);
        tc_ld32(lane_base + kTile + col, rp);
        tc_wait_ld();
        float ds[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int key = key0 + 32 * ch + c;
          float p = fast_exp2(fmaf(__uint_as_float(rs[c]), sl2, -lse2));
          if (key > qi || key >= T) p = 0.f;  // causal (only bites on the diagonal) and padding
          ds[c] = p * (__uint_as_float(rp[c]) - drow);
        }
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          store8(reinterpret_cast<__nv_bfloat16*>(sDS + (db * 2 + half) * kBox + swz(r, 4 * ch + c8)),
                 ds + 8 * c8);
      }
      tc_fence_before();
      mbar_arrive(sd_empty);
      fence_async_smem();
      mbar_arrive(ds_full0 + 8 * db);
    }
    if (ok) ok = cbar_and(mbar_wait(acc_full, 0, abort_flag, err));
    if (ok) {
      tc_fence_after();
      uint32_t rq[32];
      tc_ld32(lane_base + 2 * kTile + 32 * half, rq);
      tc_wait_ld();
      if (qi < T) {
        __nv_bfloat16* row = dqkv + ((size_t)b * T + qi) * 3 * C + (size_t)h * kHD + 32 * half;
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float a[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) a[k] = __uint_as_float(rq[i + k]) * scale;
          store8(row + i, a);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem);
}

}  // namespace

cudaError_t attention_bwd_tc(act_t* dqkv, const float* dsum, const act_t* datt, const act_t* qkv,
                             const float* lse, int B, int T, int C, int H, int* err,
                             cudaStream_t s) {
  if (C / H != kHD || (reinterpret_cast<uintptr_t>(qkv) & 15) || (reinterpret_cast<uintptr_t>(datt) & 15))
    return cudaErrorInvalidValue;
  CUtensorMap tq, td;
  cudaError_t e = attn::seq_map(&tq, qkv, B, T, 3 * C);
  if (e != cudaSuccess) return e;
  e = attn::seq_map(&td, datt, B, T, C);
  if (e != cudaSuccess) return e;
  constexpr size_t sm_a = dkdv_smem_bytes(), sm_b = dq_smem_bytes();
  static_assert(sm_a <= 232448 && sm_b <= 232448, "shared memory budget");
  static bool attr = false;
  if (!attr) {
    e = cudaFuncSetAttribute(flash_bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm_a);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(flash_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm_b);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const float sl2 = kLog2e / sqrtf((float)kHD), scale = 1.f / sqrtf((float)kHD);
  dim3 grid((T + kTile - 1) / kTile, B * H);
  flash_bwd_dkdv_tc_kernel<<<grid, kThreadsBwd, sm_a, s>>>(tq, td, lse, dsum, dqkv, T, C, H, sl2,
                                                           scale, err);
  flash_bwd_dq_tc_kernel<<<grid, kThreadsBwd, sm_b, s>>>(tq, td, lse, dsum, dqkv, T, C, H, sl2, scale,
                                                         err);
  note_launch(2);
  return cudaGetLastError();
}

}  // namespace gpt2k
