// Causal flash-attention backward on the sm_100a tensor cores (head dim 64),
// deterministic: no atomics, each gradient tile is owned by one work item.
//
// Given the forward's log-sum-exp L (natural log) and D = rowsum(dO * O):
//   P = exp(Q K^T / sqrt(d) - L),  dP = dO V^T,  dS = P * (dP - D)
//   dV = P^T dO,  dK = dS^T Q / sqrt(d),  dQ = dS K / sqrt(d)
//
// Two persistent kernels, one CTA per SM walking a static snake order over
// work items (heaviest first), 10 warps each (TMA, MMA, 8 compute warps,
// two threads per tile row):
//   dK/dV: item = (batch, head, key tile j); streams the query tiles i >= j
//          in 64-query halves (sub-tiles).  The tensor core computes
//          S^T = K Q^T and dP^T = V dO^T of a sub-tile into one of two TMEM
//          score buffers; the compute warps turn them into P^T and dS^T
//          (bf16, swizzled shared-memory tiles, also double-buffered); the
//          tensor core then accumulates dV += P^T dO and dK += dS^T Q in
//          TMEM (dO and Q read MN-major straight from their tiles).  K and V
//          are double-buffered across items.
//   dQ:    item = (batch, head, query tile i); streams the key tiles j <= i:
//          S = Q K^T and dP = dO V^T into TMEM, dS into shared memory,
//          dQ += dS K in TMEM (K read MN-major).  It runs first and also
//          forms D = rowsum(dO * O) of its rows from the dO and O tiles it
//          loads, storing it for the dK/dV kernel.
// The compute warps hand the score buffers back to the tensor core as soon
// as they have read them, so the next scores are computed while the current
// ones are finished; the gradient accumulators are double-buffered in TMEM,
// so an item's result is written while the next item runs.  Compute warps
// wait per warp (no block-wide barrier in the loop), and the causal mask is
// applied only on the diagonal tile and the one holding the end of the
// sequence.  Every wait is bounded (error word ERR_TIMEOUT).

#include <type_traits>

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
constexpr uint32_t kAccCol = 2 * kTile;  // accumulators after the two score buffers
constexpr int kAux = 1024;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ bool warp_and(bool p) { return __all_sync(0xffffffffu, p); }

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

// Work item k of this CTA in a snake order over the item list; -1 when the
// CTA has no item k.
__device__ __forceinline__ int snake_item(int k, int count) {
  const int G = gridDim.x;
  const int w = k * G + ((k & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
  return w < count ? w : -1;
}

// ------------------------------------------------------------------ dK/dV --
// The query tiles are processed in 64-query halves ("sub-tiles"), so that the
// score products of two sub-tiles fit in TMEM next to the two accumulator
// pairs: while the compute warps turn one sub-tile's S^T and dP^T into P^T
// and dS^T, the tensor core already holds (or is computing) the next
// sub-tile's scores and runs the previous sub-tile's dV and dK products.
// TMEM columns: [0,128) and [128,256) score buffers (S^T 64 | dP^T 64),
// [256,512) two accumulator pairs (dV 64 | dK 64).
constexpr int kQStages = 2;
constexpr int kSub = 64;  // queries per sub-tile
constexpr size_t dkdv_smem_bytes() {
  // [K, V] x 2 items, [Q, dO] x stages, P^T and dS^T x 2 sub-tiles (one box
  // each), each compute warp's per-column L and D of two sub-tiles, aux
  return 1024 + 4 * (size_t)kBox + 2 * (size_t)kQStages * kBox + 4 * (size_t)kBox +
         (kCT / 32) * 2 * 64 * sizeof(float) + kAux;
}

__global__ void __launch_bounds__(kThreadsBwd, 1)
    flash_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                             const __grid_constant__ CUtensorMap tmDO, const float* __restrict__ lse,
                             const float* __restrict__ dsum, __nv_bfloat16* __restrict__ dqkv, int B,
                             int T, int C, int H, float sl2, float scale, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sKV = smem;                    // [2 items][K box, V box]
  uint8_t* sQ = sKV + 4 * kBox;           // [kQStages]
  uint8_t* sDO = sQ + kQStages * kBox;    // [kQStages]
  uint8_t* sPT = sDO + kQStages * kBox;   // [2 sub-tiles]: 128 keys x 64 queries
  uint8_t* sDST = sPT + 2 * kBox;         // [2 sub-tiles]
  float* col_lse = reinterpret_cast<float*>(sDST + 2 * kBox);  // [warp][2][L 32, D 32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(col_lse + (kCT / 32) * 2 * 64);
  const uint32_t kv_full0 = smem_u32(bars + 0);     // [2]
  const uint32_t kv_empty0 = smem_u32(bars + 2);    // [2]
  const uint32_t qd_full0 = smem_u32(bars + 4);     // [2]
  const uint32_t qd_empty0 = smem_u32(bars + 6);    // [2]
  const uint32_t sd_full0 = smem_u32(bars + 8);     // [2]
  const uint32_t sd_empty0 = smem_u32(bars + 10);   // [2]
  const uint32_t pd_full0 = smem_u32(bars + 12);    // [2]
  const uint32_t pd_empty0 = smem_u32(bars + 14);   // [2]
  const uint32_t acc_full0 = smem_u32(bars + 16);   // [2]
  const uint32_t acc_empty0 = smem_u32(bars + 18);  // [2]
  const uint32_t drain = smem_u32(bars + 20);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 21);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int nq = (T + kTile - 1) / kTile;
  const int BH = B * H, items = nq * BH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 1);
      mbar_init(qd_full0 + 8 * s, 1);
      mbar_init(qd_empty0 + 8 * s, 1);
      mbar_init(sd_full0 + 8 * s, 1);
      mbar_init(sd_empty0 + 8 * s, kCT);
      mbar_init(pd_full0 + 8 * s, kCT);
      mbar_init(pd_empty0 + 8 * s, 1);
      mbar_init(acc_full0 + 8 * s, 1);
      mbar_init(acc_empty0 + 8 * s, kCT);
    }
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
      uint32_t n_item = 0, g = 0;  // items started, query tiles loaded
      uint32_t kv_issued = 0, kv_par = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++n_item) {
        const int w = snake_item(k, items);
        if (w < 0) break;
        const int j = w / BH, bh = w % BH, b = bh / H, h = bh % H;
        const int n = nq - j;  // query tiles i = j .. nq-1
        const int ks = n_item & 1;
        const uint32_t kpar = (n_item >> 1) & 1u;
        if (!mbar_wait(kv_empty0 + 8 * ks, kpar ^ 1u, abort_flag, err)) break;
        const uint32_t kb = kv_full0 + 8 * ks;
        mbar_expect_tx(kb, 2 * kBox);
        tma_load_3d(smem_u32(sKV + ks * 2 * kBox), &tmQKV, kb, C + h * kHD, j * kTile, b);
        tma_load_3d(smem_u32(sKV + ks * 2 * kBox + kBox), &tmQKV, kb, 2 * C + h * kHD, j * kTile, b);
        kv_issued |= 1u << ks;
        kv_par = (kv_par & ~(1u << ks)) | (kpar << ks);
        for (int t = 0; t < n; ++t, ++g) {
          const int st = g & 1;
          const uint32_t par = (g >> 1) & 1u;
          if (!mbar_wait(qd_empty0 + 8 * st, par ^ 1u, abort_flag, err)) {
            ok = false;
            break;
          }
          const uint32_t fb = qd_full0 + 8 * st;
          mbar_expect_tx(fb, 2 * kBox);
          tma_load_3d(smem_u32(sQ + st * kBox), &tmQKV, fb, h * kHD, (j + t) * kTile, b);
          tma_load_3d(smem_u32(sDO + st * kBox), &tmDO, fb, h * kHD, (j + t) * kTile, b);
          issued |= 1u << st;
          last_par = (last_par & ~(1u << st)) | (par << st);
        }
      }
      // every copy issued lands before the shared memory is released
      const uint64_t t0 = global_ns();
      for (int s = 0; s < 2; ++s) {
        if (kv_issued & (1u << s)) drain_wait(kv_full0 + 8 * s, (kv_par >> s) & 1u, t0);
        if (issued & (1u << s)) drain_wait(qd_full0 + 8 * s, (last_par >> s) & 1u, t0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA --
      constexpr uint32_t idS = attn::idesc(kSub, false);
      constexpr uint32_t idA = attn::idesc(kHD, true);
      // S^T = K Q_s^T and dP^T = V dO_s^T of sub-tile s (half hs of the
      // query tile in stage st) into score buffer s % 2
      auto issue_sd = [&](uint32_t s, int st, uint32_t tpar, int hs, int ks) -> bool {
        const uint32_t sb = s & 1u;
        if (!mbar_wait(qd_full0 + 8 * st, tpar, abort_flag, err)) return false;
        if (!mbar_wait(sd_empty0 + 8 * sb, ((s >> 1) & 1u) ^ 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(sKV + ks * 2 * kBox), v_base = k_base + kBox;
        const uint32_t q_base = smem_u32(sQ + st * kBox) + hs * (kSub * 128);
        const uint32_t do_base = smem_u32(sDO + st * kBox) + hs * (kSub * 128);
        const uint32_t d = tmem + sb * 2 * kSub;
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)
          tc_mma(d, desc_kmajor(k_base, k), desc_kmajor(q_base, k), idS, k > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)
          tc_mma(d + kSub, desc_kmajor(v_base, k), desc_kmajor(do_base, k), idS, k > 0 ? 1u : 0u);
        tc_commit(sd_full0 + 8 * sb);
        return true;
      };
      // dV += P^T dO_s, dK += dS^T Q_s of a sub-tile whose P^T and dS^T are
      // (being) written; releases the query tile after its second half and
      // hands the accumulators over after the item's last sub-tile
      struct Pend {
        uint32_t s, acc, ab;
        int st, hs;
        bool first, last;
      };
      auto issue_acc = [&](const Pend& p) -> bool {
        const uint32_t sb = p.s & 1u;
        if (!mbar_wait(pd_full0 + 8 * sb, (p.s >> 1) & 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + p.st * kBox), do_base = smem_u32(sDO + p.st * kBox);
        const uint32_t pt = smem_u32(sPT + sb * kBox), dst = smem_u32(sDST + sb * kBox);
#pragma unroll
        for (int k = 0; k < kSub / 16; ++k)
          tc_mma(tmem + p.acc, desc_kmajor(pt, k), desc_mnmajor(do_base, 4 * p.hs + k), idA,
                 (!p.first || k > 0) ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < kSub / 16; ++k)
          tc_mma(tmem + p.acc + kHD, desc_kmajor(dst, k), desc_mnmajor(q_base, 4 * p.hs + k), idA,
                 (!p.first || k > 0) ? 1u : 0u);
        tc_commit(pd_empty0 + 8 * sb);
        if (p.hs == 1) tc_commit(qd_empty0 + 8 * p.st);
        if (p.last) tc_commit(acc_full0 + 8 * p.ab);
        return true;
      };
      // One flat sequence over every sub-tile of every item: the scores of
      // sub-tile s are issued before the products of sub-tile s - 1.
      uint32_t n_item = 0, gs = 0, gt = 0;
      Pend pend{};
      bool have = false, ok = true;
      for (int k = 0; ok; ++k, ++n_item) {
        const int w = snake_item(k, items);
        if (w < 0) break;
        const int n = nq - w / BH;
        const int ks = n_item & 1;
        const uint32_t ab = n_item & 1u, acc = kAccCol + ab * 2 * kHD;
        ok = mbar_wait(kv_full0 + 8 * ks, (n_item >> 1) & 1u, abort_flag, err);
        if (ok) ok = mbar_wait(acc_empty0 + 8 * ab, ((n_item >> 1) & 1u) ^ 1u, abort_flag, err);
        if (!ok) break;
        tc_fence_after();
        for (int t = 0; t < n && ok; ++t, ++gt) {
          const int st = gt & 1;
          const uint32_t tpar = (gt >> 1) & 1u;
          for (int hs = 0; hs < 2; ++hs, ++gs) {
            ok = issue_sd(gs, st, tpar, hs, ks);
            if (!ok) break;
            if (t == n - 1 && hs == 1) tc_commit(kv_empty0 + 8 * ks);  // K, V no longer read
            if (have) ok = issue_acc(pend);
            if (!ok) break;
            pend = Pend{gs, acc, ab, st, hs, t == 0 && hs == 0, t == n - 1 && hs == 1};
            have = true;
          }
        }
      }
      if (ok && have) ok = issue_acc(pend);
      if (!ok) {  // let issued MMAs finish before TMEM is released
        tc_commit(drain);
        drain_wait(drain, 0, global_ns());
      }
    }
  } else {
    // -------------------------------------------------------- compute --
    // thread = key row r, owning 32 of a sub-tile's 64 query columns.  Every
    // wait is per warp (warps drift apart and overlap their latencies); each
    // warp stages the L and D of its own 32 columns.
    const int qw = warp & 3, half = (warp - 2) >> 2;
    const int r = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    float* wcl = col_lse + (warp - 2) * 2 * 64;  // [2 sub-tiles][L 32 | D 32]
    uint32_t n_item = 0, gs = 0;
    bool ok = true;
    for (int k = 0; ok; ++k, ++n_item) {
      const int w = snake_item(k, items);
      if (w < 0) break;
      const int j = w / BH, bh = w % BH, b = bh / H, h = bh % H;
      const int n = nq - j;
      const int kj = j * kTile + r;  // this thread's key row
      const float* lse_bh = lse + (size_t)bh * T;
      const float* d_bh = dsum + (size_t)bh * T;
      for (int t = 0; t < n && ok; ++t) {
        for (int hs = 0; hs < 2; ++hs, ++gs) {
          const uint32_t sb = gs & 1u;
          const int cq = kSub * hs + 32 * half;  // first column of this thread in the tile
          const int qc0 = (j + t) * kTile + cq;  // its query index
          // L (log2 units) and D of the warp's 32 columns, loaded while the
          // tensor core computes the scores
          float* cl = wcl + sb * 64;
          {
            const int q = qc0 + lane;
            cl[lane] = q < T ? lse_bh[q] * kLog2e : 0.f;
            cl[32 + lane] = q < T ? d_bh[q] : 0.f;
          }
          __syncwarp();
          // causal mask on the diagonal tile, padding past T on the last one
          const bool masked = t == 0 || qc0 - cq + kSub * (hs + 1) > T;
          ok = warp_and(mbar_wait(sd_full0 + 8 * sb, (gs >> 1) & 1u, abort_flag, err));
          if (!ok) break;
          tc_fence_after();
          const uint32_t s_col = lane_base + sb * 2 * kSub + 32 * half;
          const uint32_t pt_row = smem_u32(sPT + sb * kBox) + (uint32_t)(r * 128);
          const uint32_t dst_row = smem_u32(sDST + sb * kBox) + (uint32_t)(r * 128);
          uint32_t sa[16], pa[16], sb16[16], pb[16];
          auto ld_chunk = [&](int ch, uint32_t* s_, uint32_t* p_) {
            attn::tc_ld16(s_col + 16 * ch, s_);
            attn::tc_ld16(s_col + kSub + 16 * ch, p_);
          };
          auto do_chunk = [&](int ch, const uint32_t* s_, const uint32_t* p_, auto mask) -> bool {
            float pv[16], dv[16];
#pragma unroll
            for (int c = 0; c < 16; c += 4) {
              const float4 a = *reinterpret_cast<const float4*>(cl + 16 * ch + c);
              const float4 d = *reinterpret_cast<const float4*>(cl + 32 + 16 * ch + c);
              pv[c] = a.x; pv[c + 1] = a.y; pv[c + 2] = a.z; pv[c + 3] = a.w;
              dv[c] = d.x; dv[c + 1] = d.y; dv[c + 2] = d.z; dv[c + 3] = d.w;
            }
            const int lim = kj - qc0 - 16 * ch;  // columns c < lim are queries before the key
            const int tcut = T - qc0 - 16 * ch;  // columns c >= tcut are past the sequence
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              float p = fast_exp2(fmaf(__uint_as_float(s_[c]), sl2, -pv[c]));
              if (decltype(mask)::value && (c < lim || c >= tcut)) p = 0.f;
              pv[c] = p;
              dv[c] = p * (__uint_as_float(p_[c]) - dv[c]);
            }
            // the products of sub-tile gs - 2 have read this P^T / dS^T buffer
            if (ch == 0 &&
                !warp_and(mbar_wait(pd_empty0 + 8 * sb, ((gs >> 1) & 1u) ^ 1u, abort_flag, err)))
              return false;
#pragma unroll
            for (int c8 = 0; c8 < 2; ++c8) {
              const uint32_t off = (uint32_t)(((4 * half + 2 * ch + c8) ^ (r & 7)) << 4);
              attn::st_shared_bf16x8(pt_row + off, pv + 8 * c8);
              attn::st_shared_bf16x8(dst_row + off, dv + 8 * c8);
            }
            return true;
          };
          ld_chunk(0, sa, pa);
          tc_wait_ld();
          ld_chunk(1, sb16, pb);
          ok = masked ? do_chunk(0, sa, pa, std::true_type{}) : do_chunk(0, sa, pa, std::false_type{});
          tc_wait_ld();
          tc_fence_before();
          mbar_arrive(sd_empty0 + 8 * sb);  // the scores are read: sub-tile gs + 2 may be computed
          if (!ok) break;
          if (masked) do_chunk(1, sb16, pb, std::true_type{});
          else do_chunk(1, sb16, pb, std::false_type{});
          fence_async_smem();
          mbar_arrive(pd_full0 + 8 * sb);
        }
      }
      if (!ok) break;
      // the item's dV and dK (accumulator pair n_item % 2)
      const uint32_t ab = n_item & 1u, acc = kAccCol + ab * 2 * kHD;
      ok = warp_and(mbar_wait(acc_full0 + 8 * ab, (n_item >> 1) & 1u, abort_flag, err));
      if (!ok) break;
      tc_fence_after();
      uint32_t rv[32], rk[32];
      tc_ld32(lane_base + acc + 32 * half, rv);
      tc_ld32(lane_base + acc + kHD + 32 * half, rk);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(acc_empty0 + 8 * ab);
      if (kj < T) {
        __nv_bfloat16* row = dqkv + ((size_t)b * T + kj) * 3 * C + (size_t)h * kHD + 32 * half;
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float a[8], d[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            a[q] = __uint_as_float(rk[i + q]) * scale;
            d[q] = __uint_as_float(rv[i + q]);
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
  // Q, dO, O, [K, V] x stages, dS (two buffers of two boxes), aux
  return 1024 + 3 * (size_t)kBox + 2 * (size_t)kKVStages * kBox + 4 * (size_t)kBox + kAux;
}

__global__ void __launch_bounds__(kThreadsBwd, 1)
    flash_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                           const __grid_constant__ CUtensorMap tmDO,
                           const __grid_constant__ CUtensorMap tmO, const float* __restrict__ lse,
                           float* __restrict__ dsum, __nv_bfloat16* __restrict__ dqkv, int B,
                           int T, int C, int H, float sl2, float scale, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = sQ + kBox;
  uint8_t* sO = sDO + kBox;                // the forward's output rows (for D)
  uint8_t* sK = sO + kBox;                 // [kKVStages]
  uint8_t* sV = sK + kKVStages * kBox;     // [kKVStages]
  uint8_t* sDS = sV + kKVStages * kBox;    // [2 buffers][2 boxes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sDS + 4 * kBox);
  const uint32_t qd_full = smem_u32(bars + 0);
  const uint32_t qd_empty = smem_u32(bars + 1);
  const uint32_t kv_full0 = smem_u32(bars + 2);              // [3]
  const uint32_t kv_empty0 = smem_u32(bars + 2 + kKVStages); // [3]
  const uint32_t sd_full = smem_u32(bars + 8);
  const uint32_t sd_empty = smem_u32(bars + 9);
  const uint32_t ds_full0 = smem_u32(bars + 10);             // [2]
  const uint32_t ds_empty0 = smem_u32(bars + 12);            // [2]
  const uint32_t acc_full0 = smem_u32(bars + 14);            // [2]
  const uint32_t acc_empty0 = smem_u32(bars + 16);           // [2]
  const uint32_t drain = smem_u32(bars + 18);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int nq = (T + kTile - 1) / kTile;
  const int BH = B * H, items = nq * BH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    mbar_init(qd_empty, 1 + kCT);  // the last S/dP product, and every compute thread's D
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(sd_empty, kCT);
    for (int s = 0; s < 2; ++s) {
      mbar_init(ds_full0 + 8 * s, kCT);
      mbar_init(ds_empty0 + 8 * s, 1);
      mbar_init(acc_full0 + 8 * s, 1);
      mbar_init(acc_empty0 + 8 * s, kCT);
    }
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
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmO)) : "memory");
      uint32_t n_item = 0, gk = 0;  // items started, key tiles loaded
      uint32_t issued = 0, last_par = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++n_item) {
        const int w = snake_item(k, items);
        if (w < 0) break;
        const int i = nq - 1 - w / BH, bh = w % BH, b = bh / H, h = bh % H;
        const int n = i + 1;  // key tiles 0 .. i
        if (!mbar_wait(qd_empty, (n_item & 1u) ^ 1u, abort_flag, err)) break;
        mbar_expect_tx(qd_full, 3 * kBox);
        tma_load_3d(smem_u32(sQ), &tmQKV, qd_full, h * kHD, i * kTile, b);
        tma_load_3d(smem_u32(sDO), &tmDO, qd_full, h * kHD, i * kTile, b);
        tma_load_3d(smem_u32(sO), &tmO, qd_full, h * kHD, i * kTile, b);
        for (int jj = 0; jj < n; ++jj, ++gk) {
          const int st = gk % kKVStages;
          const uint32_t par = (gk / kKVStages) & 1u;
          if (!mbar_wait(kv_empty0 + 8 * st, par ^ 1u, abort_flag, err)) {
            ok = false;
            break;
          }
          const uint32_t fb = kv_full0 + 8 * st;
          mbar_expect_tx(fb, 2 * kBox);
          tma_load_3d(smem_u32(sK + st * kBox), &tmQKV, fb, C + h * kHD, jj * kTile, b);
          tma_load_3d(smem_u32(sV + st * kBox), &tmQKV, fb, 2 * C + h * kHD, jj * kTile, b);
          issued |= 1u << st;
          last_par = (last_par & ~(1u << st)) | (par << st);
        }
      }
      const uint64_t t0 = global_ns();
      if (n_item) drain_wait(qd_full, (n_item - 1) & 1u, t0);
      for (int s = 0; s < kKVStages; ++s)
        if (issued & (1u << s)) drain_wait(kv_full0 + 8 * s, (last_par >> s) & 1u, t0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA --
      constexpr uint32_t idS = attn::idesc(kTile, false);
      constexpr uint32_t idQ = attn::idesc(kHD, true);
      const uint32_t q_base = smem_u32(sQ), do_base = smem_u32(sDO);
      uint32_t n_item = 0, gk = 0;
      bool ok = true;
      // S and dP against the key tile with global index gg
      auto issue_sd = [&](uint32_t gg) -> bool {
        const int st = gg % kKVStages;
        if (!mbar_wait(kv_full0 + 8 * st, (gg / kKVStages) & 1u, abort_flag, err)) return false;
        if (!mbar_wait(sd_empty, (gg & 1u) ^ 1u, abort_flag, err)) return false;
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
      // dQ (+)= dS K into the accumulator at column acc
      auto issue_dq = [&](uint32_t gg, uint32_t acc, bool first) -> bool {
        const int st = gg % kKVStages, db = gg & 1;
        if (!mbar_wait(ds_full0 + 8 * db, (gg >> 1) & 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t ds = smem_u32(sDS + db * 2 * kBox), k_base = smem_u32(sK + st * kBox);
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k)
          tc_mma(tmem + acc, desc_kmajor(ds + (uint32_t)((k >> 2) * kBox), k & 3),
                 desc_mnmajor(k_base, k), idQ, (!first || k > 0) ? 1u : 0u);
        tc_commit(ds_empty0 + 8 * db);
        tc_commit(kv_empty0 + 8 * st);
        return true;
      };
      for (int k = 0; ok; ++k, ++n_item) {
        const int w = snake_item(k, items);
        if (w < 0) break;
        const int n = nq - w / BH;  // i + 1
        const uint32_t ab = n_item & 1u, acc = kAccCol + ab * kHD;
        ok = mbar_wait(qd_full, n_item & 1u, abort_flag, err);
        if (ok) ok = mbar_wait(acc_empty0 + 8 * ab, ((n_item >> 1) & 1u) ^ 1u, abort_flag, err);
        if (!ok) break;
        tc_fence_after();
        ok = issue_sd(gk);
        if (ok && n == 1) tc_commit(qd_empty);  // Q and dO are no longer read
        for (int jj = 1; jj <= n && ok; ++jj) {
          if (jj < n) {
            ok = issue_sd(gk + jj);
            if (ok && jj == n - 1) tc_commit(qd_empty);
          }
          if (ok) ok = issue_dq(gk + jj - 1, acc, jj == 1);
        }
        if (ok) tc_commit(acc_full0 + 8 * ab);
        gk += n;
      }
      if (!ok) {
        tc_commit(drain);
        drain_wait(drain, 0, global_ns());
      }
    }
  } else {
    // -------------------------------------------------------- compute --
    const int qw = warp & 3, half = (warp - 2) >> 2;
    const int r = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    uint32_t n_item = 0, gk = 0;
    bool ok = true;
    for (int k = 0; ok; ++k, ++n_item) {
      const int w = snake_item(k, items);
      if (w < 0) break;
      const int i = nq - 1 - w / BH, bh = w % BH, b = bh / H, h = bh % H;
      const int n = i + 1;
      const int qi = i * kTile + r;  // this thread's query row
      const float lse2 = qi < T ? lse[(size_t)bh * T + qi] * kLog2e : 0.f;
      // D = rowsum(dO * O) of this row from the item's dO and O tiles (rows
      // past T are zero-filled); stored for the dK/dV kernel, which runs next
      ok = warp_and(mbar_wait(qd_full, n_item & 1u, abort_flag, err));
      if (!ok) break;
      float drow = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float a[8], o[8];
        load8(reinterpret_cast<const __nv_bfloat16*>(sDO + swz(r, c)), a);
        load8(reinterpret_cast<const __nv_bfloat16*>(sO + swz(r, c)), o);
#pragma unroll
        for (int e = 0; e < 8; ++e) drow = fmaf(a[e], o[e], drow);
      }
      mbar_arrive(qd_empty);  // this thread is done with dO and O
      if (half == 0 && qi < T) dsum[(size_t)bh * T + qi] = drow;
      for (int jj = 0; jj < n && ok; ++jj) {
        const uint32_t gg = gk + jj;
        const int db = gg & 1;
        const int key0 = jj * kTile + 64 * half;
        const uint32_t ds_row = smem_u32(sDS + (db * 2 + half) * kBox) + (uint32_t)(r * 128);
        // causal mask on the diagonal tile, padding past T on the last one
        const bool masked = jj == i || (jj + 1) * kTile > T;
        ok = warp_and(mbar_wait(sd_full, gg & 1u, abort_flag, err));
        if (!ok) break;
        tc_fence_after();
        // 16 key columns per chunk; the next chunk's TMEM loads are in
        // flight while the current chunk is computed
        uint32_t sa[16], pa[16], sb[16], pb[16];
        auto ld_chunk = [&](int ch, uint32_t* s_, uint32_t* p_) {
          const uint32_t col = (uint32_t)(64 * half + 16 * ch);
          attn::tc_ld16(lane_base + col, s_);
          attn::tc_ld16(lane_base + kTile + col, p_);
        };
        auto do_chunk = [&](int ch, const uint32_t* s_, const uint32_t* p_, auto mask) -> bool {
          const int lim = qi - key0 - 16 * ch;  // columns c > lim are keys after the query
          const int tcut = T - key0 - 16 * ch;  // columns c >= tcut are past the sequence
          float ds[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float p = fast_exp2(fmaf(__uint_as_float(s_[c]), sl2, -lse2));
            if (decltype(mask)::value && (c > lim || c >= tcut)) p = 0.f;
            ds[c] = p * (__uint_as_float(p_[c]) - drow);
          }
          // the product two tiles back has read this dS buffer
          if (ch == 0 &&
              !warp_and(mbar_wait(ds_empty0 + 8 * db, ((gg >> 1) & 1u) ^ 1u, abort_flag, err)))
            return false;
#pragma unroll
          for (int c8 = 0; c8 < 2; ++c8)
            attn::st_shared_bf16x8(ds_row + (uint32_t)(((2 * ch + c8) ^ (r & 7)) << 4), ds + 8 * c8);
          return true;
        };
        auto run = [&](auto mask) {
          ld_chunk(0, sa, pa);
          tc_wait_ld();
          ld_chunk(1, sb, pb);
          ok = do_chunk(0, sa, pa, mask);
          tc_wait_ld();
          if (ok) {
            ld_chunk(2, sa, pa);
            do_chunk(1, sb, pb, mask);
            tc_wait_ld();
            ld_chunk(3, sb, pb);
            do_chunk(2, sa, pa, mask);
            tc_wait_ld();
            tc_fence_before();
            mbar_arrive(sd_empty);  // both score buffers are read: the next tile's may be computed
            do_chunk(3, sb, pb, mask);
          }
        };
        if (masked) run(std::true_type{});
        else run(std::false_type{});
        if (!ok) break;
        fence_async_smem();
        mbar_arrive(ds_full0 + 8 * db);
      }
      if (!ok) break;
      const uint32_t ab = n_item & 1u, acc = kAccCol + ab * kHD;
      ok = warp_and(mbar_wait(acc_full0 + 8 * ab, (n_item >> 1) & 1u, abort_flag, err));
      if (!ok) break;
      tc_fence_after();
      uint32_t rq[32];
      tc_ld32(lane_base + acc + 32 * half, rq);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(acc_empty0 + 8 * ab);
      if (qi < T) {
        __nv_bfloat16* row = dqkv + ((size_t)b * T + qi) * 3 * C + (size_t)h * kHD + 32 * half;
#pragma unroll
        for (int q = 0; q < 32; q += 8) {
          float a[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(rq[q + e]) * scale;
          store8(row + q, a);
        }
      }
      gk += n;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem);
}

}  // namespace

cudaError_t attention_bwd_tc(act_t* dqkv, float* dsum, const act_t* datt, const act_t* qkv,
                             const act_t* att, const float* lse, int B, int T, int C, int H,
                             int* err, cudaStream_t s) {
  if (C / H != kHD || (reinterpret_cast<uintptr_t>(qkv) & 15) ||
      (reinterpret_cast<uintptr_t>(datt) & 15) || (reinterpret_cast<uintptr_t>(att) & 15))
    return cudaErrorInvalidValue;
  CUtensorMap tq, td, to;
  cudaError_t e = attn::seq_map(&tq, qkv, B, T, 3 * C);
  if (e != cudaSuccess) return e;
  e = attn::seq_map(&td, datt, B, T, C);
  if (e != cudaSuccess) return e;
  e = attn::seq_map(&to, att, B, T, C);
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
  const int items = ((T + kTile - 1) / kTile) * B * H;
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = items < sms ? items : sms;
  // dQ first: it forms D = rowsum(dO * O) of its query tiles for dK/dV
  flash_bwd_dq_tc_kernel<<<grid, kThreadsBwd, sm_b, s>>>(tq, td, to, lse, dsum, dqkv, B, T, C, H,
                                                         sl2, scale, err);
  flash_bwd_dkdv_tc_kernel<<<grid, kThreadsBwd, sm_a, s>>>(tq, td, lse, dsum, dqkv, B, T, C, H, sl2,
                                                           scale, err);
  note_launch(2);
  return cudaGetLastError();
}

}  // namespace gpt2k
