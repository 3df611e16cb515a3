// Causal flash-attention backward on the sm_100a tensor cores (head dim 64),
// deterministic: no atomics, each gradient tile is owned by one work item.
//
// Given the forward's log-sum-exp L (natural log) and D = rowsum(dO * O):
//   P = exp(Q K^T / sqrt(d) - L),  dP = dO V^T,  dS = P * (dP - D)
//   dV = P^T dO,  dK = dS^T Q / sqrt(d),  dQ = dS K / sqrt(d)
//
// Two persistent kernels, one CTA per SM walking a static snake order over
// work items (heaviest first): a TMA warp, two MMA-issuing warps (scores,
// and the products that accumulate the gradients) and the compute warps
// (four threads per key row in dK/dV, two per query row in dQ).  In both,
// the second product of each step takes its A operand (P^T and dS^T, or dS)
// from TMEM, where the compute warps write it as packed bf16, so shared
// memory only feeds the tensor core the operands that TMA brings in; each
// compute warp writes its rows of the item's gradients into a shared-memory
// box of its own that one TMA store sends out (measured: 194 -> 178 us for
// both kernels at B16 x T1024 x H12, against per-thread row stores):
//   dQ:    item = (batch, head, query tile i); streams the key tiles j <= i:
//          S = Q K^T and dP = dO V^T into TMEM, dS into one of two TMEM
//          buffers, dQ += dS K in one of two TMEM accumulators (K read
//          MN-major).  It runs first: it also forms D = rowsum(dO * O) of
//          its rows from the dO and O tiles it loads, and stores, per
//          128-row query tile, the 128 values of -L log2(e) followed by the
//          128 values of D for the dK/dV kernel, padded to whole tiles (rows
//          past T get -L log2(e) = -inf, D = 0, which makes their P exactly
//          0 there).
//   dK/dV: item = (batch, head, key tile j); streams the query tiles i >= j
//          in 64-query halves (sub-tiles).  The tensor core computes
//          S^T = K Q^T and dP^T = V dO^T of a sub-tile into one of two TMEM
//          score buffers; the compute warps turn them into P^T and dS^T in
//          one of two TMEM operand buffers; the tensor core then accumulates
//          dV += P^T dO and dK += dS^T Q in TMEM (dO and Q read MN-major
//          straight from their tiles).  The (L, D) values of each query tile
//          arrive by a bulk copy next to its Q and dO tiles.
// Each compute thread loads its part of the scores from TMEM in one round
// trip and hands the buffer straight back, so the tensor core computes the
// next scores while the current ones are exponentiated.  The causal mask is
// applied only on the diagonal tile.  Every wait is bounded (error word
// ERR_TIMEOUT).

#include <type_traits>

#include "attention_tc.cuh"

namespace gpt2k {

namespace {

using namespace tc;
using attn::kBox;
using attn::kHD;
using attn::kTile;

// dK/dV: KV_SPLIT compute threads per key row (four warps per lane quarter
// of TMEM with KV_SPLIT = 4), each owning 64 / KV_SPLIT of a sub-tile's
// query columns
#ifndef KV_SPLIT
#define KV_SPLIT 4
#endif
constexpr int kKvSplit = KV_SPLIT;
constexpr int kCTkv = 128 * kKvSplit;
constexpr int kThreadsKV = 64 + kCTkv + 32;
constexpr int kMma2KV = kThreadsKV / 32 - 1;
constexpr int kColsKV = 64 / kKvSplit;  // query columns per thread and sub-tile
// dQ: Q_SPLIT compute threads per query row, each owning 128 / Q_SPLIT of a
// key tile's columns (measured: 2 beats 4 here, 180 vs 202 us for the
// backward at B16 x T1024)
#ifndef Q_SPLIT
#define Q_SPLIT 2
#endif
constexpr int kQSplit = Q_SPLIT;
constexpr int kCTq = 128 * kQSplit;
constexpr int kThreadsQ = 64 + kCTq + 32;
constexpr int kMma2Q = kThreadsQ / 32 - 1;
constexpr int kColsQ = kTile / kQSplit;
constexpr uint32_t kTmemCols = 512;
constexpr int kAux = 1024;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kNegInf = 0xff800000u;

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

// 32 lanes x 16 consecutive 32-bit columns from registers into TMEM.
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns from registers into TMEM.
__device__ __forceinline__ void tc_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
// TMEM load (16 or 32 columns) / store (8, 16 or 32 columns) for this lane.
template <int N>
__device__ __forceinline__ void tc_ldn(uint32_t taddr, uint32_t* r) {
  static_assert(N == 16 || N == 32, "TMEM load width");
  if constexpr (N == 32) tc_ld32(taddr, r);
  else attn::tc_ld16(taddr, r);
}
template <int N>
__device__ __forceinline__ void tc_stn(uint32_t taddr, const uint32_t* r) {
  static_assert(N == 8 || N == 16 || N == 32, "TMEM store width");
  if constexpr (N == 32) attn::tc_st32(taddr, r);
  else if constexpr (N == 16) tc_st16(taddr, r);
  else tc_st8(taddr, r);
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
// TMEM columns: [0, 256) two score buffers (S^T 64 | dP^T 64, fp32);
// [256, 384) two operand buffers (P^T 32 | dS^T 32, bf16 pairs of the 64
// sub-tile queries); [384, 512) the accumulators dV 64 | dK 64.
constexpr int kQStages = 3;
constexpr int kSub = 64;  // queries per sub-tile
constexpr uint32_t kOpCol = 256;
constexpr uint32_t kAccColKV = 384;
constexpr int kPairBytes = kTile * 8;  // -L log2e [128], then D [128], of one query tile
constexpr int kOutBoxKV = 32 * (kHD / kKvSplit) * 2 * 2;  // a compute warp's dK and dV slots: 32 rows each
constexpr size_t dkdv_smem_bytes() {
  // [K, V] x 2 items, [Q, dO] x stages, (L, D) pairs x stages, the compute
  // warps' dK / dV boxes, aux
  return 1024 + 4 * (size_t)kBox + 2 * (size_t)kQStages * kBox + (size_t)kQStages * kPairBytes +
         (kCTkv / 32) * (size_t)kOutBoxKV + kAux;
}

__global__ void __launch_bounds__(kThreadsKV, 1)
    flash_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                             const __grid_constant__ CUtensorMap tmDO,
                             const __grid_constant__ CUtensorMap tmDKV,
                             const float2* __restrict__ pairs, int B, int T, int C, int H,
                             float sl2, float scale, int* err) {
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sKV = smem;                    // [2 items][K box, V box]
  uint8_t* sQ = sKV + 4 * kBox;           // [kQStages]
  uint8_t* sDO = sQ + kQStages * kBox;    // [kQStages]
  uint8_t* sLD = sDO + kQStages * kBox;   // [kQStages][-L log2e x 128, D x 128]
  uint8_t* sOut = sLD + kQStages * kPairBytes;  // [compute warp][dK box, dV box]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + (kCTkv / 32) * kOutBoxKV);
  const uint32_t kv_full0 = smem_u32(bars + 0);     // [2]
  const uint32_t kv_empty0 = smem_u32(bars + 2);    // [2]
  const uint32_t qd_full0 = smem_u32(bars + 4);     // [kQStages]
  const uint32_t qd_empty0 = smem_u32(bars + 4 + kQStages);   // [kQStages]
  const uint32_t sd_full0 = smem_u32(bars + 4 + 2 * kQStages);   // [2]
  const uint32_t sd_empty0 = sd_full0 + 16;         // [2]
  const uint32_t pd_full0 = sd_full0 + 32;          // [2]
  const uint32_t pd_empty0 = sd_full0 + 48;         // [2]
  const uint32_t acc_full = sd_full0 + 64;
  const uint32_t acc_empty = sd_full0 + 72;
  const uint32_t drain0 = sd_full0 + 80;  // [2] abort path only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 + 2 * kQStages + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int nq = (T + kTile - 1) / kTile;
  const int Tp = nq * kTile;
  const int BH = B * H, items = nq * BH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 1);
      mbar_init(sd_full0 + 8 * s, 1);
      mbar_init(sd_empty0 + 8 * s, kCTkv);
      mbar_init(pd_full0 + 8 * s, kCTkv);
      mbar_init(pd_empty0 + 8 * s, 1);
    }
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(qd_full0 + 8 * s, 1);
      mbar_init(qd_empty0 + 8 * s, 2);  // the scores and the products read Q and dO
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kCTkv);
    mbar_init(drain0, 1);
    mbar_init(drain0 + 8, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // set-up done; the inputs written by the previous kernels are complete from here on

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
          const int st = g % kQStages;
          const uint32_t par = (g / kQStages) & 1u;
          if (!mbar_wait(qd_empty0 + 8 * st, par ^ 1u, abort_flag, err)) {
            ok = false;
            break;
          }
          const uint32_t fb = qd_full0 + 8 * st;
          mbar_expect_tx(fb, 2 * kBox + kPairBytes);
          tma_load_3d(smem_u32(sQ + st * kBox), &tmQKV, fb, h * kHD, (j + t) * kTile, b);
          tma_load_3d(smem_u32(sDO + st * kBox), &tmDO, fb, h * kHD, (j + t) * kTile, b);
          bulk_load_1d(smem_u32(sLD + st * kPairBytes),
                       pairs + (size_t)bh * Tp + (size_t)(j + t) * kTile, kPairBytes, fb);
          issued |= 1u << st;
          last_par = (last_par & ~(1u << st)) | (par << st);
        }
      }
      // every copy issued lands before the shared memory is released
      const uint64_t t0 = global_ns();
      for (int s = 0; s < 2; ++s)
        if (kv_issued & (1u << s)) drain_wait(kv_full0 + 8 * s, (kv_par >> s) & 1u, t0);
      for (int s = 0; s < kQStages; ++s)
        if (issued & (1u << s)) drain_wait(qd_full0 + 8 * s, (last_par >> s) & 1u, t0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------- MMA: scores --
      // S^T = K Q_s^T and dP^T = V dO_s^T of sub-tile s (half hs of the
      // query tile in stage st) into score buffer s % 2.  The products run
      // from their own warp, so the scores of the next sub-tiles never wait
      // behind them.
      constexpr uint32_t idS = attn::idesc(kSub, false);
      uint32_t n_item = 0, gs = 0, gt = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++n_item) {
        const int w = snake_item(k, items);
        if (w < 0) break;
        const int n = nq - w / BH;
        const int ks = n_item & 1;
        ok = mbar_wait(kv_full0 + 8 * ks, (n_item >> 1) & 1u, abort_flag, err);
        if (!ok) break;
        const uint32_t k_base = smem_u32(sKV + ks * 2 * kBox), v_base = k_base + kBox;
        for (int t = 0; t < n && ok; ++t, ++gt) {
          const int st = gt % kQStages;
          ok = mbar_wait(qd_full0 + 8 * st, (gt / kQStages) & 1u, abort_flag, err);
          for (int hs = 0; hs < 2 && ok; ++hs, ++gs) {
            const uint32_t sb = gs & 1u;
            ok = mbar_wait(sd_empty0 + 8 * sb, ((gs >> 1) & 1u) ^ 1u, abort_flag, err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t q_base = smem_u32(sQ + st * kBox) + hs * (kSub * 128);
            const uint32_t do_base = smem_u32(sDO + st * kBox) + hs * (kSub * 128);
            const uint32_t d = tmem + sb * 2 * kSub;
#pragma unroll
            for (int kk = 0; kk < kHD / 16; ++kk)
              tc_mma(d, desc_kmajor(k_base, kk), desc_kmajor(q_base, kk), idS, kk > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < kHD / 16; ++kk)
              tc_mma(d + kSub, desc_kmajor(v_base, kk), desc_kmajor(do_base, kk), idS,
                     kk > 0 ? 1u : 0u);
            tc_commit(sd_full0 + 8 * sb);
            if (hs == 1) tc_commit(qd_empty0 + 8 * st);  // the scores are done with Q, dO
          }
        }
        if (ok) tc_commit(kv_empty0 + 8 * ks);  // K, V no longer read
      }
      if (!ok) {  // let issued MMAs finish before TMEM is released
        tc_commit(drain0);
        drain_wait(drain0, 0, global_ns());
      }
    }
  } else if (warp == kMma2KV) {
    if (lane == 0) {
      // ------------------------------------------------ MMA: products --
      // dV += P^T dO_s, dK += dS^T Q_s of each sub-tile once its P^T and
      // dS^T are in TMEM; the accumulators go to the compute warps after the
      // item's last sub-tile.
      constexpr uint32_t idA = attn::idesc(kHD, true);
      uint32_t n_item = 0, gs = 0, gt = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++n_item) {
        const int w = snake_item(k, items);
        if (w < 0) break;
        const int n = nq - w / BH;
        // the previous item's dV and dK have been read out
        ok = mbar_wait(acc_empty, (n_item & 1u) ^ 1u, abort_flag, err);
        for (int t = 0; t < n && ok; ++t, ++gt) {
          const int st = gt % kQStages;
          ok = mbar_wait(qd_full0 + 8 * st, (gt / kQStages) & 1u, abort_flag, err);
          const uint32_t q_base = smem_u32(sQ + st * kBox), do_base = smem_u32(sDO + st * kBox);
          for (int hs = 0; hs < 2 && ok; ++hs, ++gs) {
            const uint32_t sb = gs & 1u;
            ok = mbar_wait(pd_full0 + 8 * sb, (gs >> 1) & 1u, abort_flag, err);
            if (!ok) break;
            tc_fence_after();
            const bool first = t == 0 && hs == 0;
            const uint32_t pt = tmem + kOpCol + sb * kSub, dst = pt + kSub / 2;
#pragma unroll
            for (int kk = 0; kk < kSub / 16; ++kk)
              attn::tc_mma_ts(tmem + kAccColKV, pt + (uint32_t)(8 * kk),
                              desc_mnmajor(do_base, 4 * hs + kk), idA, (!first || kk > 0) ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < kSub / 16; ++kk)
              attn::tc_mma_ts(tmem + kAccColKV + kHD, dst + (uint32_t)(8 * kk),
                              desc_mnmajor(q_base, 4 * hs + kk), idA, (!first || kk > 0) ? 1u : 0u);
            tc_commit(pd_empty0 + 8 * sb);
            if (hs == 1) tc_commit(qd_empty0 + 8 * st);  // the products are done with Q, dO
          }
        }
        if (ok) tc_commit(acc_full);
      }
      if (!ok) {
        tc_commit(drain0 + 8);
        drain_wait(drain0 + 8, 0, global_ns());
      }
    }
  } else {
    // -------------------------------------------------------- compute --
    // thread = key row r, owning kColsKV of a sub-tile's 64 query columns
    // (slot `part` of the row).  Every wait is per warp (warps drift apart
    // and overlap their latencies).
    const int qw = warp & 3, part = (warp - 2) >> 2;
    const int r = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    uint32_t n_item = 0, gs = 0, gt = 0;
    bool ok = true;
    // An item's dV and dK are read out of TMEM after the next item's first
    // sub-tile has been handed to the products warp, which by then has
    // finished the item's last products; the next item's products wait for
    // the read-out (one accumulator pair).
    struct PendingKV {
      uint32_t n_item;
      int b, h, j;
      bool live;
    };
    PendingKV pend{0, 0, 0, 0, false};
    auto read_out = [&](const PendingKV& it) {
      // this thread's 64 / kKvSplit columns of each
      if (!warp_and(mbar_wait(acc_full, it.n_item & 1u, abort_flag, err))) return false;
      tc_fence_after();
      constexpr int kAccCols = kHD / kKvSplit;
      uint32_t rv[kAccCols], rk[kAccCols];
      tc_ldn<kAccCols>(lane_base + kAccColKV + kAccCols * part, rv);
      tc_ldn<kAccCols>(lane_base + kAccColKV + kHD + kAccCols * part, rk);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(acc_empty);
      // this warp's 32 rows x kAccCols columns of dK and of dV into its two
      // boxes, out by one TMA store each (rows past T are clipped)
      constexpr int kRowBytes = kAccCols * 2;
      uint8_t* box_k = sOut + (warp - 2) * kOutBoxKV;
      uint8_t* box_v = box_k + 32 * kRowBytes;
      if (lane == 0) bulk_wait_read<0>();  // the boxes' previous stores have read them
      __syncwarp();
#pragma unroll
      for (int q = 0; q < kAccCols; q += 8) {
        uint4 wk, wv;
        uint32_t* pk4 = reinterpret_cast<uint32_t*>(&wk);
        uint32_t* pv4 = reinterpret_cast<uint32_t*>(&wv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pk4[e] = attn::pack_bf16x2(__uint_as_float(rk[q + 2 * e]) * scale,
                                     __uint_as_float(rk[q + 2 * e + 1]) * scale);
          pv4[e] = attn::pack_bf16x2(__uint_as_float(rv[q + 2 * e]),
                                     __uint_as_float(rv[q + 2 * e + 1]));
        }
        *reinterpret_cast<uint4*>(box_k + lane * kRowBytes + q * 2) = wk;
        *reinterpret_cast<uint4*>(box_v + lane * kRowBytes + q * 2) = wv;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int x0 = it.h * kHD + kAccCols * part, y0 = it.j * kTile + qw * 32;
        tma_store_3d(&tmDKV, smem_u32(box_k), C + x0, y0, it.b);
        tma_store_3d(&tmDKV, smem_u32(box_v), 2 * C + x0, y0, it.b);
        bulk_commit();
      }
      return true;
    };
    for (int k = 0; ok; ++k, ++n_item) {
      const int w = snake_item(k, items);
      if (w < 0) break;
      const int j = w / BH, bh = w % BH, b = bh / H, h = bh % H;
      const int n = nq - j;
      for (int t = 0; t < n && ok; ++t, ++gt) {
        const int st = gt % kQStages;
        const float* ldq = reinterpret_cast<const float*>(sLD + st * kPairBytes);
        for (int hs = 0; hs < 2; ++hs, ++gs) {
          const uint32_t sb = gs & 1u;
          const int cq = kSub * hs + kColsKV * part;  // first query column of this thread in the tile
          ok = warp_and(mbar_wait(sd_full0 + 8 * sb, (gs >> 1) & 1u, abort_flag, err));
          if (!ok) break;
          tc_fence_after();
          uint32_t sr[kColsKV], dp[kColsKV];
          tc_ldn<kColsKV>(lane_base + sb * 2 * kSub + kColsKV * part, sr);
          tc_ldn<kColsKV>(lane_base + sb * 2 * kSub + kSub + kColsKV * part, dp);
          tc_wait_ld();
          tc_fence_before();
          mbar_arrive(sd_empty0 + 8 * sb);  // the scores are read: sub-tile gs + 2 may be computed
          if (t == 0) {  // the diagonal tile: queries before the key are masked
#pragma unroll
            for (int c = 0; c < kColsKV; ++c)
              if (cq + c < r) sr[c] = kNegInf;
          }
          uint32_t pk[kColsKV / 2], dk[kColsKV / 2];
#pragma unroll
          for (int c = 0; c < kColsKV; c += 4) {
            // -L log2e and D of queries cq + c .. cq + c + 3 (query-tile stage st)
            const float4 nl = *reinterpret_cast<const float4*>(ldq + cq + c);
            const float4 dd = *reinterpret_cast<const float4*>(ldq + kTile + cq + c);
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              float2 p = f2_fma(make_float2(__uint_as_float(sr[c + e]), __uint_as_float(sr[c + e + 1])),
                                f2_splat(sl2), e ? make_float2(nl.z, nl.w) : make_float2(nl.x, nl.y));
              p = make_float2(fast_exp2(p.x), fast_exp2(p.y));
              const float2 ds = f2_mul(
                  p, f2_sub(make_float2(__uint_as_float(dp[c + e]), __uint_as_float(dp[c + e + 1])),
                            e ? make_float2(dd.z, dd.w) : make_float2(dd.x, dd.y)));
              pk[(c + e) / 2] = attn::pack_bf16x2(p.x, p.y);
              dk[(c + e) / 2] = attn::pack_bf16x2(ds.x, ds.y);
            }
          }
          // the products of sub-tile gs - 2 have read this operand buffer
          ok = warp_and(mbar_wait(pd_empty0 + 8 * sb, ((gs >> 1) & 1u) ^ 1u, abort_flag, err));
          if (!ok) break;
          tc_fence_after();
          const uint32_t op = lane_base + kOpCol + sb * kSub + (kColsKV / 2) * part;
          tc_stn<kColsKV / 2>(op, pk);
          tc_stn<kColsKV / 2>(op + kSub / 2, dk);
          attn::tc_wait_st();
          tc_fence_before();
          mbar_arrive(pd_full0 + 8 * sb);
          if (pend.live) {  // the previous item's dV and dK, after this item's first sub-tile
            ok = read_out(pend);
            pend.live = false;
            if (!ok) break;
          }
        }
      }
      if (!ok) break;
      pend = PendingKV{n_item, b, h, j, true};
    }
    if (ok && pend.live) ok = read_out(pend);
    if (lane == 0) bulk_wait_all();  // the dK / dV stores complete before the CTA leaves
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem);
}

// --------------------------------------------------------------------- dQ --
// TMEM columns: [0, 128) S, [128, 256) dP (fp32); [256, 384) two dS buffers
// (bf16 pairs of 128 keys); [384, 512) two dQ accumulators.
constexpr int kKVStages = 3;
constexpr uint32_t kDSCol = 256;
constexpr uint32_t kAccColQ = 384;
constexpr int kOutBoxQ = 32 * 32 * 2;  // a compute warp's dQ slot: 32 rows x 32 columns
constexpr size_t dq_smem_bytes() {
  // [Q, dO, O] x 2 items, [K, V] x stages, the compute warps' dQ boxes, aux
  return 1024 + 6 * (size_t)kBox + 2 * (size_t)kKVStages * kBox + (kCTq / 32) * (size_t)kOutBoxQ +
         kAux;
}

__global__ void __launch_bounds__(kThreadsQ, 1)
    flash_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                           const __grid_constant__ CUtensorMap tmDO,
                           const __grid_constant__ CUtensorMap tmO, const float* __restrict__ lse,
                           const __grid_constant__ CUtensorMap tmDQ, float2* __restrict__ pairs,
                           int B, int T, int C, int H, float sl2, float scale, int* err) {
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // Q, dO and O (the forward's output rows, for D) of two items: the next
  // item's tiles arrive while the current one runs
  uint8_t* sQ0 = smem;                     // [2 items][Q, dO, O]
  uint8_t* sK = sQ0 + 6 * kBox;            // [kKVStages]
  uint8_t* sV = sK + kKVStages * kBox;     // [kKVStages]
  uint8_t* sOut = sV + kKVStages * kBox;   // [compute warp][kOutBoxQ]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + (kCTq / 32) * kOutBoxQ);
  const uint32_t qd_full0 = smem_u32(bars + 0);             // [2 items]
  const uint32_t qd_empty0 = smem_u32(bars + 2);            // [2 items]
  const uint32_t kv_full0 = smem_u32(bars + 4);              // [kKVStages]
  const uint32_t kv_empty0 = smem_u32(bars + 4 + kKVStages); // [kKVStages]
  const uint32_t sd_full = smem_u32(bars + 4 + 2 * kKVStages);
  const uint32_t sd_empty = sd_full + 8;
  const uint32_t ds_full0 = sd_full + 16;                    // [2]
  const uint32_t ds_empty0 = sd_full + 32;                   // [2]
  const uint32_t acc_full0 = sd_full + 48;                   // [2]
  const uint32_t acc_empty0 = sd_full + 64;                  // [2]
  const uint32_t drain0 = sd_full + 80;                      // [2] abort path only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 + 2 * kKVStages + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int nq = (T + kTile - 1) / kTile;
  const int Tp = nq * kTile;
  const int BH = B * H, items = nq * BH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(qd_full0 + 8 * s, 1);
      mbar_init(qd_empty0 + 8 * s, 1 + kCTq);  // the last S/dP product, and every compute thread's D
    }
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 2);  // the scores read K, V; the products K
    }
    mbar_init(sd_full, 1);
    mbar_init(sd_empty, kCTq);
    for (int s = 0; s < 2; ++s) {
      mbar_init(ds_full0 + 8 * s, kCTq);
      mbar_init(ds_empty0 + 8 * s, 1);
      mbar_init(acc_full0 + 8 * s, 1);
      mbar_init(acc_empty0 + 8 * s, kCTq);
      mbar_init(drain0 + 8 * s, 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // set-up done; the inputs written by the previous kernels are complete from here on

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
        const uint32_t qb = n_item & 1u, qfb = qd_full0 + 8 * qb;
        if (!mbar_wait(qd_empty0 + 8 * qb, ((n_item >> 1) & 1u) ^ 1u, abort_flag, err)) break;
        uint8_t* sq = sQ0 + qb * 3 * kBox;
        mbar_expect_tx(qfb, 3 * kBox);
        tma_load_3d(smem_u32(sq), &tmQKV, qfb, h * kHD, i * kTile, b);
        tma_load_3d(smem_u32(sq + kBox), &tmDO, qfb, h * kHD, i * kTile, b);
        tma_load_3d(smem_u32(sq + 2 * kBox), &tmO, qfb, h * kHD, i * kTile, b);
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
      for (uint32_t m = n_item > 2 ? n_item - 2 : 0; m < n_item; ++m)
        drain_wait(qd_full0 + 8 * (m & 1u), (m >> 1) & 1u, t0);
      for (int s = 0; s < kKVStages; ++s)
        if (issued & (1u << s)) drain_wait(kv_full0 + 8 * s, (last_par >> s) & 1u, t0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------- MMA: scores --
      // S = Q K_j^T and dP = dO V_j^T for every key tile j of every item;
      // the dQ products run from their own warp.
      constexpr uint32_t idS = attn::idesc(kTile, false);
      uint32_t n_item = 0, gk = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++n_item) {
        const int w = snake_item(k, items);
        if (w < 0) break;
        const int n = nq - w / BH;  // i + 1
        const uint32_t qb = n_item & 1u;
        const uint32_t q_base = smem_u32(sQ0 + qb * 3 * kBox), do_base = q_base + kBox;
        ok = mbar_wait(qd_full0 + 8 * qb, (n_item >> 1) & 1u, abort_flag, err);
        for (int jj = 0; jj < n && ok; ++jj) {
          const uint32_t gg = gk + jj;
          const int st = gg % kKVStages;
          ok = mbar_wait(kv_full0 + 8 * st, (gg / kKVStages) & 1u, abort_flag, err);
          if (ok) ok = mbar_wait(sd_empty, (gg & 1u) ^ 1u, abort_flag, err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t k_base = smem_u32(sK + st * kBox), v_base = smem_u32(sV + st * kBox);
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk)  // S = Q K^T
            tc_mma(tmem, desc_kmajor(q_base, kk), desc_kmajor(k_base, kk), idS, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk)  // dP = dO V^T
            tc_mma(tmem + kTile, desc_kmajor(do_base, kk), desc_kmajor(v_base, kk), idS,
                   kk > 0 ? 1u : 0u);
          tc_commit(sd_full);
          tc_commit(kv_empty0 + 8 * st);  // the scores are done with K_j, V_j
          if (jj == n - 1) tc_commit(qd_empty0 + 8 * qb);  // Q and dO are no longer read
        }
        gk += n;
      }
      if (!ok) {
        tc_commit(drain0);
        drain_wait(drain0, 0, global_ns());
      }
    }
  } else if (warp == kMma2Q) {
    if (lane == 0) {
      // ------------------------------------------------ MMA: products --
      // dQ (+)= dS_j K_j (dS from TMEM) into the item's accumulator.
      constexpr uint32_t idQ = attn::idesc(kHD, true);
      uint32_t n_item = 0, gk = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++n_item) {
        const int w = snake_item(k, items);
        if (w < 0) break;
        const int n = nq - w / BH;
        const uint32_t ab = n_item & 1u, acc = kAccColQ + ab * kHD;
        ok = mbar_wait(acc_empty0 + 8 * ab, ((n_item >> 1) & 1u) ^ 1u, abort_flag, err);
        for (int jj = 0; jj < n && ok; ++jj) {
          const uint32_t gg = gk + jj;
          const int st = gg % kKVStages, db = gg & 1;
          ok = mbar_wait(kv_full0 + 8 * st, (gg / kKVStages) & 1u, abort_flag, err);
          if (ok) ok = mbar_wait(ds_full0 + 8 * db, (gg >> 1) & 1u, abort_flag, err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t ds = tmem + kDSCol + (uint32_t)(db * kHD), k_base = smem_u32(sK + st * kBox);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            attn::tc_mma_ts(tmem + acc, ds + (uint32_t)(8 * kk), desc_mnmajor(k_base, kk), idQ,
                            (jj > 0 || kk > 0) ? 1u : 0u);
          tc_commit(ds_empty0 + 8 * db);
          tc_commit(kv_empty0 + 8 * st);  // the products are done with K_j
        }
        if (ok) tc_commit(acc_full0 + 8 * ab);
        gk += n;
      }
      if (!ok) {
        tc_commit(drain0 + 8);
        drain_wait(drain0 + 8, 0, global_ns());
      }
    }
  } else {
    // -------------------------------------------------------- compute --
    // thread = query row r, owning kColsQ of a key tile's 128 columns (slot
    // `part` of the row)
    const int qw = warp & 3, part = (warp - 2) >> 2;
    const int r = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    uint32_t n_item = 0, gk = 0;
    bool ok = true;
    // this row's L of an item, loaded one item ahead (the load's latency
    // would otherwise sit at the start of every item)
    auto row_lse = [&](int k) {
      const int w = snake_item(k, items);
      if (w < 0) return 0.f;
      const int qi = (nq - 1 - w / BH) * kTile + r;
      return qi < T ? lse[(size_t)(w % BH) * T + qi] : 0.f;
    };
    float lse_next = row_lse(0);
    // An item's dQ is read out of its TMEM accumulator (there are two) after
    // the first key tile of the next item, by when its last products have
    // finished, so the compute warps do not wait for them at the item's end.
    struct PendingDQ {
      uint32_t n_item;
      int b, h, i;
      bool live;
    };
    PendingDQ pend{0, 0, 0, 0, false};
    auto read_out = [&](const PendingDQ& it) {
      const uint32_t ab = it.n_item & 1u, acc = kAccColQ + ab * kHD;
      if (!warp_and(mbar_wait(acc_full0 + 8 * ab, (it.n_item >> 1) & 1u, abort_flag, err)))
        return false;
      tc_fence_after();
      constexpr int kAccCols = kHD / kQSplit;
      uint32_t rq[kAccCols];
      tc_ldn<kAccCols>(lane_base + acc + kAccCols * part, rq);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(acc_empty0 + 8 * ab);
      // this warp's 32 rows x kAccCols columns of dQ into its box, out by
      // one TMA store (rows past T are clipped by the tensor map)
      static_assert(kAccCols == 32, "one 64-byte box row per thread");
      uint8_t* box = sOut + (warp - 2) * kOutBoxQ;
      if (lane == 0) bulk_wait_read<0>();  // the box's previous store has read it
      __syncwarp();
#pragma unroll
      for (int q = 0; q < kAccCols; q += 8) {
        uint4 w;
        uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          wp[e] = attn::pack_bf16x2(__uint_as_float(rq[q + 2 * e]) * scale,
                                    __uint_as_float(rq[q + 2 * e + 1]) * scale);
        *reinterpret_cast<uint4*>(box + lane * 64 + q * 2) = w;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(&tmDQ, smem_u32(box), it.h * kHD + kAccCols * part, it.i * kTile + qw * 32,
                     it.b);
        bulk_commit();
      }
      return true;
    };
    for (int k = 0; ok; ++k, ++n_item) {
      const int w = snake_item(k, items);
      if (w < 0) break;
      const int i = nq - 1 - w / BH, bh = w % BH, b = bh / H, h = bh % H;
      const int n = i + 1;
      const int qi = i * kTile + r;  // this thread's query row
      const float lse2 = lse_next * kLog2e;
      lse_next = row_lse(k + 1);
      // D = rowsum(dO * O) of this row from the item's dO and O tiles (rows
      // past T are zero-filled; every thread of the row forms it); stored
      // with L for the dK/dV kernel
      const uint32_t qb = n_item & 1u;
      ok = warp_and(mbar_wait(qd_full0 + 8 * qb, (n_item >> 1) & 1u, abort_flag, err));
      if (!ok) break;
      const uint8_t* sDO = sQ0 + qb * 3 * kBox + kBox;
      const uint8_t* sO = sDO + kBox;
      float drow = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float a[8], o[8];
        load8(reinterpret_cast<const __nv_bfloat16*>(sDO + swz(r, c)), a);
        load8(reinterpret_cast<const __nv_bfloat16*>(sO + swz(r, c)), o);
#pragma unroll
        for (int e = 0; e < 8; ++e) drow = fmaf(a[e], o[e], drow);
      }
      mbar_arrive(qd_empty0 + 8 * qb);  // this thread is done with dO and O
      if (part == 0) {  // the query tile's 128 values of -L log2e, then its 128 values of D
        float* ld = reinterpret_cast<float*>(pairs + (size_t)bh * Tp + (size_t)i * kTile);
        ld[r] = qi < T ? -lse2 : -INFINITY;
        ld[kTile + r] = qi < T ? drow : 0.f;
      }
      for (int jj = 0; jj < n && ok; ++jj) {
        const uint32_t gg = gk + jj;
        const int db = gg & 1;
        ok = warp_and(mbar_wait(sd_full, gg & 1u, abort_flag, err));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[kColsQ], dp[kColsQ];
#pragma unroll
        for (int c = 0; c < kColsQ; c += 32) {
          tc_ld32(lane_base + kColsQ * part + c, sr + c);
          tc_ld32(lane_base + kTile + kColsQ * part + c, dp + c);
        }
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(sd_empty);  // S and dP are read: the next key tile's may be computed
        if (jj == i) {  // the diagonal tile: keys after the query are masked
#pragma unroll
          for (int c = 0; c < kColsQ; ++c)
            if (kColsQ * part + c > r) sr[c] = kNegInf;
        }
        uint32_t dk[kColsQ / 2];
#pragma unroll
        for (int c = 0; c < kColsQ; c += 2) {
          float2 p = f2_fma(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                            f2_splat(sl2), f2_splat(-lse2));
          p = make_float2(fast_exp2(p.x), fast_exp2(p.y));
          const float2 ds = f2_mul(
              p, f2_sub(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), f2_splat(drow)));
          dk[c / 2] = attn::pack_bf16x2(ds.x, ds.y);
        }
        // the product two tiles back has read this dS buffer
        ok = warp_and(mbar_wait(ds_empty0 + 8 * db, ((gg >> 1) & 1u) ^ 1u, abort_flag, err));
        if (!ok) break;
        tc_fence_after();
        tc_stn<kColsQ / 2>(lane_base + kDSCol + (uint32_t)(db * kHD) + (kColsQ / 2) * part, dk);
        attn::tc_wait_st();
        tc_fence_before();
        mbar_arrive(ds_full0 + 8 * db);
        if (jj == 0 && pend.live) {  // the previous item's dQ
          ok = read_out(pend);
          pend.live = false;
        }
      }
      if (!ok) break;
      pend = PendingDQ{n_item, b, h, i, true};
      gk += n;
    }
    if (ok && pend.live) ok = read_out(pend);
    if (lane == 0) bulk_wait_all();  // the dQ stores complete before the CTA leaves
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem);
}

}  // namespace

size_t attention_bwd_tc_scratch_floats(int B, int T, int H) {
  const size_t Tp = (size_t)(T + kTile - 1) / kTile * kTile;
  return 2 * (size_t)B * H * Tp;
}

cudaError_t attention_bwd_tc(act_t* dqkv, float* scratch, const act_t* datt, const act_t* qkv,
                             const act_t* att, const float* lse, int B, int T, int C, int H,
                             int* err, cudaStream_t s) {
  if (C / H != kHD || (reinterpret_cast<uintptr_t>(qkv) & 15) ||
      (reinterpret_cast<uintptr_t>(datt) & 15) || (reinterpret_cast<uintptr_t>(att) & 15) ||
      (reinterpret_cast<uintptr_t>(scratch) & 15))
    return cudaErrorInvalidValue;
  CUtensorMap tq, td, to, tdq, tdkv;
  cudaError_t e = attn::seq_map(&tq, qkv, B, T, 3 * C);
  if (e != cudaSuccess) return e;
  e = attn::seq_map(&td, datt, B, T, C);
  if (e != cudaSuccess) return e;
  e = attn::seq_map(&to, att, B, T, C);
  if (e != cudaSuccess) return e;
  // the gradients leave through per-warp boxes: 32 rows of 32 (dQ) or
  // kColsKV (dK, dV) columns, no swizzle
  e = attn::seq_map(&tdq, dqkv, B, T, 3 * C, 32, 32, false);
  if (e != cudaSuccess) return e;
  e = attn::seq_map(&tdkv, dqkv, B, T, 3 * C, 32, kHD / kKvSplit, false);
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
  float2* pairs = reinterpret_cast<float2*>(scratch);
  // dQ first: it forms D = rowsum(dO * O) of its query tiles and stores the
  // (L, D) pairs for dK/dV
  launch_kernel(flash_bwd_dq_tc_kernel, grid, kThreadsQ, sm_b, s, tq, td, to, lse, tdq, pairs, B, T,
                C, H, sl2, scale, err);
  launch_kernel(flash_bwd_dkdv_tc_kernel, grid, kThreadsKV, sm_a, s, tq, td, tdkv, pairs, B, T, C,
                H, sl2, scale, err);
  note_launch(2);
  return cudaGetLastError();
}

}  // namespace gpt2k
