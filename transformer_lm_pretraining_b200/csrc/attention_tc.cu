// Causal flash-attention forward on the sm_100a tensor cores (head dim 64).
//
// Persistent: one CTA per SM walks a static list of work items, each a pair
// of adjacent 128-row query tiles (A = 2p, B = 2p + 1) of one (batch, head).
// Items are ordered heaviest first and dealt to the CTAs in a snake order,
// which balances the causal work across SMs.  11 warps:
//   warp 0     TMA: the item's two Q tiles, then its K/V tiles of 128 keys
//              into a 4-stage ring (128-byte swizzle, zero fill past the
//              sequence), running ahead into the next item;
//   warps 1, 10  MMA issuers of tiles A and B (warp 1 also owns TMEM):
//              S_t = Q_t K_j^T (M=128, N=128,
//              K=64) into one TMEM buffer per tile t, and O_t += P_t V_j
//              (M=128, N=64, K=128) with P_t read from TMEM as the A operand
//              and V read MN-major from its shared-memory tile; O_t
//              accumulates in TMEM over the item's key tiles.  S for key
//              tile j+1 is issued before PV for key tile j;
//   warps 2-5  softmax of tile A, warps 6-9 softmax of tile B: one thread
//              per query row.  A thread loads its whole row of S from TMEM
//              into registers at once and hands the buffer straight back (so
//              the next S is computed while this one is exponentiated),
//              takes the row max, forms P = 2^(S log2e / sqrt(d) - m) and
//              writes it as packed bf16 into its tile's P columns of TMEM.
//              The reference max m is raised only when a tile's max exceeds
//              it by more than 2^8 (P stays below 256); then the row of O in
//              TMEM and the running sum are rescaled first.  No thread waits
//              for another thread's row.
// T x T is never materialised.  The output row is normalised by the
// running sum and written into the softmax warp's own 32-row shared-memory
// box, which one TMA store per warp sends out (measured: 70.7 -> 62.6 us at
// B16 x T1024 x H12 against per-thread 16-byte stores of each row, which left
// every lane writing to a different row); the natural-log log-sum-exp of each
// row is stored for the backward pass.  Every wait is bounded (error word
// ERR_TIMEOUT).
//
// TMEM columns: [0, 256) S_A | S_B (fp32), [256, 384) O_A | O_B (fp32),
// [384, 512) P_A | P_B (128 keys as 64 columns of bf16 pairs).
// Softmax threads per row: one.  Two (the row max and sum exchanged through
// shared memory) measured 78.5 vs 70.5 us, and a split of each row into key
// halves with their own accumulators 90.3 us.

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
using attn::kTile;

constexpr int kKVStages = 4;
constexpr int kRowThreads = 128;  // softmax threads per query tile (one per row)
constexpr int kThreadsAttn = 64 + 2 * kRowThreads + 32;  // + the MMA warp of tile B
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 2 * kTile;         // O_t at kOCol + t * kHD
constexpr uint32_t kPCol = kOCol + 2 * kHD;   // P_t at kPCol + t * kHD (bf16 pairs)
constexpr float kRescaleLog2 = 8.0f;  // raise the reference max past this margin
constexpr int kAux = 1024;  // barriers
constexpr uint32_t kNegInf = 0xff800000u;

constexpr int kOutBox = 4096;  // one softmax warp's output rows: 32 x 64 bf16, 128-byte swizzle

constexpr size_t attn_smem_bytes() {
  // Q (two tiles), K ring, V ring, the eight softmax warps' output boxes, aux
  return 1024 + 2 * (size_t)kBox + 2 * (size_t)kKVStages * kBox + 8 * (size_t)kOutBox + kAux;
}

// Work item k of this CTA (snake order over the heaviest-first item list);
// false when the CTA has no item k.
struct FwdItem {
  int b, h, qa, qb, nkv_a, nkv_b;  // nkv_b = 0: no tile B
};
__device__ __forceinline__ bool fwd_item(int k, int B, int H, int nq, FwdItem& it) {
  const int G = gridDim.x;
  const int w = k * G + ((k & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
  const int BH = B * H;
  const int npairs = (nq + 1) >> 1;
  if (w >= npairs * BH) return false;
  const int p = npairs - 1 - w / BH, bh = w % BH;
  it.b = bh / H;
  it.h = bh % H;
  it.qa = 2 * p;
  it.qb = 2 * p + 1;
  it.nkv_a = it.qa + 1;
  it.nkv_b = it.qb < nq ? it.qb + 1 : 0;
  return true;
}

__global__ void __launch_bounds__(kThreadsAttn, 1)
    flash_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                        const __grid_constant__ CUtensorMap tmOut, float* __restrict__ lse, int B,
                        int T, int C, int H, float sl2, int* err) {
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                           // [2 tiles][kBox]
  uint8_t* sK = sQ + 2 * kBox;                  // [kKVStages][kBox]
  uint8_t* sV = sK + kKVStages * kBox;          // [kKVStages][kBox]
  uint8_t* sOut = sV + kKVStages * kBox;        // [2 tiles][4 lane quarters][kOutBox]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + 8 * kOutBox);
  const uint32_t q_full = smem_u32(bars + 0);
  const uint32_t q_empty = smem_u32(bars + 1);
  const uint32_t kv_full0 = smem_u32(bars + 2);                  // [kKVStages]
  const uint32_t kv_empty0 = smem_u32(bars + 2 + kKVStages);     // [kKVStages]
  const uint32_t s_full0 = smem_u32(bars + 2 + 2 * kKVStages);   // [2 tiles]
  const uint32_t s_empty0 = s_full0 + 16;                        // [2 tiles]
  const uint32_t p_full0 = s_full0 + 32;                         // [2 tiles]
  const uint32_t o_full0 = s_full0 + 48;                         // [2 tiles]
  const uint32_t drain0 = s_full0 + 64;                          // [2 tiles] abort path only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 + 2 * kKVStages + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int nq = (T + kTile - 1) / kTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 2);  // both MMA warps
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 2);  // both MMA warps
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full0 + 8 * t, 1);
      mbar_init(s_empty0 + 8 * t, kRowThreads);
      mbar_init(p_full0 + 8 * t, kRowThreads);
      mbar_init(o_full0 + 8 * t, 1);
      mbar_init(drain0 + 8 * t, 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // TMEM owner
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // set-up done; the inputs written by the previous kernels are complete from here on

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA --
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQKV)) : "memory");
      uint32_t n_item = 0, q_issued = 0;
      uint32_t g = 0;  // K/V tiles loaded so far (ring position)
      uint32_t issued = 0, last_parity = 0;
      bool ok = true;
      FwdItem it;
      for (int k = 0; ok && fwd_item(k, B, H, nq, it); ++k, ++n_item) {
        if (!mbar_wait(q_empty, (n_item & 1u) ^ 1u, abort_flag, err)) break;
        mbar_expect_tx(q_full, it.nkv_b ? 2 * kBox : kBox);
        tma_load_3d(smem_u32(sQ), &tmQKV, q_full, it.h * kHD, it.qa * kTile, it.b);
        if (it.nkv_b) tma_load_3d(smem_u32(sQ + kBox), &tmQKV, q_full, it.h * kHD, it.qb * kTile, it.b);
        q_issued = n_item + 1;
        const int nkv = it.nkv_b ? it.nkv_b : it.nkv_a;
        for (int j = 0; j < nkv; ++j, ++g) {
          const int st = g % kKVStages;
          const uint32_t ph = (g / kKVStages) & 1u;
          if (!mbar_wait(kv_empty0 + 8 * st, ph ^ 1u, abort_flag, err)) {
            ok = false;
            break;
          }
          const uint32_t fb = kv_full0 + 8 * st;
          mbar_expect_tx(fb, 2 * kBox);
          tma_load_3d(smem_u32(sK + st * kBox), &tmQKV, fb, C + it.h * kHD, j * kTile, it.b);
          tma_load_3d(smem_u32(sV + st * kBox), &tmQKV, fb, 2 * C + it.h * kHD, j * kTile, it.b);
          issued |= 1u << st;
          last_parity = (last_parity & ~(1u << st)) | (ph << st);
        }
      }
      // every copy issued lands before the shared memory is released (the
      // MMA warp has already waited for all of them unless it gave up)
      const uint64_t t0 = global_ns();
      if (q_issued)
        while (!mbar_try_wait(q_full, (q_issued - 1) & 1u) && global_ns() - t0 < kWaitLimitNs) {
        }
      for (int s2 = 0; s2 < kKVStages; ++s2) {
        if (!(issued & (1u << s2))) continue;
        while (!mbar_try_wait(kv_full0 + 8 * s2, (last_parity >> s2) & 1u) &&
               global_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1 || warp == kThreadsAttn / 32 - 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA --
      // One issuing warp per query tile (warp 1: tile A, the last warp:
      // tile B), so that neither tile's products wait behind the other's
      // barriers.  Both release each K/V stage and the Q tiles (the
      // barriers count two arrivals).
      const int t = warp == 1 ? 0 : 1;
      constexpr uint32_t idS = attn::idesc(kTile, false);
      constexpr uint32_t idO = attn::idesc(kHD, true);
      uint32_t n_item = 0, g = 0;
      uint32_t cs = 0, co = 0;  // S / PV products issued for this tile
      bool ok = true;
      const uint32_t q_base = smem_u32(sQ + t * kBox);
      const uint32_t p_t = tmem + kPCol + (uint32_t)(t * kHD);
      const uint32_t o_t = tmem + kOCol + (uint32_t)(t * kHD);
      const uint32_t s_t = tmem + (uint32_t)(t * kTile);
      FwdItem it;
      for (int k = 0; ok && fwd_item(k, B, H, nq, it); ++k, ++n_item) {
        ok = mbar_wait(q_full, n_item & 1u, abort_flag, err);
        if (!ok) break;
        tc_fence_after();
        const int nkv = it.nkv_b ? it.nkv_b : it.nkv_a;
        const int mine = t ? it.nkv_b : it.nkv_a;  // key tiles of this query tile (0: none)
        if (mine == 0) tc_commit(q_empty);
        for (int j = 0; j <= nkv && ok; ++j) {
          if (j < mine) {  // S_t = Q_t K_j^T
            const uint32_t gj = g + j, st = gj % kKVStages;
            ok = mbar_wait(kv_full0 + 8 * st, (gj / kKVStages) & 1u, abort_flag, err);
            if (ok) ok = mbar_wait(s_empty0 + 8 * t, (cs & 1u) ^ 1u, abort_flag, err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t k_base = smem_u32(sK + st * kBox);
#pragma unroll
            for (int kk = 0; kk < kHD / 16; ++kk)
              tc_mma(s_t, desc_kmajor(q_base, kk), desc_kmajor(k_base, kk), idS, kk > 0 ? 1u : 0u);
            tc_commit(s_full0 + 8 * t);
            ++cs;
            if (j == mine - 1) tc_commit(q_empty);  // this tile's Q is read
          }
          if (j >= 1) {
            const uint32_t st = (g + j - 1) % kKVStages;
            if (j - 1 < mine) {  // O_t (+)= P_t V_{j-1}, P_t from TMEM
              ok = mbar_wait(p_full0 + 8 * t, co & 1u, abort_flag, err);
              if (!ok) break;
              tc_fence_after();
              const uint32_t v_base = smem_u32(sV + st * kBox);
#pragma unroll
              for (int kk = 0; kk < kTile / 16; ++kk)
                attn::tc_mma_ts(o_t, p_t + (uint32_t)(8 * kk), desc_mnmajor(v_base, kk), idO,
                                (kk > 0 || j > 1) ? 1u : 0u);
              tc_commit(o_full0 + 8 * t);
              ++co;
            }
            tc_commit(kv_empty0 + 8 * st);  // this tile no longer reads key tile j-1
          }
        }
        g += nkv;
      }
      if (!ok) {  // let issued MMAs finish before TMEM is released
        tc_commit(drain0 + 8 * t);
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(drain0 + 8 * t, 0) && global_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // -------------------------------------------------------- softmax --
    const int t = (warp - 2) >> 2;  // query tile of the item: 0 = A, 1 = B
    const int qw = warp & 3;        // TMEM lane quarter
    const int r = qw * 32 + lane;   // row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const uint32_t s_col = lane_base + (uint32_t)(t * kTile);
    const uint32_t o_col = lane_base + kOCol + (uint32_t)(t * kHD);
    const uint32_t p_col = lane_base + kPCol + (uint32_t)(t * kHD);
    uint8_t* obox = sOut + (t * 4 + qw) * kOutBox;  // this warp's 32 output rows
    if (warp == 2 && lane == 0)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmOut)) : "memory");
    uint32_t cs = 0, co = 0;  // S tiles read / PV products waited for by this tile's threads
    bool ok = true;
    // wait for the next PV product of this tile (every completion is
    // waited for, in order, so that the barrier parity stays in step)
    auto wait_pv = [&]() -> bool {
      const bool r2 = __all_sync(0xffffffffu, mbar_wait(o_full0 + 8 * t, co & 1u, abort_flag, err));
      ++co;
      return r2;
    };
    FwdItem it;
    for (int k = 0; ok && fwd_item(k, B, H, nq, it); ++k) {
      const int nk = t ? it.nkv_b : it.nkv_a;
      if (nk == 0) continue;  // the item has no tile B
      const int qt = t ? it.qb : it.qa;
      const int qi = qt * kTile + r;  // query index in the sequence
      float m = -INFINITY, l = 0.f;  // reference max (log2 units) and the sum against it
      for (int j = 0; j < nk && ok; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_full0 + 8 * t, cs & 1u, abort_flag, err));
        if (!ok) break;
        ++cs;
        tc_fence_after();
        // the whole row of S in one round trip; the buffer goes straight back
        uint32_t sr[kTile];
#pragma unroll
        for (int c = 0; c < kTile; c += 32) tc_ld32(s_col + c, sr + c);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(s_empty0 + 8 * t);  // S_t is read: the next S_t may be computed
        if (j == nk - 1) {  // the diagonal tile: keys after the query are masked
#pragma unroll
          for (int c = 0; c < kTile; ++c)
            if (c > r) sr[c] = kNegInf;
        }
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < kTile; c += 2)
          mx4[(c >> 1) & 3] = attn::fmax3(mx4[(c >> 1) & 3], __uint_as_float(sr[c]),
                                          __uint_as_float(sr[c + 1]));
        const float mt = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
        const bool raise = mt > m + kRescaleLog2;  // always on the first key tile
        const float mn = raise ? mt : m;
        // P in registers (bf16 pairs) and its row sum
        uint32_t pk[kTile / 2];
        float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < kTile / 2; ++c) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(sr[2 * c]), sl2, -mn));
          const float p1 = fast_exp2(fmaf(__uint_as_float(sr[2 * c + 1]), sl2, -mn));
          sum4[(2 * c) & 3] += p0;
          sum4[(2 * c + 1) & 3] += p1;
          pk[c] = attn::pack_bf16x2(p0, p1);
        }
        // the previous product is complete: P_t is free and O_t may be rescaled
        if (j >= 1) {
          ok = wait_pv();
          if (!ok) break;
          tc_fence_after();
          if (raise) {  // rescale the row of O and the sum to the new reference
            const float f = fast_exp2(m - mn);
            l *= f;
#pragma unroll
            for (int hf = 0; hf < kHD; hf += 32) {
              uint32_t o[32];
              tc_ld32(o_col + hf, o);
              tc_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
              attn::tc_st32(o_col + hf, o);
            }
          }
        }
        m = mn;
        attn::tc_st32(p_col, pk);
        attn::tc_st32(p_col + 32, pk + 32);
        attn::tc_wait_st();
        tc_fence_before();
        mbar_arrive(p_full0 + 8 * t);  // P_t (and a rescaled O_t) may be consumed
        l += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      }
      if (!ok) break;
      // the item's last product, then the normalised row into this warp's
      // box and out by one TMA store per warp (rows past T are clipped by
      // the tensor map)
      ok = wait_pv();
      if (!ok) break;
      tc_fence_after();
      uint32_t ra[kHD];
#pragma unroll
      for (int c = 0; c < kHD; c += 32) tc_ld32(o_col + c, ra + c);
      tc_wait_ld();
      tc_fence_before();  // O is read before the next item's first product overwrites it
      const float inv = 1.f / l;
      if (lane == 0) bulk_wait_read<0>();  // the box's previous store has read it
      __syncwarp();
#pragma unroll
      for (int i = 0; i < kHD / 8; ++i) {
        uint4 w;
        uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          wp[q] = attn::pack_bf16x2(__uint_as_float(ra[8 * i + 2 * q]) * inv,
                                    __uint_as_float(ra[8 * i + 2 * q + 1]) * inv);
        *reinterpret_cast<uint4*>(obox + swz(lane, i)) = w;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(&tmOut, smem_u32(obox), it.h * kHD, qt * kTile + qw * 32, it.b);
        bulk_commit();
      }
      if (qi < T) lse[((size_t)it.b * H + it.h) * T + qi] = (m + log2f(l)) * 0.6931471805599453f;
    }
    if (lane == 0) bulk_wait_all();  // the output stores complete before the CTA leaves
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

cudaError_t seq_map(CUtensorMap* tm, const void* base, int B, int T, int cols, int box_rows,
                    int box_cols, bool swizzle) {
  using Key = std::tuple<const void*, int, int, int, int, int, bool>;
  static std::map<Key, CUtensorMap> cache;
  static std::mutex mu;
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  const Key key{base, B, T, cols, box_rows, box_cols, swizzle};
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
  cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  if (enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
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
  if (!attention_fwd_tc_supported(C, H) || (reinterpret_cast<uintptr_t>(qkv) & 15) ||
      (reinterpret_cast<uintptr_t>(att) & 15))
    return cudaErrorInvalidValue;
  CUtensorMap tm, tmo;
  cudaError_t e = attn::seq_map(&tm, qkv, B, T, 3 * C);
  if (e != cudaSuccess) return e;
  e = attn::seq_map(&tmo, att, B, T, C, 32);  // one softmax warp's 32 output rows per box
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
  const int items = (((T + kTile - 1) / kTile + 1) / 2) * B * H;
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = items < sms ? items : sms;
  launch_kernel(flash_fwd_tc_kernel, grid, kThreadsAttn, smem, s, tm, tmo, lse, B, T, C, H, sl2, err);
  note_launch();
  return cudaGetLastError();
}

}  // namespace gpt2k
