// bf16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Persistent, warp-specialised kernel, one CTA per SM:
//   warp 0     TMA producer: 128x64 A and BNx64 B tiles (128-byte swizzle)
//              into a STAGES-deep shared-memory ring;
//   warp 1     allocates TMEM and issues tcgen05.mma (M=128, N=BN, K=16)
//              from one elected lane, accumulating fp32 in TMEM;
//   warps 2-9  epilogue, two warps per TMEM lane quarter: each warp owns
//              32 rows and every other 64-column group of the tile.  Per
//              group: tcgen05.ld of the accumulator (thread = row), bias /
//              GELU / residual / GELU-backward, the result written to the
//              warp's own 128-byte-swizzled shared-memory box and sent with
//              one TMA bulk store (TMA reduce-add for the fp32 gradient
//              accumulation).  Residual and pre-activation inputs arrive by
//              TMA in the same box ahead of the accumulator read.  Warps
//              synchronise only within themselves, so no epilogue step
//              waits for another warp.
// CTA pairs (template argument CG = 2, a cluster of two CTAs on neighbouring
// SMs): 256 x 256 output tiles.  Each CTA stages its own 128 rows of A and
// half of the B tile (its ring stages are 32 KB, six of them), its TMA
// copies completing on the even CTA's full barrier; the even CTA's MMA
// thread issues tcgen05.mma.cta_group::2 (M = 256), so each SM computes its
// 128 x 256 half of the tile while reading only half of B from shared
// memory.  Stage releases and tile completions reach both CTAs through
// multicast tcgen05.commit; each epilogue warp of either CTA returns the
// accumulator with one arrival on the even CTA's barrier.  TMEM is
// allocated and freed by one warp of each CTA together, after cluster
// barriers.  No TMA load multicasts.
// The TMEM accumulator is double-buffered so the epilogue of one tile runs
// under the main loop of the next.  Both operands may be K-major or
// MN-major (the tensor core reads either from the descriptor), which covers
// the forward (A, B K-major), data-gradient (B MN-major) and
// weight-gradient (both MN-major) products without any transpose copies.
//
// Every mbarrier wait is bounded: after ~2 s a role sets an abort flag and
// the device error word (ERR_TIMEOUT), the other roles see the flag and
// leave their loops, the producer waits (bounded) for its copies in flight,
// and TMEM is freed before the kernel returns.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "gemm_epi.cuh"
#include "tc_util.cuh"

namespace gpt2k {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
// The GELU backward on CTA pairs sums its output's columns (the W_fc bias
// gradient) in a warp of its own after the epilogue warps, fed box by box
// (in a pair the epilogue sets the pace, and the sums would add a third to
// its instructions); on single CTAs the epilogue warps sum their own boxes.
constexpr bool sums_warp(int epi, int cg) { return epi == EPI_DGELU && cg == 2; }
constexpr int kSumsWarps = 2;  // each sums the boxes of half the epilogue warps
constexpr int kernel_threads(int epi, int cg) {
  return 64 + kEpiThreads + (sums_warp(epi, cg) ? 32 * kSumsWarps : 0);
}
constexpr int kWarpBox = 4096;  // one warp's epilogue box: 32 rows x 128 bytes

// Epilogues that read a second [M, N] input (residual or pre-activation).
constexpr bool epi_has_input(int epi) { return epi == EPI_BIAS_RESID || epi == EPI_DGELU; }
// Boxes per epilogue warp.  With two, a warp writes one box while TMA still
// reads the other (output epilogues), or the next group's input streams into
// a box of its own while the current group is computed (input epilogues).
// The second box costs a ring stage, which is worth it only for the GELU
// backward (measured: one ring stage less slows the store, bias, GELU and
// fp32 forms more than the second box gains).
constexpr int epi_boxes(int epi) { return epi == EPI_DGELU ? 2 : 1; }
// Operand ring depth: what the shared memory holds next to the epilogue boxes
// (a CTA of a pair holds half of the B tile, so its stages are smaller).
constexpr int ring_stages(int bn, int epi, int cg) {
  return cg == 2 ? (epi_boxes(epi) == 2 ? 5 : 6)
                 : bn == 256 ? (epi_boxes(epi) == 2 ? 3 : 4) : (epi_boxes(epi) == 2 ? 5 : 6);
}

// Instruction descriptor: bf16 x bf16 -> fp32, M = 128 per CTA (256 for a
// pair), N = BN.
template <int BN, bool A_MN, bool B_MN, int CG>
__host__ __device__ constexpr uint32_t make_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((A_MN ? 1u : 0u) << 15) |
         ((B_MN ? 1u : 0u) << 16) | ((uint32_t)(BN >> 3) << 17) |
         ((uint32_t)((BM * CG) >> 4) << 24);
}

template <int BN>
constexpr uint32_t tmem_cols() {
  return 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
}

template <int BN, int EPI, int CG>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)ring_stages(BN, EPI, CG) * (BM * BK * 2 + (BN / CG) * BK * 2) +
         (size_t)kEpiWarps * epi_boxes(EPI) * kWarpBox + 256 + (sums_warp(EPI, CG) ? 128 : 0);
}

template <int BN, int STAGES, bool A_MN, bool B_MN, int EPI, int CG>
__global__ void __launch_bounds__(kernel_threads(EPI, CG), 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmOut,
                   const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                   const __grid_constant__ CUtensorMap tmOut2, const EpiParams ep, int K,
                   int tiles_m, int tiles_n, int splits, int kb_per_split, int n_fast, int tiles_m1,
                   int M2, int* err) {
  constexpr int A_BYTES = BM * BK * 2;
  constexpr int B_BYTES = (BN / CG) * BK * 2;  // this CTA's rows of the B tile
  constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = tmem_cols<BN>();
  constexpr bool HAS_IN = epi_has_input(EPI);
  constexpr bool SW = sums_warp(EPI, CG);
  static_assert(STAGES == ring_stages(BN, EPI, CG), "ring depth");
  static_assert(CG == 1 || (CG == 2 && BN == 256), "CTA pairs use 256 x 256 tiles");
  // CTA pair: rank 0 (the leader) issues the MMAs for both CTAs; each CTA
  // loads its 128 rows of A and BN / 2 rows of B and runs the epilogue of
  // its 128 rows of the tile.
  pdl_launch_dependents();
  const uint32_t rank = CG == 2 ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  constexpr bool F32_OUT = (EPI == EPI_F32_ACC || EPI == EPI_F32_STORE);
  constexpr bool HAS_BIAS = (EPI == EPI_BIAS || EPI == EPI_BIAS_GELU || EPI == EPI_BIAS_RESID);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  constexpr int NBOX = epi_boxes(EPI);
  uint8_t* sBox = smem + STAGES * (A_BYTES + B_BYTES);  // [kEpiWarps][NBOX] boxes, 1024-aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(sBox + kEpiWarps * NBOX * kWarpBox);
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4 + kEpiWarps + (SW ? 2 * kEpiWarps : 0));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + 2);
  const uint32_t in_full0 = smem_u32(bars + 2 * STAGES + 4);  // [kEpiWarps]
  // sums warp: an epilogue warp's output box holds a group / has been summed
  const uint32_t cs_full0 = smem_u32(bars + 2 * STAGES + 4 + kEpiWarps);       // [kEpiWarps]
  const uint32_t cs_empty0 = smem_u32(bars + 2 * STAGES + 4 + 2 * kEpiWarps);  // [kEpiWarps]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kb_total = (K + BK - 1) / BK;
  const int tiles = tiles_m * tiles_n;
  const int units = tiles * splits;
  const int unit0 = blockIdx.x / CG, unit_step = gridDim.x / CG;  // a pair shares its units

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, CG * kEpiWarps);  // one arrival per epilogue warp of the pair
    }
    for (int w = 0; w < kEpiWarps; ++w) mbar_init(in_full0 + 8 * w, 1);
    if (SW)
      for (int w = 0; w < kEpiWarps; ++w) {
        mbar_init(cs_full0 + 8 * w, 32);
        mbar_init(cs_empty0 + 8 * w, 32);
      }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // for a pair: one warp of each CTA allocates collectively
    if (CG == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
  }
  tc_fence_before();
  if (CG == 2) cluster_sync();  // the peer's barriers are initialised before any remote use
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // set-up done; the operands of the previous kernels are complete from here on

  auto decode = [&](int u, int& tm, int& tn, int& kb0, int& kb1, int& sp) {
    sp = u / tiles;
    const int r = u - sp * tiles;
    if (n_fast) {
      tm = r / tiles_n;
      tn = r - tm * tiles_n;
    } else {
      tn = r / tiles_m;
      tm = r - tn * tiles_m;
    }
    kb0 = sp * kb_per_split;
    kb1 = min(kb0 + kb_per_split, kb_total);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- producer --
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0;  // stages that received at least one load
      uint32_t last_parity = 0;  // parity of the latest fill of each stage
      bool ok = true;
      for (int u = unit0; u < units && ok; u += unit_step) {
        int tm, tn, kb0, kb1, sp;
        decode(u, tm, tn, kb0, kb1, sp);
        // row tiles from tiles_m1 on belong to the second product
        const bool p2 = tm >= tiles_m1;
        const CUtensorMap* mA = p2 ? &tmA2 : &tmA;
        const CUtensorMap* mB = p2 ? &tmB2 : &tmB;
        const int am = (p2 ? tm - tiles_m1 : tm) * BM * CG + (int)rank * BM;  // this CTA's rows of A
        const int bn0 = tn * BN + (int)rank * (BN / CG);       // and of B
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, err)) {
            ok = false;
            break;
          }
          if (ep.expiry_test > 0 && blockIdx.x == 0 && u == unit0 && kb == kb0 + ep.expiry_test - 1) {
            // test of the bounded waits: this stage is never filled
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t a_dst = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * B_BYTES);
          if (CG == 1) {
            mbar_expect_tx(fb, STAGE_TX);
            if (!A_MN) {
              tma_load_2d(a_dst, mA, fb, kb * BK, am);
            } else {
              tma_load_2d(a_dst, mA, fb, am, kb * BK);
              tma_load_2d(a_dst + 8192, mA, fb, am + 64, kb * BK);
            }
            if (!B_MN) {
              tma_load_2d(b_dst, mB, fb, kb * BK, bn0);
            } else {
#pragma unroll
              for (int j = 0; j < BN / 64; ++j) tma_load_2d(b_dst + 8192 * j, mB, fb, bn0 + 64 * j, kb * BK);
            }
          } else {
            // both CTAs' copies complete on the leader's full barrier, which
            // expects the pair's bytes
            if (leader) mbar_expect_tx(fb, CG * STAGE_TX);
            const uint32_t lfb = map_shared(fb, 0);
            if (!A_MN) {
              tma_load_2d_pair(a_dst, mA, lfb, kb * BK, am);
            } else {
              tma_load_2d_pair(a_dst, mA, lfb, am, kb * BK);
              tma_load_2d_pair(a_dst + 8192, mA, lfb, am + 64, kb * BK);
            }
            if (!B_MN) {
              tma_load_2d_pair(b_dst, mB, lfb, kb * BK, bn0);
            } else {
#pragma unroll
              for (int j = 0; j < BN / CG / 64; ++j)
                tma_load_2d_pair(b_dst + 8192 * j, mB, lfb, bn0 + 64 * j, kb * BK);
            }
          }
          issued_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && CG == 2 && !leader) {
        // this CTA's copies complete on the leader's barriers: give them a
        // short bounded time to land
        const uint64_t t0 = global_ns();
        while (global_ns() - t0 < 200000ull) {
        }
      } else if (!ok) {
        // Give the copies already issued a bounded time to land before the
        // shared memory they target is released.
        const uint64_t t0 = global_ns();
        for (int s = 0; s < STAGES; ++s) {
          if (!(issued_mask & (1u << s))) continue;
          const uint32_t par = (last_parity >> s) & 1u;
          while (!mbar_try_wait(full0 + 8 * s, par)) {
            if (global_ns() - t0 > kWaitLimitNs) break;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // --------------------------------------------------------- MMA --
      constexpr uint32_t idesc = make_idesc<BN, A_MN, B_MN, CG>();
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = unit0; u < units && ok; u += unit_step) {
        int tm, tn, kb0, kb1, sp;
        decode(u, tm, tn, kb0, kb1, sp);
        if (CG == 2 ? !mbar_wait_cluster(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, err)
                    : !mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, err))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = A_MN ? desc_mnmajor(a_base, k) : desc_kmajor(a_base, k);
            const uint64_t bd = B_MN ? desc_mnmajor(b_base, k) : desc_kmajor(b_base, k);
            if (CG == 1) tc_mma(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
            else tc_mma_pair(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          if (CG == 1) tc_commit(empty0 + 8 * stage);
          else tc_commit_pair(empty0 + 8 * stage, 0x3);  // the stage is free in both CTAs
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (CG == 1) tc_commit(tfull0 + 8 * acc);
        else tc_commit_pair(tfull0 + 8 * acc, 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {
        // let MMAs already issued finish before TMEM is released
        if (CG == 1) tc_commit(tfull0 + 8 * acc);
        else tc_commit_pair(tfull0 + 8 * acc, 0x1);
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(tfull0 + 8 * acc, acc_phase)) {
          if (global_ns() - t0 > kWaitLimitNs) break;
        }
      }
    }
  } else if (SW && warp >= 2 + kEpiWarps) {
    // -------------------------------------------------------------- sums --
    // Sums warp sw takes the epilogue warps whose groups are sw, sw + 2 of
    // each tile, in their order (each warp's k-th group, warp by warp).
    // Once a warp's output box holds a group, lane l reads 16-byte chunk
    // l % 8 (8 columns) of rows l / 8 + 4i, i = 0..7, adds them in row order,
    // the four lanes of a chunk are added pairwise (rows r, r + 1, then
    // r + 2), and lanes 0-7 write the group's 64 column sums into its slab of
    // ep.colsum; then the box goes back to its warp.
    if (ep.colsum) {
      const int sw = warp - 2 - kEpiWarps;
      uint32_t gcw[kEpiWarps / kSumsWarps];
#pragma unroll
      for (int i = 0; i < kEpiWarps / kSumsWarps; ++i) gcw[i] = 0;
      bool ok = true;
      const int ch = lane & 7, r0l = lane >> 3;  // this lane's chunk and first row
      for (int u = unit0; u < units && ok; u += unit_step) {
        int tm, tn, kb0, kb1, sp;
        decode(u, tm, tn, kb0, kb1, sp);
        const int m0 = tm * BM * CG + (int)rank * BM, nt0 = tn * BN;
        const int ngroups = (min(BN, ep.N - nt0) + 63) >> 6;
        for (int k = 0; k < 2 && ok; ++k) {
#pragma unroll
          for (int i = 0; i < kEpiWarps / kSumsWarps; ++i) {
            const int w = sw * (kEpiWarps / kSumsWarps) + i;  // epilogue warp w + 2
            const int g = (w >> 2) + 2 * k;                    // its k-th group
            const int r0 = m0 + ((w + 2) & 3) * 32;            // and its slab
            if (!ok || g >= ngroups || r0 >= ep.M) continue;
            ok = __all_sync(0xffffffffu, mbar_wait(cs_full0 + 8 * w, gcw[i] & 1u, abort_flag, err));
            if (!ok) continue;
            const uint8_t* box = sBox + w * NBOX * kWarpBox;  // the warp's output box
            const int rows = min(32, ep.M - r0);
            float2 cs[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
              const int row = r0l + 4 * rr;
              if (row < rows) {
                const uint4 v = *reinterpret_cast<const uint4*>(box + swz(row, ch));
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  cs[e] = f2_add(cs[e], make_float2(__uint_as_float(wv[e] << 16),
                                                    __uint_as_float(wv[e] & 0xffff0000u)));
              }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              cs[e].x += __shfl_xor_sync(0xffffffffu, cs[e].x, 8);
              cs[e].y += __shfl_xor_sync(0xffffffffu, cs[e].y, 8);
              cs[e].x += __shfl_xor_sync(0xffffffffu, cs[e].x, 16);
              cs[e].y += __shfl_xor_sync(0xffffffffu, cs[e].y, 16);
            }
            const int col = nt0 + 64 * g + 8 * ch;
            if (lane < 8) {
              float* dst = ep.colsum + (size_t)(r0 >> 5) * ep.N + col;
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (col + 2 * e < ep.N)  // N even: both columns of a pair in range
                  *reinterpret_cast<float2*>(dst + 2 * e) = cs[e];
            }
            __syncwarp();
            mbar_arrive(cs_empty0 + 8 * w);
            ++gcw[i];
          }
        }
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;   // groups h, h + 2, ... of each tile
    uint8_t* wbox = sBox + (warp - 2) * NBOX * kWarpBox;  // this warp's boxes
    // input epilogues: the input box (the second box, or the only one)
    uint8_t* ibox = wbox + (NBOX - 1) * kWarpBox;
    const uint32_t ibox_u = smem_u32(ibox);
    int ob = 0;  // output box of the next store (alternates when the output has two)
    const uint32_t in_full = in_full0 + 8 * (warp - 2);
    uint32_t in_phase = 0;
    bool in_pend = false;  // an input copy is in flight
    bool pre = false;      // the input of this warp's next group is already requested
    if (warp == 2 && lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmOut)) : "memory");
      if (EPI == EPI_BIAS_GELU || HAS_IN)
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
    }
    // Write 8 16-byte chunks of this thread's row into the warp's box and
    // send the box with `send` from lane 0 once every lane's writes are
    // visible to the async proxy.  The box is reused only after the
    // previous store has read it.
    // With two output boxes used in turn, every store but the latest (which
    // read the other box) must have read its box.
    constexpr int OUT_BOXES = HAS_IN ? 1 : NBOX;
    auto put_box = [&](auto write_row, auto send) {
      uint8_t* box = wbox + ob * kWarpBox;
      if (lane == 0) {
        if (OUT_BOXES == 2) bulk_wait_read<1>();
        else bulk_wait_read<0>();
      }
      __syncwarp();
      write_row(box);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        send(smem_u32(box));
        bulk_commit();
      }
      if (OUT_BOXES == 2) ob ^= 1;
    };
    // This warp has read its accumulator columns of the tile: one arrival
    // per warp on the leader's barrier (the peer CTA's warps arrive remotely;
    // relaxed, as the leader's MMAs only overwrite TMEM columns whose loads
    // have returned).
    const uint32_t tempty_leader = CG == 2 ? map_shared(tempty0, 0) : 0u;
    auto release_acc = [&](int a) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 1) mbar_arrive(tempty0 + 8 * a);
        else mbar_arrive_cluster_relaxed(tempty_leader + 8 * a);
      }
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t gc = 0;  // groups this warp has handed to the sums warp
    bool ok = true;
    for (int u = unit0; u < units && ok; u += unit_step) {
      int tm, tn, kb0, kb1, sp;
      decode(u, tm, tn, kb0, kb1, sp);
      const bool p2 = tm >= tiles_m1;  // a tile of the second product
      const CUtensorMap* mOut = p2 ? &tmOut2 : &tmOut;
      const int mlim = p2 ? M2 : ep.M;
      const int m0 = (p2 ? tm - tiles_m1 : tm) * BM * CG + (int)rank * BM, nt0 = tn * BN;
      const int r0 = m0 + q * 32;  // first row of this warp's slab
      const int ngroups = (min(BN, ep.N - nt0) + 63) >> 6;  // 64-column groups in range
      ok = __all_sync(0xffffffffu, mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, err));
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      if (h >= ngroups) release_acc(acc);  // no group for this warp in a narrow tile
#pragma unroll 1
      for (int g = h; g < ngroups; g += 2) {
        const int nb = nt0 + 64 * g;  // first column of the group
        const bool live = r0 < mlim;  // rows of this slab exist
        if (HAS_IN && live && !pre && lane == 0) {
          // the group's input slab, ahead of the accumulator read (a shared
          // box is free once the previous store has read it)
          if (NBOX == 1) bulk_wait_read<0>();
          mbar_expect_tx(in_full, kWarpBox);
          tma_load_3d(ibox_u, &tmX, in_full, nb, r0, 0);
          in_pend = true;
        }
        pre = false;
        float v[64];
        {
          uint32_t r[64];
          tc_ld32(t_row + (uint32_t)(64 * g), r);
          tc_ld32(t_row + (uint32_t)(64 * g + 32), r + 32);
          tc_wait_ld();
          if (g + 2 >= ngroups) release_acc(acc);  // every TMEM read of this warp for the tile is done
#pragma unroll
          for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
        }
        if (ep.alpha != 1.0f) {  // uniform: the forward and most gradients take alpha = 1
#pragma unroll
          for (int i = 0; i < 64; i += 2) set2(v, i, f2_mul(get2(v, i), f2_splat(ep.alpha)));
        }
        if (HAS_BIAS && ep.bias) {
          if (nb + 64 <= ep.N) {
            const float4* b4 = reinterpret_cast<const float4*>(ep.bias + nb);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float4 b = __ldg(b4 + j);
              set2(v, 4 * j, f2_add(get2(v, 4 * j), make_float2(b.x, b.y)));
              set2(v, 4 * j + 2, f2_add(get2(v, 4 * j + 2), make_float2(b.z, b.w)));
            }
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (nb + i < ep.N) v[i] += ep.bias[nb + i];
          }
        }
        if (!live) continue;  // slab entirely below the matrix: nothing to store
        if (HAS_IN) {
          ok = __all_sync(0xffffffffu, mbar_wait(in_full, in_phase, abort_flag, err));
          if (!ok) break;
          in_phase ^= 1u;
          in_pend = false;
          uint4 xin[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) xin[c] = *reinterpret_cast<const uint4*>(ibox + swz(lane, c));
          __syncwarp();  // every lane has read the input box
          if (NBOX == 2) {
            // request this warp's next input now: group g + 2 of this tile, or
            // group h of the next tile
            int pn = -1, pr = 0;
            if (g + 2 < ngroups) {
              pn = nb + 128;
              pr = r0;
            } else if (u + unit_step < units) {
              int tm2, tn2, kb02, kb12, sp2;
              decode(u + unit_step, tm2, tn2, kb02, kb12, sp2);
              const int nt2 = tn2 * BN, r2 = tm2 * BM * CG + (int)rank * BM + q * 32;
              if (h < ((min(BN, ep.N - nt2) + 63) >> 6) && r2 < ep.M) {
                pn = nt2 + 64 * h;
                pr = r2;
              }
            }
            if (pn >= 0) {
              if (lane == 0) {
                fence_async_smem();  // the reads above come before the copy's writes
                mbar_expect_tx(in_full, kWarpBox);
                tma_load_3d(ibox_u, &tmX, in_full, pn, pr, 0);
                in_pend = true;
              }
              pre = true;
            }
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xin[c]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 x = __bfloat1622float2(x2[i]);
              const int e = 8 * c + 2 * i;
              if (EPI == EPI_BIAS_RESID) set2(v, e, f2_add(get2(v, e), x));
              else set2(v, e, f2_mul(get2(v, e), gelu_tanh_grad2(x)));
            }
          }
        }
        if (F32_OUT) {
          // two 32-column fp32 boxes, one after the other
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if (half == 1 && nb + 32 >= ep.N) break;
            put_box(
                [&](uint8_t* box) {
#pragma unroll
                  for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<float4*>(box + swz(lane, j)) =
                        make_float4(v[32 * half + 4 * j], v[32 * half + 4 * j + 1],
                                    v[32 * half + 4 * j + 2], v[32 * half + 4 * j + 3]);
                },
                [&](uint32_t box_u) {
                  if (EPI == EPI_F32_ACC) tma_reduce_add_3d(mOut, box_u, nb + 32 * half, r0, 0);
                  else tma_store_3d(mOut, box_u, nb + 32 * half, r0, sp);
                });
          }
        } else {
          if (EPI == EPI_BIAS_GELU) {
            // the pre-activation u first (saved for the backward), then GELU
            // of u as stored (bf16), which a backward that recomputes GELU
            // from u reproduces bit for bit
            uint4 up[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&up[j]);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                h2[i] = __floats2bfloat162_rn(v[8 * j + 2 * i], v[8 * j + 2 * i + 1]);
                const float2 f = __bfloat1622float2(h2[i]);
                v[8 * j + 2 * i] = f.x;
                v[8 * j + 2 * i + 1] = f.y;
              }
            }
            put_box(
                [&](uint8_t* box) {
#pragma unroll
                  for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(box + swz(lane, j)) = up[j];
                },
                [&](uint32_t box_u) { tma_store_3d(&tmX, box_u, nb, r0, 0); });
#pragma unroll
            for (int i = 0; i < 64; i += 2) set2(v, i, gelu_tanh2(get2(v, i)));
          }
          if (SW && ep.colsum) {  // the sums warp has read the box's previous group
            ok = __all_sync(0xffffffffu,
                            mbar_wait(cs_empty0 + 8 * (warp - 2), (gc & 1u) ^ 1u, abort_flag, err));
            if (!ok) break;
          }
          put_box(
              [&](uint8_t* box) {
#pragma unroll
                for (int j = 0; j < 8; ++j) store8(reinterpret_cast<act_t*>(box + swz(lane, j)), v + 8 * j);
              },
              [&](uint32_t box_u) { tma_store_3d(mOut, box_u, nb, r0, 0); });
          if (SW && ep.colsum) {
            mbar_arrive(cs_full0 + 8 * (warp - 2));  // the box holds this group
            ++gc;
          } else if (EPI == EPI_DGELU && ep.colsum) {
            // column sums of the stored slab: lane l adds columns 2l, 2l + 1
            // of the box's rows in order (the TMA store reads the same box;
            // the next group's writes wait for both)
            const uint8_t* box = wbox + (ob ^ (OUT_BOXES == 2 ? 1 : 0)) * kWarpBox;
            const int rows = min(32, ep.M - r0);
            const uint32_t cof = (uint32_t)(lane & 3) * 4u;
            float2 cs = make_float2(0.f, 0.f);
#pragma unroll 8
            for (int r = 0; r < rows; ++r) {
              const uint32_t w = *reinterpret_cast<const uint32_t*>(box + swz(r, lane >> 2) + cof);
              cs = f2_add(cs, make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)));
            }
            const int col = nb + 2 * lane;
            if (col < ep.N)  // N even: both columns in range
              *reinterpret_cast<float2*>(ep.colsum + (size_t)(r0 >> 5) * ep.N + col) = cs;
          }
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) {
      bulk_wait_all();
      // an input copy still in flight lands before the shared memory is released
      const uint64_t t0 = global_ns();
      while (in_pend && !mbar_try_wait(in_full, in_phase) && global_ns() - t0 < kWaitLimitNs) {
      }
    }
  }

  tc_fence_before();
  // a pair leaves together: no MMA of the leader, copy or remote arrival
  // still targets the peer when it exits
  if (CG == 2) cluster_sync();
  else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if (CG == 1)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(TMEM_COLS));
    else
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(TMEM_COLS));
  }
}

// ------------------------------------------------------------ host side --
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::mutex g_mu;

static cudaError_t get_encoder() {
  if (g_encode) return cudaSuccess;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess) return e;
  if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

// Tensor map with 128-byte swizzle over a row-major [outer][inner] array
// (`ld` elements between rows), box box_inner x box_outer.  depth = 0 gives
// a rank-2 map (GEMM operands); depth >= 1 a rank-3 map over `depth` such
// arrays `dstride` elements apart (epilogue boxes, addressed with 3-D
// coordinates), box depth 1.  fp32 = element type float, else bf16.
static cudaError_t make_tmap(CUtensorMap* tm, const void* ptr, bool fp32, uint64_t inner,
                             uint64_t outer, uint64_t ld, uint32_t box_inner, uint32_t box_outer,
                             uint64_t depth = 0, uint64_t dstride = 0) {
  using Key = std::tuple<const void*, bool, uint64_t, uint64_t, uint64_t, uint32_t, uint32_t,
                         uint64_t, uint64_t>;
  static std::map<Key, CUtensorMap> cache;
  const Key key{ptr, fp32, inner, outer, ld, box_inner, box_outer, depth, dstride};
  {
    std::lock_guard<std::mutex> g(g_mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *tm = it->second;
      return cudaSuccess;
    }
  }
  cudaError_t e = get_encoder();
  if (e != cudaSuccess) return e;
  const uint64_t es = fp32 ? 4 : 2;
  const cuuint32_t rank = depth >= 1 ? 3 : 2;
  cuuint64_t dims[3] = {inner, outer, depth >= 1 ? depth : 1};
  cuuint64_t strides[2] = {ld * es, (depth > 1 ? dstride : ld * outer) * es};
  cuuint32_t box[3] = {box_inner, box_outer, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = g_encode(tm, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        rank, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> g(g_mu);
  if (cache.size() > 4096) cache.clear();
  cache[key] = *tm;
  return cudaSuccess;
}

static int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = kNumSMs;
  }
  return n;
}

template <int BN, bool A_MN, bool B_MN, int EPI, int CG>
static cudaError_t launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& to,
                          const CUtensorMap& tx, const CUtensorMap& ta2, const CUtensorMap& tb2,
                          const CUtensorMap& to2, int M2, const EpiParams& ep, int K, int splits,
                          int kb_per_split, int n_fast, cudaStream_t s, int* err) {
  auto kern = gemm_tc_kernel<BN, ring_stages(BN, EPI, CG), A_MN, B_MN, EPI, CG>;
  constexpr size_t smem = smem_bytes<BN, EPI, CG>();
  static_assert(smem <= 232448, "shared memory budget");
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int tiles_m1 = (ep.M + BM * CG - 1) / (BM * CG);
  const int tiles_m = tiles_m1 + (M2 + BM * CG - 1) / (BM * CG);
  const int tiles_n = (ep.N + BN - 1) / BN;
  const int units = tiles_m * tiles_n * splits;
  const int slots = num_sms() / CG;  // persistent CTAs (pairs)
  const int grid = CG * (units < slots ? units : slots);
  // a pair is a cluster of two CTAs along x
  const cudaError_t e = launch_kernel_cluster(kern, dim3(grid), dim3(kernel_threads(EPI, CG)), smem, s, CG, ta, tb,
                                              to, tx, ta2, tb2, to2, ep, K, tiles_m, tiles_n, splits,
                                              kb_per_split, n_fast, tiles_m1, M2, err);
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

template <int BN, int CG>
static cudaError_t dispatch(const GemmArgs& a, const CUtensorMap& ta, const CUtensorMap& tb,
                            const CUtensorMap& to, const CUtensorMap& tx, const CUtensorMap& ta2,
                            const CUtensorMap& tb2, const CUtensorMap& to2, int M2,
                            const EpiParams& ep, int epi, int splits, int kb_per_split, int n_fast,
                            cudaStream_t s, int* err) {
#define GPT2_TC(AM, BMJ, E)                                                                      \
    if (a.a_mn == AM && a.b_mn == BMJ && epi == E)                                               \
      return launch<BN, AM, BMJ, E, CG>(ta, tb, to, tx, ta2, tb2, to2, M2, ep, a.K, splits,      \
                                        kb_per_split, n_fast, s, err);
  GPT2_TC(0, 0, EPI_STORE)
  GPT2_TC(0, 0, EPI_BIAS)
  GPT2_TC(0, 0, EPI_BIAS_GELU)
  GPT2_TC(0, 0, EPI_BIAS_RESID)
  GPT2_TC(0, 1, EPI_STORE)
  GPT2_TC(0, 1, EPI_DGELU)
  GPT2_TC(1, 1, EPI_F32_ACC)
  GPT2_TC(1, 1, EPI_F32_STORE)
  GPT2_TC(1, 0, EPI_STORE)
  GPT2_TC(0, 0, EPI_F32_STORE)  // split small-M products
#undef GPT2_TC
  return cudaErrorInvalidValue;
}

}  // namespace tc

// The epilogue of a split small-M product: element (m, n) gets the sum of
// its split partials ws[s][m][n], s ascending, then the product's epilogue.
template <int EPI>
__global__ void splitk_epilogue_kernel(EpiParams e, const float* __restrict__ ws, int splits) {
  pdl_start();
  const size_t total = (size_t)e.M * e.N;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    float acc = ws[i];
    for (int k = 1; k < splits; ++k) acc += ws[(size_t)k * total + i];
    epi_scalar<EPI>(e, (int)(i / e.N), (int)(i % e.N), acc);
  }
}

__global__ void splitk_reduce_kernel(float* out32, long ldo32, const float* ws, int splits, int M,
                                     int N) {
  pdl_start();
  const size_t total = (size_t)M * N;
  if (ldo32 == N && (total & 3) == 0) {  // contiguous output: float4 path
    const size_t t4 = total / 4;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < t4;
         i += (size_t)gridDim.x * blockDim.x) {
      float4 s = reinterpret_cast<const float4*>(ws)[i];
      for (int k = 1; k < splits; ++k) {
        const float4 w = reinterpret_cast<const float4*>(ws + (size_t)k * total)[i];
        s.x += w.x; s.y += w.y; s.z += w.z; s.w += w.w;
      }
      float4 o = reinterpret_cast<float4*>(out32)[i];
      o.x += s.x; o.y += s.y; o.z += s.z; o.w += s.w;
      reinterpret_cast<float4*>(out32)[i] = o;
    }
    return;
  }
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(i / N), n = (int)(i % N);
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += ws[(size_t)k * total + i];
    out32[(size_t)m * ldo32 + n] += s;
  }
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool gemm_colsum_supported() { return true; }

static int g_cta_pairs = 1;
int gemm_set_cta_pairs(int enable) {
  const int prev = g_cta_pairs;
  g_cta_pairs = enable ? 1 : 0;
  return prev;
}

// The product and the one stacked under it, one launch each.
static cudaError_t gemm_in_turn(const GemmArgs& a, cudaStream_t s, int* err) {
  GemmArgs first = a;
  first.M2 = 0;
  const cudaError_t e = gemm(first, s, err);
  if (e != cudaSuccess) return e;
  return gemm(gemm_second(a), s, err);
}

cudaError_t gemm(const GemmArgs& a, cudaStream_t s, int* err) {
  using namespace tc;
  if (a.M2 > 0 && (a.M <= 0 || a.N <= 0 || a.K <= 0)) return gemm(gemm_second(a), s, err);
  if (a.M <= 0 || a.N <= 0 || a.K <= 0) return cudaSuccess;
  // A second product stacked under this one (same N and K, fp32 accumulate)
  // shares the launch when both are whole 256-row pair tiles and the split
  // plan needs no partials; otherwise the two run one after the other.
  const bool grouped = a.M2 > 0;
  if (grouped) {
    const bool can = a.epi == EPI_F32_ACC && g_cta_pairs && a.N >= 256 && a.a_mn && a.b_mn &&
                     a.M % (2 * BM) == 0 && a.M2 % (2 * BM) == 0 && aligned16(a.A2) &&
                     aligned16(a.B2) && a.out32_2 && aligned16(a.out32_2) && a.lda2 % 8 == 0 &&
                     a.ldb2 % 8 == 0 && a.ldo32_2 % 4 == 0;
    if (!can) return gemm_in_turn(a, s, err);
  }
  const int Mt = a.M + (grouped ? a.M2 : 0);  // rows of both products
  // TMA: 16-byte aligned bases and row strides for every operand and output
  if (!aligned16(a.A) || !aligned16(a.B) || (a.lda % 8) || (a.ldb % 8)) return cudaErrorInvalidValue;
  const bool f32_out = a.epi == EPI_F32_ACC || a.epi == EPI_F32_STORE;
  if (f32_out ? (!a.out32 || !aligned16(a.out32) || (a.ldo32 % 4))
              : (!a.out || !aligned16(a.out) || (a.ldo % 8)))
    return cudaErrorInvalidValue;
  if (a.epi == EPI_BIAS_RESID && (!a.resid || !aligned16(a.resid) || (a.ldr % 8)))
    return cudaErrorInvalidValue;
  if ((a.epi == EPI_BIAS_GELU || a.epi == EPI_DGELU) && (!a.aux || !aligned16(a.aux) || (a.ldaux % 8)))
    return cudaErrorInvalidValue;
  if (a.bias && !aligned16(a.bias)) return cudaErrorInvalidValue;
  const int BN = a.N >= 256 ? 256 : 128;
  CUtensorMap ta, tb, to, tx;
  std::memset(&to, 0, sizeof(to));
  std::memset(&tx, 0, sizeof(tx));
  cudaError_t e;
  if (!a.a_mn) e = make_tmap(&ta, a.A, false, a.K, a.M, a.lda, 64, BM);
  else e = make_tmap(&ta, a.A, false, a.M, a.K, a.lda, 64, 64);
  if (e != cudaSuccess) return e;

  if (a.colsum && (a.epi != EPI_DGELU || a.N % 2 || !aligned16(a.colsum))) return cudaErrorInvalidValue;
  EpiParams ep{a.M, a.N, a.alpha, a.out, a.ldo, a.out32, a.ldo32, a.bias, a.resid, a.ldr, a.aux, a.ldaux,
               a.expiry_test, a.colsum};
  // 256 x 256 tiles over CTA pairs for the wide products (measured: 5-11 %
  // faster where the main loop sets the pace, and 10-12 % for the GELU
  // forward, at M = 16384, N = 3072, K = 768, once the accumulator release
  // became a relaxed arrival).  The GELU backward keeps single CTAs: with
  // its fused column sums it measured 85 us in pairs against 82 us.
  const int CG = (g_cta_pairs && BN == 256 && a.M > BM) ? 2 : 1;
  const int slots = num_sms() / CG;  // persistent CTAs or pairs
  const int tiles = ((Mt + BM * CG - 1) / (BM * CG)) * ((a.N + BN - 1) / BN);
  const int kb_total = (a.K + BK - 1) / BK;

  // split-K for the weight-gradient products with few output tiles: pick the
  // split count with the lowest estimated time = whole waves of units at
  // ~8.5 TFLOP/s per SM + the partials' write/read and the output update
  // at ~6 TB/s (at least 4 k-blocks per split; partials must fit)
  // (a two-way split into a zero accumulator adds both partials in place:
  // no partials to write and read back)
  int splits = 1;
  int epi = a.epi;
  if (a.epi == EPI_F32_ACC && a.max_splits > 1 && a.split_ws && tiles < slots &&
      aligned16(a.split_ws) && a.N % 4 == 0) {
    double best = 1e30;
    const double out_bytes = 4.0 * Mt * a.N;
    for (int sp = 1; sp <= a.max_splits; ++sp) {
      if (sp > 1 && (sp > kb_total / 4 || (size_t)sp * Mt * a.N > a.split_ws_floats)) break;
      const int waves = (tiles * sp + slots - 1) / slots;
      const double t_unit = 2.0 * BM * BN * ((double)kb_total * BK / sp) / 8.5e12;
      const double t_red = sp == 1 ? 0.0
                           : (sp == 2 && a.acc_zero) ? out_bytes / 6.0e12
                                                     : (2.0 * sp + 2.0) * out_bytes / 6.0e12;
      const double t = waves * t_unit + t_red;
      if (t < best * 0.98) {
        best = t;
        splits = sp;
      }
    }
  }
  // products of a single 128-row tile with a bf16 epilogue (one position
  // per sequence in generation): a few tiles would leave most SMs idle, so K
  // is split until the units fill the machine; the fp32 partials are summed
  // in split order and the epilogue applied by splitk_epilogue_kernel
  const bool small_m = !f32_out && a.M <= BM && a.epi != EPI_DGELU && !a.colsum &&
                       a.max_splits > 1 && a.split_ws && aligned16(a.split_ws) && a.N % 4 == 0;
  if (small_m) {
    int sp = min(min(slots / tiles, a.max_splits), kb_total);
    while (sp > 1 && (size_t)sp * a.M * a.N > a.split_ws_floats) --sp;
    splits = sp > 1 ? sp : 1;
  }
  int kb_per_split = (kb_total + splits - 1) / splits;
  splits = (kb_total + kb_per_split - 1) / kb_per_split;  // no empty split
  const bool in_place = splits == 2 && a.acc_zero;  // both halves reduce-add into out32
  if (grouped && splits > 1 && !in_place) return gemm_in_turn(a, s, err);
  if (!a.b_mn) e = make_tmap(&tb, a.B, false, a.K, a.N, a.ldb, 64, BN / CG);
  else e = make_tmap(&tb, a.B, false, a.N, a.K, a.ldb, 64, 64);
  if (e != cudaSuccess) return e;
  // epilogue tensor maps
  // epilogue tensor maps: one warp's 32-row slab per box
  if (splits > 1 && !in_place) {
    epi = EPI_F32_STORE;
    e = make_tmap(&to, a.split_ws, true, a.N, a.M, a.N, 32, 32, splits, (uint64_t)a.M * a.N);
  } else if (f32_out) {
    e = make_tmap(&to, a.out32, true, a.N, a.M, a.ldo32, 32, 32, 1);
  } else {
    e = make_tmap(&to, a.out, false, a.N, a.M, a.ldo, 64, 32, 1);
  }
  if (e != cudaSuccess) return e;
  if (a.epi == EPI_BIAS_RESID) e = make_tmap(&tx, a.resid, false, a.N, a.M, a.ldr, 64, 32, 1);
  else if (a.epi == EPI_BIAS_GELU || a.epi == EPI_DGELU)
    e = make_tmap(&tx, a.aux, false, a.N, a.M, a.ldaux, 64, 32, 1);
  if (e != cudaSuccess) return e;
  // the second product's operands and output (both operands MN-major)
  CUtensorMap ta2 = ta, tb2 = tb, to2 = to;
  if (grouped) {
    e = make_tmap(&ta2, a.A2, false, a.M2, a.K, a.lda2, 64, 64);
    if (e == cudaSuccess) e = make_tmap(&tb2, a.B2, false, a.N, a.K, a.ldb2, 64, 64);
    if (e == cudaSuccess) e = make_tmap(&to2, a.out32_2, true, a.N, a.M2, a.ldo32_2, 32, 32, 1);
    if (e != cudaSuccess) return e;
  }
  const int M2 = grouped ? a.M2 : 0;
  // The larger operand is reused by consecutive tiles (L2 locality).
  const double a_bytes = (double)Mt * a.K, b_bytes = (double)a.N * a.K;
  const int n_fast = a_bytes > b_bytes ? 1 : 0;
  if (CG == 2)
    e = dispatch<256, 2>(a, ta, tb, to, tx, ta2, tb2, to2, M2, ep, epi, splits, kb_per_split, n_fast, s, err);
  else if (BN == 256)
    e = dispatch<256, 1>(a, ta, tb, to, tx, ta2, tb2, to2, M2, ep, epi, splits, kb_per_split, n_fast, s, err);
  else
    e = dispatch<128, 1>(a, ta, tb, to, tx, ta2, tb2, to2, M2, ep, epi, splits, kb_per_split, n_fast, s, err);
  if (e != cudaSuccess) return e;
  if (splits > 1 && small_m) {
    const size_t total = (size_t)a.M * a.N;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 8 * num_sms()) blocks = 8 * num_sms();
    EpiParams ep1 = ep;
    ep1.alpha = 1.f;  // the partials are already scaled
    switch (a.epi) {
      case EPI_STORE: launch_kernel(splitk_epilogue_kernel<EPI_STORE>, blocks, 256, 0, s, ep1, a.split_ws, splits); break;
      case EPI_BIAS: launch_kernel(splitk_epilogue_kernel<EPI_BIAS>, blocks, 256, 0, s, ep1, a.split_ws, splits); break;
      case EPI_BIAS_GELU: launch_kernel(splitk_epilogue_kernel<EPI_BIAS_GELU>, blocks, 256, 0, s, ep1, a.split_ws, splits); break;
      case EPI_BIAS_RESID: launch_kernel(splitk_epilogue_kernel<EPI_BIAS_RESID>, blocks, 256, 0, s, ep1, a.split_ws, splits); break;
      default: return cudaErrorInvalidValue;
    }
    note_launch();
    e = cudaGetLastError();
  } else if (splits > 1 && !in_place) {
    const size_t total = (size_t)a.M * a.N;
    int blocks = (int)((total / 4 + 255) / 256);
    if (blocks > 8 * num_sms()) blocks = 8 * num_sms();
    if (blocks < 1) blocks = 1;
    launch_kernel(splitk_reduce_kernel, blocks, 256, 0, s, a.out32, a.ldo32, a.split_ws, splits, a.M, a.N);
    note_launch();
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace gpt2k
