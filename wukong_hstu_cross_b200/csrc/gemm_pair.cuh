// gemm_pair.cuh — the token-side GEMM with hi/lo operand pairs on CTA pairs (cta_group::2).
//
// Same operation, epilogues and outputs as gemm_tc_kernel with SPLIT (see gemm_tc.cuh), on
// 256 x BN output tiles: a cluster of two CTAs on two SMs, each staging its own 128 rows of A
// (hi and lo) and its own BN/2 rows of W per 64-deep K block; the even CTA issues
// tcgen05.mma.cta_group::2 (M = 256, N = BN) and each CTA's TMEM receives the accumulator of its
// 128 rows. Per SM a K block streams 32 KB of A plus BN/2 rows of W instead of BN rows: a quarter
// fewer operand bytes at BN = 256, a sixth fewer at BN = 128. On the 2048-row token batch this did
// not shorten the main loops (selected with WHALE_GEMM_PAIR=1; one CTA per tile is the default).
//
// Per CTA: warp 0 TMA producer (both CTAs; copies counted on the even CTA's `full` barrier),
// warp 1 TMEM allocation (2 x BN columns, two accumulators) and, in the even CTA, the MMA thread,
// warps 2..5 epilogue (thread i of quadrant q owns row 32q + i of the CTA's 128 rows; the shared
// epilogue of gemm_tc.cuh), and with ROWNORM warps 6..9 row statistics of the CTA's own A rows and
// warp 10 (even CTA) relaying "stage s landed" to both CTAs' `ready[s]`.
// Barriers (same offsets in both CTAs): full[s] (even only), ready[s] (ROWNORM), empty[s] (MMA
// commit to both + 4 local statistic warps with ROWNORM), tfull[2] (commit to both), tempty[2]
// (even only: 4 + 4 epilogue warps), nfull[2], edone[2] (local). Every wait is bounded; every
// thread of both CTAs reaches the closing cluster barrier on every path.
#pragma once

#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace whale {

template <int BN>
struct PairSmem {
  static constexpr int BK = 64;
  static constexpr uint32_t A_BYTES = 128 * BK * 2;       // this CTA's 128 rows of one source half
  static constexpr uint32_t A_ALL = 2 * A_BYTES;          // hi | lo
  static constexpr uint32_t B_BYTES = (BN / 2) * BK * 2;  // this CTA's BN/2 rows of W
  static constexpr uint32_t STAGE_BYTES = A_ALL + B_BYTES;
  static constexpr int FIXED = 1024 /*alignment slack*/ + 2 * 128 * 4 /*row factors*/ + 512 /*barriers*/;
  static constexpr int STAGES =
      ((232448 - FIXED) / (int)STAGE_BYTES) > 8 ? 8 : ((232448 - FIXED) / (int)STAGE_BYTES);
  static constexpr size_t BYTES = FIXED + STAGES * (size_t)STAGE_BYTES;
  static_assert(STAGE_BYTES % 1024 == 0, "stages stay 1024-byte aligned for the 128-byte swizzle");
};

template <bool ROWNORM>
constexpr int pair_threads() {
  return ROWNORM ? 352 : 192;
}

template <int BN, int EPI, bool ROWNORM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads<ROWNORM>(), 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA0lo,
                     const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmA1lo,
                     const __grid_constant__ CUtensorMap tmB, const GemmArgs args) {
  using L = PairSmem<BN>;
  constexpr int STAGES = L::STAGES;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* rbuf = reinterpret_cast<float*>(smem + STAGES * L::STAGE_BYTES);  // [2][128] row factors
  uint64_t* full = reinterpret_cast<uint64_t*>(rbuf + 2 * 128);
  uint64_t* ready = full + STAGES;
  uint64_t* empty = ready + STAGES;
  uint64_t* tfull = empty + STAGES;  // [2]
  uint64_t* tempty = tfull + 2;      // [2]
  uint64_t* nfull = tempty + 2;      // [2]
  uint64_t* edone = nfull + 2;       // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(edone + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KB = args.kb0 + args.kb1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 1);
      mbar_init(&empty[s], 1 + (ROWNORM ? 4 : 0));
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);
      mbar_init(&nfull[i], 4);
      mbar_init(&edone[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA0lo);
    tma_prefetch_desc(&tmB);
    if (args.kb1 > 0) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmA1lo);
    }
  }
  if (warp == 1) {
    tmem_alloc_cg2(tmem_slot, TMEM_COLS);
    tmem_relinquish_cg2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrive or counted copy
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int kg = 0;
      bool stop = false;
      for (int tile = pair; tile < args.num_tiles && !stop; tile += npairs) {
        const int m0 = (tile / args.tiles_n) * 256 + (int)rank * 128;
        const int nb = (tile % args.tiles_n) * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < KB; ++kb, ++kg) {
          const int s = kg % STAGES, u = kg / STAGES;
          if (kg >= STAGES && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag)) {
            stop = true;
            break;
          }
          uint8_t* st = smem + s * L::STAGE_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * L::STAGE_BYTES);  // both CTAs' bytes
          const bool first = kb < args.kb0;
          const int kc = (first ? kb : kb - args.kb0) * L::BK;
          tma_load_2d_cg2(st, first ? &tmA0 : &tmA1, kc, m0, bar);
          tma_load_2d_cg2(st + L::A_BYTES, first ? &tmA0lo : &tmA1lo, kc, m0, bar);
          tma_load_2d_cg2(st + L::A_ALL, &tmB, kb * L::BK, nb, bar);
        }
      }
      if (leader && *abort_flag) {
        // Unwinding after a timeout: the copies of both CTAs are counted here; let the issued
        // stages land before the cluster leaves (the odd CTA waits at the closing barrier).
        volatile int quiet = 0;
        for (int k = (kg > STAGES ? kg - STAGES : 0); k < kg; ++k)
          mbar_wait(&full[k % STAGES], (k / STAGES) & 1, &quiet);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (even CTA): tile i accumulates into buffer i % 2 ----------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, BN);
      int kg = 0, it = 0;
      bool stop = false;
      for (int tile = pair; tile < args.num_tiles && !stop; tile += npairs, ++it) {
        const int acc = it & 1, ua = it >> 1;
        if (it >= 2 && !mbar_wait(&tempty[acc], (ua - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < KB; ++kb, ++kg) {
          const int s = kg % STAGES, u = kg / STAGES;
          if (!mbar_wait(&full[s], u & 1, abort_flag)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * L::STAGE_BYTES);
          const uint32_t b_base = a_base + L::A_ALL;
#pragma unroll
          for (int kk = 0; kk < L::BK / 16; ++kk) {
            const uint64_t bdesc = sdesc_k_sw128(b_base + kk * 32);
            umma_f16_cg2(d_tmem, sdesc_k_sw128(a_base + kk * 32), bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            umma_f16_cg2(d_tmem, sdesc_k_sw128(a_base + L::A_BYTES + kk * 32), bdesc, idesc, 1u);
          }
          umma_commit_cg2_mc(&empty[s], 0x3);
        }
        umma_commit_cg2_mc(&tfull[acc], 0x3);  // also on abort: arrives once all issued MMAs are done
      }
    }
  } else if (ROWNORM && warp == 10) {
    // ---------------- relay (even CTA): "stage s landed" to both CTAs' statistic warps ----------
    if (leader && lane == 0) {
      const uint32_t peer_ready0 = mapa_shared(smem_u32(&ready[0]), 1);
      const int total = ((args.num_tiles - pair + npairs - 1) / npairs) * KB;
      for (int kg = 0; kg < total; ++kg) {
        const int s = kg % STAGES, u = kg / STAGES;
        if (!mbar_wait(&full[s], u & 1, abort_flag)) break;
        mbar_arrive(&ready[s]);
        mbar_arrive_cluster(peer_ready0 + s * 8);
      }
    }
  } else if (ROWNORM && warp >= 6) {
    // ---------------- row statistics of this CTA's 128 rows (sum of squares of A0 = hi + lo) ----------
    const int row = (warp & 3) * 32 + lane;
    int kg = 0, it = 0;
    for (int tile = pair; tile < args.num_tiles; tile += npairs, ++it) {
      const int acc = it & 1, ua = it >> 1;
      float ss = 0.f;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++kg) {
        const int s = kg % STAGES, u = kg / STAGES;
        if (!mbar_wait(&ready[s], u & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (kb < args.kb0) {
          // the row's 16-byte chunk c sits at c ^ (row % 8) (128-byte swizzle), in hi and lo alike
          const uint8_t* st = smem + s * L::STAGE_BYTES + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int pc = c ^ (row & 7);
            float f[8], fl[8];
            bf16x8_to_f32(reinterpret_cast<const uint4*>(st)[pc], f);
            bf16x8_to_f32(reinterpret_cast<const uint4*>(st + L::A_BYTES)[pc], fl);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float x = f[j] + fl[j];
              ss = fmaf(x, x, ss);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      if (!ok) break;
      if (it >= 2 && !mbar_wait(&edone[acc], (ua - 1) & 1, abort_flag)) break;
      rbuf[acc * 128 + row] = rsqrtf(ss * args.inv_k + args.eps);
      __syncwarp();
      if (lane == 0) mbar_arrive(&nfull[acc]);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---------------- epilogue (both CTAs): the CTA's 128 rows of each 256-row tile ----------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    float4 pre[EpiPre<BN, EPI>::kN];
    int it = 0;
    for (int tile = pair; tile < args.num_tiles; tile += npairs, ++it) {
      const int acc = it & 1, ua = it >> 1;
      const int m0 = (tile / args.tiles_n) * 256 + (int)rank * 128, n0 = (tile % args.tiles_n) * BN;
      const long long gm = (long long)m0 + row;
      const bool row_ok = gm < args.M;
      epi_load_resid<BN, EPI>(args, gm, row_ok, n0, pre);
      if (!mbar_wait(&tfull[acc], ua & 1, abort_flag)) break;
      if (ROWNORM && !mbar_wait(&nfull[acc], ua & 1, abort_flag)) break;
      tc_fence_after();
      const float r = ROWNORM ? rbuf[acc * 128 + row] : 1.0f;
      epi_tile<BN, EPI>(args, tmem_base + acc * BN + ((uint32_t)(q * 32) << 16), r, gm, row_ok, n0, pre);
      // this accumulator buffer (both CTAs' halves) and the row factors may be reused
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&edone[acc]);
        mbar_arrive_cluster(tempty0 + acc * 8);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still count copies or MMAs into it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_cg2(tmem_base, TMEM_COLS);
  }
}

}  // namespace whale
