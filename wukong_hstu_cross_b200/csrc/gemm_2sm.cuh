// gemm_2sm.cuh — persistent 2-SM (cta_group::2) tcgen05 GEMM with the fused RMSNorm row factor,
// for the large history-side projection K|V = r(H_s) * H_s (W diag(g))^T.
//
// A cluster of two CTAs on two SMs computes 256 x 256 output tiles: each CTA stages its own 128
// rows of A and its own 128 rows (output columns) of W per 64-wide K block, the even CTA issues
// tcgen05.mma.cta_group::2 (M = 256, N = 256), and each CTA's TMEM receives its 128 rows of the
// accumulator. Per SM this streams 32 KB of operands per 64-deep K block against 2 MFLOP of
// MMA work — half the operand bytes per FLOP of a one-SM 128 x 256 tile — so six stages cover
// twice the load latency.
//
// Per CTA (480 threads): warp 0 TMA producer (both CTAs; completion counted on the even CTA's
// `full` barrier), warp 1 TMEM allocation (2 x 256 columns: two accumulators) and, in the even
// CTA, the MMA thread, warps 2..9 epilogue (two warps per TMEM lane quadrant, 128 columns each:
// TMEM -> row factor -> bf16 -> swizzled staging -> TMA store), warps 10..13 row statistics (sum
// of squares of each row of A from the staged tiles), warp 14 (even CTA) relays "stage s landed"
// to both CTAs' `ready[s]`, so the statistic warps of the odd CTA, whose bytes are counted on the
// even CTA's barrier, know when to read.
// Barriers (same offsets in both CTAs): full[s] (even only), ready[s], empty[s] (MMA commit
// multicast to both + 4 local statistic warps), tfull[2] (commit multicast), tempty[2] (even
// only: 8 + 8 epilogue warps), nfull[2], edone[2] (local). Every wait is bounded; every thread of
// both CTAs reaches the closing cluster barrier on every path.
#pragma once

#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace whale {

struct G2Args {
  int M, N;
  int kb;          // 64-column K blocks
  int tiles_n;     // N / 256
  int num_tiles;   // ceil(M / 256) * tiles_n
  float inv_k, eps;
};

struct G2Smem {
  static constexpr int BK = 64;
  static constexpr uint32_t A_BYTES = 128 * BK * 2;   // this CTA's 128 rows of A
  static constexpr uint32_t B_BYTES = 128 * BK * 2;   // this CTA's 128 rows of W
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t EPI_BYTES = 8 * 32 * 128;  // one 32 x 64 bf16 staging tile per epilogue warp
  static constexpr int FIXED = 1024 + EPI_BYTES + 2 * 128 * 4 + 512;
  static constexpr int STAGES = (232448 - FIXED) / (int)STAGE_BYTES > 8 ? 8 : (232448 - FIXED) / (int)STAGE_BYTES;
  static constexpr size_t BYTES = FIXED + STAGES * (size_t)STAGE_BYTES;
};

constexpr int kG2Threads = 480;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kG2Threads, 1)
    gemm_rownorm_2sm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmOut, const G2Args args) {
  using L = G2Smem;
  constexpr int ST = L::STAGES;
  constexpr uint32_t TMEM_COLS = 512;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = smem + ST * L::STAGE_BYTES;
  float* rbuf = reinterpret_cast<float*>(epi + L::EPI_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(rbuf + 2 * 128);
  uint64_t* ready = full + ST;
  uint64_t* empty = ready + ST;
  uint64_t* tfull = empty + ST;   // [2]
  uint64_t* tempty = tfull + 2;   // [2]
  uint64_t* nfull = tempty + 2;   // [2]
  uint64_t* edone = nfull + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(edone + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KB = args.kb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 1);
      mbar_init(&empty[s], 1 + 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 16);
      mbar_init(&nfull[i], 4);
      mbar_init(&edone[i], 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmOut);
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
        const int n0 = (tile % args.tiles_n) * 256 + (int)rank * 128;
        for (int kb = 0; kb < KB; ++kb, ++kg) {
          const int s = kg % ST, u = kg / ST;
          if (kg >= ST && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag)) {
            stop = true;
            break;
          }
          uint8_t* st = smem + s * L::STAGE_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * L::STAGE_BYTES);  // both CTAs' bytes
          tma_load_2d_cg2(st, &tmA, kb * L::BK, m0, bar);
          tma_load_2d_cg2(st + L::A_BYTES, &tmB, kb * L::BK, n0, bar);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (even CTA) ----------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256);
      int kg = 0, it = 0;
      bool stop = false;
      for (int tile = pair; tile < args.num_tiles && !stop; tile += npairs, ++it) {
        const int acc = it & 1, ua = it >> 1;
        if (it >= 2 && !mbar_wait(&tempty[acc], (ua - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        for (int kb = 0; kb < KB; ++kb, ++kg) {
          const int s = kg % ST, u = kg / ST;
          if (!mbar_wait(&full[s], u & 1, abort_flag)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * L::STAGE_BYTES);
          const uint32_t b_base = a_base + L::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < L::BK / 16; ++kk)
            umma_f16_cg2(d_tmem, sdesc_k_sw128(a_base + kk * 32), sdesc_k_sw128(b_base + kk * 32), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_cg2_mc(&empty[s], 0x3);
        }
        umma_commit_cg2_mc(&tfull[acc], 0x3);
      }
    }
  } else if (warp == 14) {
    // ---------------- relay (even CTA): "stage s landed" to both CTAs' statistic warps ----------
    // (kept off the MMA thread: the cluster-scope release of the remote arrive is a fence)
    if (leader && lane == 0) {
      const uint32_t peer_ready0 = mapa_shared(smem_u32(&ready[0]), 1);
      const int total = ((args.num_tiles - pair + npairs - 1) / npairs) * KB;
      for (int kg = 0; kg < total; ++kg) {
        const int s = kg % ST, u = kg / ST;
        if (!mbar_wait(&full[s], u & 1, abort_flag)) break;
        mbar_arrive(&ready[s]);
        mbar_arrive_cluster(peer_ready0 + s * 8);
      }
    }
  } else if (warp >= 10) {
    // ---------------- row statistics (both CTAs) ----------------
    const int row = (warp & 3) * 32 + lane;
    int kg = 0, it = 0;
    for (int tile = pair; tile < args.num_tiles; tile += npairs, ++it) {
      const int acc = it & 1, ua = it >> 1;
      float ss = 0.f;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++kg) {
        const int s = kg % ST, u = kg / ST;
        if (!mbar_wait(&ready[s], u & 1, abort_flag)) {
          ok = false;
          break;
        }
        const uint4* rp = reinterpret_cast<const uint4*>(smem + s * L::STAGE_BYTES + row * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
          bf16x8_to_f32(rp[c ^ (row & 7)], f);
#pragma unroll
          for (int j = 0; j < 8; ++j) ss = fmaf(f[j], f[j], ss);
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
  } else {
    // ---------------- epilogue (warps 2..9, both CTAs): two warps per TMEM lane quadrant ----------
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;  // columns [128 * half, 128 * half + 128) of the tile
    const int row = q * 32 + lane;
    uint8_t* sbuf = epi + (warp - 2) * 4096;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    int it = 0, nstore = 0;
    for (int tile = pair; tile < args.num_tiles; tile += npairs, ++it) {
      const int acc = it & 1, ua = it >> 1;
      const int m0 = (tile / args.tiles_n) * 256 + (int)rank * 128, n0 = (tile % args.tiles_n) * 256;
      if (!mbar_wait(&tfull[acc], ua & 1, abort_flag)) break;
      if (!mbar_wait(&nfull[acc], ua & 1, abort_flag)) break;
      tc_fence_after();
      const float r = rbuf[acc * 128 + row];
      const uint32_t t_row = tmem_base + acc * 256 + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc, ++nstore) {
        const int c = 2 * half + cc;
        uint32_t v0[32], v1[32];
        tmem_ld_32x32b_x32(t_row + c * 64, v0);
        tmem_ld_32x32b_x32(t_row + c * 64 + 32, v1);
        tmem_ld_wait();
        uint8_t* sb = sbuf;
        // the TMA store issued from this buffer for the previous chunk must have read it
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        uint4* dst = reinterpret_cast<uint4*>(sb + lane * 128);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v0[8 * j + 0]) * r, __uint_as_float(v0[8 * j + 1]) * r);
          w.y = pack_bf16x2(__uint_as_float(v0[8 * j + 2]) * r, __uint_as_float(v0[8 * j + 3]) * r);
          w.z = pack_bf16x2(__uint_as_float(v0[8 * j + 4]) * r, __uint_as_float(v0[8 * j + 5]) * r);
          w.w = pack_bf16x2(__uint_as_float(v0[8 * j + 6]) * r, __uint_as_float(v0[8 * j + 7]) * r);
          dst[j ^ (lane & 7)] = w;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v1[8 * j + 0]) * r, __uint_as_float(v1[8 * j + 1]) * r);
          w.y = pack_bf16x2(__uint_as_float(v1[8 * j + 2]) * r, __uint_as_float(v1[8 * j + 3]) * r);
          w.z = pack_bf16x2(__uint_as_float(v1[8 * j + 4]) * r, __uint_as_float(v1[8 * j + 5]) * r);
          w.w = pack_bf16x2(__uint_as_float(v1[8 * j + 6]) * r, __uint_as_float(v1[8 * j + 7]) * r);
          dst[(4 + j) ^ (lane & 7)] = w;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmOut, sb, n0 + c * 64, m0 + q * 32);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&edone[acc]);
        mbar_arrive_cluster(tempty0 + acc * 8);  // the even CTA's MMA may reuse this accumulator
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its shared memory or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_cg2(tmem_base, TMEM_COLS);
  }
}

}  // namespace whale
