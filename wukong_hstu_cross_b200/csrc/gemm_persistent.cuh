// gemm_persistent.cuh — persistent tcgen05 GEMM with the fused RMSNorm row factor, for the
// large history-side projection  K|V = r(H_s) * H_s (W diag(g))^T  (M = sum of history
// lengths, up to ~10^6 rows; N = 2d; K = d).
//
// One CTA per SM walks the 128 x BN output tiles tile = blockIdx.x + i * gridDim.x (N-tiles of a
// row block are adjacent, so the A rows are fetched from HBM once and re-read from L2).
// Warp roles (320 threads):
//   warp 0      TMA producer over a STAGES-deep ring of [A 128x64 | W BNx64] stages.
//   warp 1      TMEM allocation (2 x BN columns: two accumulators) and the single MMA thread.
//               Tile i accumulates into buffer i % 2, so the epilogue of tile i overlaps the
//               MMAs of tile i+1.
//   warps 2..5  epilogue: TMEM -> registers (tcgen05.ld), scale by the row factor, bf16, into a
//               128-byte-swizzled staging tile in shared memory, then a TMA store (the store
//               un-swizzles; rows past M are clipped by the tensor bounds).
//   warps 6..9  row statistics: each thread reads its row of every A stage from shared memory
//               (logical chunk order) and publishes r = 1/sqrt(mean(x^2)+eps) per tile.
// Barriers: full/empty per stage; tmem_full/tmem_empty and norm_full per accumulator buffer.
// Every wait is bounded (mbar_wait).
#pragma once

#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace whale {

struct PGemmArgs {
  int M, N;
  int kb;          // 64-column K blocks
  int tiles_n;     // N / BN
  int num_tiles;   // tiles_m * tiles_n
  float inv_k, eps;
};

template <int BN>
struct PGemmSmem {
  static constexpr int BM = 128, BK = 64;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t EPI_BYTES = 4 /*warps*/ * 2 /*buffers*/ * 32 * 128;  // 32 rows x 64 bf16
  // 227 KB per CTA: alignment slack, staging tiles, row factors and barriers, the rest stages
  static constexpr int FIXED = 1024 + EPI_BYTES + 2 * 128 * 4 + 256;
  static constexpr int STAGES = (232448 - FIXED) / (int)STAGE_BYTES > 8 ? 8 : (232448 - FIXED) / (int)STAGE_BYTES;
  static constexpr size_t BYTES = FIXED + STAGES * (size_t)STAGE_BYTES;
};

constexpr int kPGemmThreads = 320;

template <int BN>
__global__ void __launch_bounds__(kPGemmThreads, 1)
    gemm_rownorm_persistent_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                   const __grid_constant__ CUtensorMap tmOut, const PGemmArgs args) {
  using L = PGemmSmem<BN>;
  constexpr int ST = L::STAGES;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = smem + ST * L::STAGE_BYTES;                       // [warp][buf] 4 KB staging tiles
  float* rbuf = reinterpret_cast<float*>(epi + L::EPI_BYTES);       // [2][128] row factors
  uint64_t* full = reinterpret_cast<uint64_t*>(rbuf + 2 * 128);
  uint64_t* empty = full + ST;
  uint64_t* tfull = empty + ST;    // [2]
  uint64_t* tempty = tfull + 2;    // [2]
  uint64_t* nfull = tempty + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(nfull + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = args.kb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
      mbar_init(&nfull[i], 4);
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
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int kg = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < args.num_tiles && !stop; tile += gridDim.x) {
        const int m0 = (tile / args.tiles_n) * L::BM, n0 = (tile % args.tiles_n) * BN;
        for (int kb = 0; kb < KB; ++kb, ++kg) {
          const int s = kg % ST, u = kg / ST;
          if (kg >= ST && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag)) {
            stop = true;
            break;
          }
          uint8_t* st = smem + s * L::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], L::STAGE_BYTES);
          tma_load_2d(st, &tmA, kb * L::BK, m0, &full[s]);
          tma_load_2d(st + L::A_BYTES, &tmB, kb * L::BK, n0, &full[s]);
        }
      }
      if (*abort_flag) {
        volatile int quiet = 0;
        for (int k = (kg > ST ? kg - ST : 0); k < kg; ++k) mbar_wait(&full[k % ST], (k / ST) & 1, &quiet);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
      int kg = 0, it = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < args.num_tiles && !stop; tile += gridDim.x, ++it) {
        const int acc = it & 1, ua = it >> 1;
        if (it >= 2 && !mbar_wait(&tempty[acc], (ua - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
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
            umma_f16(d_tmem, sdesc_k_sw128(a_base + kk * 32), sdesc_k_sw128(b_base + kk * 32), idesc,
                     (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        umma_commit(&tfull[acc]);
      }
    }
  } else if (warp >= 6) {
    // ---------------- row statistics ----------------
    const int row = (warp & 3) * 32 + lane;
    int kg = 0, it = 0;
    for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1, ua = it >> 1;
      float ss = 0.f;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++kg) {
        const int s = kg % ST, u = kg / ST;
        if (!mbar_wait(&full[s], u & 1, abort_flag)) {
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
      // rbuf[acc] is free once the epilogue of tile it-2 released its accumulator buffer
      if (it >= 2 && !mbar_wait(&tempty[acc], (ua - 1) & 1, abort_flag)) break;
      rbuf[acc * 128 + row] = rsqrtf(ss * args.inv_k + args.eps);
      __syncwarp();
      if (lane == 0) mbar_arrive(&nfull[acc]);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    uint8_t* stage0 = epi + (warp - 2) * 2 * 4096;
    int it = 0, nstore = 0;
    for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1, ua = it >> 1;
      const int m0 = (tile / args.tiles_n) * L::BM, n0 = (tile % args.tiles_n) * BN;
      if (!mbar_wait(&tfull[acc], ua & 1, abort_flag)) break;
      if (!mbar_wait(&nfull[acc], ua & 1, abort_flag)) break;
      tc_fence_after();
      const float r = rbuf[acc * 128 + row];
      const uint32_t t_row = tmem_base + acc * BN + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / 64; ++c, ++nstore) {
        uint32_t v0[32], v1[32];
        tmem_ld_32x32b_x32(t_row + c * 64, v0);
        tmem_ld_32x32b_x32(t_row + c * 64 + 32, v1);
        tmem_ld_wait();
        uint8_t* sb = stage0 + (nstore & 1) * 4096;
        // the TMA store issued two chunks ago from this buffer must have finished reading it
        if (lane == 0) bulk_wait_read<1>();
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
      // the accumulator buffer and its row factors may be reused
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace whale
