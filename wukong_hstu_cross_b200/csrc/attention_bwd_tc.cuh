// attention_bwd_tc.cuh — backward of Eq. (4) on the 5th-generation tensor cores (bf16 mode, d_h = 64,
// up to 32 queries per example), the same products and schedule as attention_bwd.cuh:
//   S^T = K Q^T,  dP^T = V dA^T,  P^T = 2^(S^T log2(e)/sqrt(d_h) - lse),  dS^T = P^T (dP^T - delta),
//   dV = P^T dA,  dK = (dS^T / sqrt(d_h)) Q,  dQ^T += K^T (dS^T / sqrt(d_h)).
// KV-parallel (gist.science technical summary of WHALE, section 2.2, Asymmetric Backward Variants):
// a CTA owns one head of a chunk of history rows of one example (kBwdChunkTc rows at most), keeps the example's
// queries (q, dA as bf16 pairs) in shared memory and walks the chunk in blocks of 128 rows, so dK and
// dV of a block are complete inside the CTA and only dQ (N d_h values per chunk) is added to global
// memory with fp32 atomics.
//
// Per block, with every operand a hi/lo bf16 pair:
//   tensor memory: S^T | dP^T (double-buffered, 32 + 32 columns), dV and dK (double-buffered, 64
//   columns each) and the running dQ^T (64 x 128: see below), all fp32;
//   shared memory: the K|V block ring (TMA, 128-byte swizzle); P^T and dS^T written by the softmax
//   threads in the K-major 128-byte-swizzled layout the MMA reads, each as one tile whose 128-byte
//   rows hold the hi half (queries 0-31) then the lo half; and the dK|dV drain's staging.
// S^T, dP^T, dV and dK take three MMAs per k-step (hi hi, lo hi, hi lo). dQ^T takes one: its A
// operand is the K tile MN-major with M = 128, whose two 64-element MN groups are the K hi and K lo
// tiles (adjacent in the stage), and its B operand the dS^T tile MN-major with N = 64 (the hi and lo
// halves side by side), so TMEM lane (g 64 + m), column (h 32 + n) holds K_g^T dS_h for d_h index m
// and query n, and dQ is the sum of the four (g, h) products.
// Warp roles (320 threads): warp 0 TMA producer, warp 1 TMEM allocation + MMA issue (one thread),
// warps 2..5 the softmax backward (the next block's while a block's MMAs run), warps 6..9 the dK|dV
// drain while the next block is computed: rows scaled by r, split into pairs, written into the warp's
// staging and stored from there with tensor stores (boxes of 32 rows x 64 columns: tmDKV, tmDKVlo).
// A K|V stage is refilled as soon as the MMAs of its block are complete. Thread i of TMEM lane
// quadrant q owns block row 32q + i.
// Rows past the chunk (the next example's, or past the states) and queries past N are read but give
// P = 0 and dS = 0: lse is +inf for the missing queries and the rows past the chunk are masked.
#pragma once

#include "attention_bwd.cuh"
#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace whale {

constexpr int kBwdChunkTc = 2048;  // history rows per CTA (sixteen blocks of 128)

struct AttnBwdTcSmem {
  static constexpr uint32_t TILE_Q = 32 * 128;    // 32 queries x 64 d_h bf16
  static constexpr uint32_t TILE_KV = 128 * 128;  // 128 rows x 64 d_h bf16
  static constexpr uint32_t OFF_Q = 0;            // q, q_lo, da, da_lo
  static constexpr uint32_t OFF_KV = 4 * TILE_Q;  // [2 stages][k, k_lo, v, v_lo]
  static constexpr uint32_t OFF_STG = OFF_KV + 2 * 4 * TILE_KV;  // [p | p_lo], [ds | ds_lo]
  static constexpr uint32_t OFF_DST = OFF_STG + 2 * TILE_KV;     // drain: [4 warps][hi 32 rows | lo 32 rows]
  static constexpr uint32_t OFF_LSE = OFF_DST + 4 * 8192;        // lse[32], delta[32]
  static constexpr uint32_t OFF_BAR = OFF_LSE + 256;
  static constexpr uint32_t BYTES = OFF_BAR + 256 + 1024;  // + alignment slack
};
static_assert(AttnBwdTcSmem::BYTES <= 232448, "shared memory");
constexpr int kAttnBwdTcThreads = 320;

__global__ void __launch_bounds__(kAttnBwdTcThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmKV, const __grid_constant__ CUtensorMap tmKVlo,
                       const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQlo,
                       const __grid_constant__ CUtensorMap tmDA, const __grid_constant__ CUtensorMap tmDAlo,
                       const __grid_constant__ CUtensorMap tmDKV, const __grid_constant__ CUtensorMap tmDKVlo,
                       const AttnBwdArgs a) {
  using L = AttnBwdTcSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* lse_s = reinterpret_cast<float*>(smem + L::OFF_LSE);
  float* del_s = lse_s + 32;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;           // queries landed
  uint64_t* kv_full = bars + 1;      // [2]
  uint64_t* sp_full = bars + 5;      // [2] S^T | dP^T computed
  uint64_t* sp_empty = bars + 7;     // [2] S^T | dP^T read by the 4 epilogue warps
  uint64_t* pd_full = bars + 9;      // P^T, dS^T staged by the 4 softmax warps
  uint64_t* dvk_full = bars + 10;    // [2] dV, dK (and dQ^T so far) computed; the staging and the K|V
                                     //     stage of the block are free again
  uint64_t* dvk_empty = bars + 12;   // [2] dV, dK read by the 4 drain warps
  uint64_t* fin = bars + 14;         // every MMA issued has completed (unwinding)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x, head = blockIdx.y;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&sp_full[i], 1);
      mbar_init(&sp_empty[i], 4);
    }
    mbar_init(pd_full, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&dvk_full[i], 1);
      mbar_init(&dvk_empty[i], 4);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  // ---- this CTA's example and rows (uniform across the CTA) ----
  const int U = a.cstart[a.B];
  bool active = chunk < U;
  int b = 0;
  long long k0 = 0, k1 = 0;
  if (active) {
    int lo = 0, hi = a.B - 1;  // largest b with cstart[b] <= chunk
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.cstart[mid] <= chunk) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
    auto clampo = [&](int e) -> long long {
      long long o = a.offsets[e];
      return o < 0 ? 0 : (o > a.total_L ? a.total_L : o);
    };
    const long long lo_b = clampo(b);
    long long hi_b = clampo(b + 1);
    if (hi_b < lo_b) hi_b = lo_b;
    k0 = lo_b + (long long)(chunk - a.cstart[b]) * a.chunk;
    k1 = min(hi_b, k0 + a.chunk);
    active = k0 < k1;
  }
  const int nblk = active ? (int)((k1 - k0 + 127) / 128) : 0;
  const int colk = head * 64, colv = a.v_col0 + head * 64;

  // TMEM columns
  const uint32_t t_sp = tmem_base;          // [2][S^T 32 | dP^T 32]
  const uint32_t t_dv = tmem_base + 128;    // [2][64]
  const uint32_t t_dk = tmem_base + 256;    // [2][64]
  const uint32_t t_dq = tmem_base + 384;    // 64 (dQ^T: lanes = (K hi | K lo) x d_h, columns = (dS hi | dS lo) x queries)

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && nblk > 0) {
      tma_prefetch_desc(&tmKV);
      tma_prefetch_desc(&tmKVlo);
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmDA);
      const int qrow = b * a.N;
      mbar_arrive_expect_tx(q_full, 4 * L::TILE_Q);
      tma_load_2d(smem + L::OFF_Q + 0 * L::TILE_Q, &tmQ, colk, qrow, q_full);
      tma_load_2d(smem + L::OFF_Q + 1 * L::TILE_Q, &tmQlo, colk, qrow, q_full);
      tma_load_2d(smem + L::OFF_Q + 2 * L::TILE_Q, &tmDA, colk, qrow, q_full);
      tma_load_2d(smem + L::OFF_Q + 3 * L::TILE_Q, &tmDAlo, colk, qrow, q_full);
      const uint32_t kv_bytes = (a.shared_kv ? 2 : 4) * L::TILE_KV;
      int issued = 0;
      for (int blk = 0; blk < nblk; ++blk, ++issued) {
        const int s = blk & 1, u = blk >> 1;
        if (blk >= 2 && !mbar_wait(&dvk_full[s], (u - 1) & 1, abort_flag)) break;  // block blk - 2 is done
        uint8_t* st = smem + L::OFF_KV + s * 4 * L::TILE_KV;
        const int r0 = (int)(k0 + 128ll * blk);
        mbar_arrive_expect_tx(&kv_full[s], kv_bytes);
        tma_load_2d(st + 0 * L::TILE_KV, &tmKV, colk, r0, &kv_full[s]);
        tma_load_2d(st + 1 * L::TILE_KV, &tmKVlo, colk, r0, &kv_full[s]);
        if (!a.shared_kv) {
          tma_load_2d(st + 2 * L::TILE_KV, &tmKV, colv, r0, &kv_full[s]);
          tma_load_2d(st + 3 * L::TILE_KV, &tmKVlo, colv, r0, &kv_full[s]);
        }
      }
      if (*abort_flag) {  // let the copies in flight land before the CTA exits
        volatile int quiet = 0;
        mbar_wait(q_full, 0, &quiet, 100000000ull);
        for (int k = (issued > 2 ? issued - 2 : 0); k < issued; ++k)
          mbar_wait(&kv_full[k & 1], (k >> 1) & 1, &quiet, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && nblk > 0) {
      constexpr uint32_t id_sp = idesc_bf16_f32(128, 32);                            // K-major A and B
      constexpr uint32_t id_kv = idesc_bf16_f32(128, 64) | kIdescBMnMajor;           // dV, dK
      constexpr uint32_t id_dq = idesc_bf16_f32(128, 64) | kIdescAMnMajor | kIdescBMnMajor;  // dQ^T
      const uint32_t q_s = smem_u32(smem + L::OFF_Q);
      const uint32_t ql_s = q_s + L::TILE_Q, da_s = q_s + 2 * L::TILE_Q, dal_s = q_s + 3 * L::TILE_Q;
      const uint32_t stg = smem_u32(smem + L::OFF_STG);
      const uint32_t p_s = stg, pl_s = stg + 64, ds_s = stg + L::TILE_KV, dsl_s = stg + L::TILE_KV + 64;
      bool ok = mbar_wait(q_full, 0, abort_flag);
      // S^T and dP^T of block `blk` into buffer blk & 1
      auto issue_sp = [&](int blk) -> bool {
        const int s = blk & 1, u = blk >> 1;
        if (!mbar_wait(&kv_full[s], u & 1, abort_flag)) return false;
        if (blk >= 2 && !mbar_wait(&sp_empty[s], (u - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kst = smem_u32(smem + L::OFF_KV + s * 4 * L::TILE_KV);
        const uint32_t k_s = kst, kl_s = kst + L::TILE_KV;
        const uint32_t v_s = a.shared_kv ? k_s : kst + 2 * L::TILE_KV;
        const uint32_t vl_s = a.shared_kv ? kl_s : kst + 3 * L::TILE_KV;
        const uint32_t d_s = t_sp + s * 64, d_p = t_sp + s * 64 + 32;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = kk > 0 ? 1u : 0u;
          umma_f16(d_s, sdesc_k_sw128(k_s + kk * 32), sdesc_k_sw128(q_s + kk * 32), id_sp, acc);
          umma_f16(d_s, sdesc_k_sw128(kl_s + kk * 32), sdesc_k_sw128(q_s + kk * 32), id_sp, 1u);
          umma_f16(d_s, sdesc_k_sw128(k_s + kk * 32), sdesc_k_sw128(ql_s + kk * 32), id_sp, 1u);
          umma_f16(d_p, sdesc_k_sw128(v_s + kk * 32), sdesc_k_sw128(da_s + kk * 32), id_sp, acc);
          umma_f16(d_p, sdesc_k_sw128(vl_s + kk * 32), sdesc_k_sw128(da_s + kk * 32), id_sp, 1u);
          umma_f16(d_p, sdesc_k_sw128(v_s + kk * 32), sdesc_k_sw128(dal_s + kk * 32), id_sp, 1u);
        }
        umma_commit(&sp_full[s]);
        return true;
      };
      if (ok) ok = issue_sp(0);
      int sp_next = 1;  // the next block whose S^T | dP^T is to be issued
      // S^T | dP^T of the next block goes ahead of this block's products when its K|V stage has landed
      // (the stage is refilled only after the MMAs of two blocks back are complete)
      auto sp_ready = [&](int nb) {
        return mbar_test(&kv_full[nb & 1], (nb >> 1) & 1) &&
               (nb < 2 || mbar_test(&sp_empty[nb & 1], ((nb >> 1) - 1) & 1));
      };
      for (int blk = 0; blk < nblk && ok; ++blk) {
        if (sp_next == blk + 1 && sp_next < nblk && sp_ready(sp_next)) {
          if (!issue_sp(sp_next)) break;
          ++sp_next;
        }
        if (!mbar_wait(pd_full, blk & 1, abort_flag)) break;
        const int db = blk & 1;  // dV|dK buffer
        if (blk >= 2 && !mbar_wait(&dvk_empty[db], ((blk >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const int s = blk & 1;
        const uint32_t k_s = smem_u32(smem + L::OFF_KV + s * 4 * L::TILE_KV);
        // dV = P^T dA and dK = (dS^T / sqrt(d_h)) Q: K = 32 queries (two k-steps); with shared K = V
        // both accumulate into dV's columns
        const uint32_t d_v = t_dv + db * 64;
        const uint32_t d_k = a.shared_kv ? d_v : t_dk + db * 64;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint32_t acc = kk > 0 ? 1u : 0u;
          const uint64_t bda = sdesc_mn_sw128(da_s + kk * 2048, 8192, 1024);
          const uint64_t bdal = sdesc_mn_sw128(dal_s + kk * 2048, 8192, 1024);
          const uint64_t bq = sdesc_mn_sw128(q_s + kk * 2048, 8192, 1024);
          const uint64_t bql = sdesc_mn_sw128(ql_s + kk * 2048, 8192, 1024);
          umma_f16(d_v, sdesc_k_sw128(p_s + kk * 32), bda, id_kv, acc);
          umma_f16(d_v, sdesc_k_sw128(pl_s + kk * 32), bda, id_kv, 1u);
          umma_f16(d_v, sdesc_k_sw128(p_s + kk * 32), bdal, id_kv, 1u);
          const uint32_t acck = a.shared_kv ? 1u : acc;
          umma_f16(d_k, sdesc_k_sw128(ds_s + kk * 32), bq, id_kv, acck);
          umma_f16(d_k, sdesc_k_sw128(dsl_s + kk * 32), bq, id_kv, 1u);
          umma_f16(d_k, sdesc_k_sw128(ds_s + kk * 32), bql, id_kv, 1u);
        }
        // dQ^T += K^T (dS^T / sqrt(d_h)), all four hi/lo products in one MMA per k-step: A = the K
        // tile MN-major (M = 128: the K hi tile's 64 d_h, then the K lo tile's, one tile apart), B =
        // the dS^T tile MN-major (N = 64: its hi then lo queries), K = the block's 128 rows
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (blk > 0 || kk > 0) ? 1u : 0u;
          umma_f16(t_dq, sdesc_mn_sw128(k_s + kk * 2048, L::TILE_KV, 1024), sdesc_mn_sw128(ds_s + kk * 2048, 8192, 1024),
                   id_dq, acc);
        }
        umma_commit(&dvk_full[db]);  // dV, dK, dQ^T so far; the staging tiles and the K|V stage are free
        if (sp_next == blk + 1 && sp_next < nblk) {
          if (!issue_sp(sp_next)) break;
          ++sp_next;
        }
      }
      umma_commit(fin);  // arrives once every MMA issued above has completed
      volatile int quiet = 0;
      mbar_wait(fin, 0, &quiet, 100000000ull);
    }
  } else if (warp < 6 && nblk > 0) {
    // ---------------- softmax backward (warps 2..5) ----------------
    const int qd = warp & 3;
    const int rloc = qd * 32 + lane;  // block row of this thread (= TMEM lane)
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    // lse (+inf past N: p = 0) and delta of this head
    if (warp == 2) {
      const long long idx = ((long long)b * a.N + lane) * a.n_heads + head;
      lse_s[lane] = lane < a.N ? a.lse[idx] : INFINITY;
      del_s[lane] = lane < a.N ? a.delta[idx] : 0.f;
    }
    named_bar_sync(1, 128);
    uint8_t* rowp = smem + L::OFF_STG + rloc * 128;  // this thread's row of each staging tile
    const uint32_t sw = (uint32_t)(rloc & 7);
    // P^T and dS^T / sqrt(d_h) of one block for this row as bf16 pairs
    uint32_t ph[16], pl[16], dh[16], dl[16];
    auto softmax = [&](int blk) -> bool {
      const int s = blk & 1, u = blk >> 1;
      if (!mbar_wait(&sp_full[s], u & 1, abort_flag)) return false;
      tc_fence_after();
      uint32_t sv[32], dpv[32];
      tmem_ld_32x32b_x32(t_sp + s * 64 + lane_off, sv);
      tmem_ld_32x32b_x32(t_sp + s * 64 + 32 + lane_off, dpv);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sp_empty[s]);
      const bool row_ok = k0 + 128ll * blk + rloc < k1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float p0 = 0.f, p1 = 0.f, g0 = 0.f, g1 = 0.f;
        if (row_ok) {
          p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * j]), a.scale_log2, -lse_s[2 * j]));
          p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * j + 1]), a.scale_log2, -lse_s[2 * j + 1]));
          g0 = p0 * (__uint_as_float(dpv[2 * j]) - del_s[2 * j]) * a.scale;
          g1 = p1 * (__uint_as_float(dpv[2 * j + 1]) - del_s[2 * j + 1]) * a.scale;
        }
        split2(p0, p1, ph[j], pl[j]);
        split2(g0, g1, dh[j], dl[j]);
      }
      return true;
    };
    bool ok = softmax(0);
    for (int blk = 0; blk < nblk && ok; ++blk) {
      // the staging is free once the previous block's MMAs have completed
      if (blk >= 1 && !mbar_wait(&dvk_full[(blk - 1) & 1], ((blk - 1) >> 1) & 1, abort_flag)) break;
      // P^T and dS^T in the K-major 128-byte-swizzled layout (row rloc: 16-byte chunk c at position
      // c ^ (rloc % 8)); the hi halves of queries 0..31 fill chunks 0..3, the lo halves chunks 4..7
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t oh = ((uint32_t)c ^ sw) * 16, ol = ((uint32_t)(c + 4) ^ sw) * 16;
        *reinterpret_cast<uint4*>(rowp + oh) = make_uint4(ph[4 * c], ph[4 * c + 1], ph[4 * c + 2], ph[4 * c + 3]);
        *reinterpret_cast<uint4*>(rowp + ol) = make_uint4(pl[4 * c], pl[4 * c + 1], pl[4 * c + 2], pl[4 * c + 3]);
        *reinterpret_cast<uint4*>(rowp + L::TILE_KV + oh) = make_uint4(dh[4 * c], dh[4 * c + 1], dh[4 * c + 2], dh[4 * c + 3]);
        *reinterpret_cast<uint4*>(rowp + L::TILE_KV + ol) = make_uint4(dl[4 * c], dl[4 * c + 1], dl[4 * c + 2], dl[4 * c + 3]);
      }
      fence_proxy_async_smem();  // the MMAs read the staging through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(pd_full);
      // the next block's softmax runs while this block's MMAs do
      if (blk + 1 < nblk) ok = softmax(blk + 1);
    }
  } else if (nblk > 0) {
    // ---------------- dK|dV drain (warps 6..9) ----------------
    const int qd = warp & 3;
    const int rloc = qd * 32 + lane;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const int nw = a.shared_kv ? 1 : 2;
    const uint32_t sw = (uint32_t)(lane & 7);
    uint8_t* dst = smem + L::OFF_DST + qd * 8192;  // this warp's staging: hi then lo, 32 rows of 128 bytes
    uint8_t* rowp = dst + lane * 128;
    int done = 0;  // blocks drained (all of them unless a wait ran out)
    for (int blk = 0; blk < nblk; ++blk) {
      const int db = blk & 1;
      const long long row = k0 + 128ll * blk + rloc;
      const bool row_ok = row < k1;
      const float rs = (a.row_scale && row_ok) ? a.row_scale[row] : 1.0f;  // before the wait
      const long long slice0 = k0 + 128ll * blk + qd * 32;
      const bool full_slice = slice0 + 32 <= k1;  // uniform across the warp
      if (!mbar_wait(&dvk_full[db], (blk >> 1) & 1, abort_flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int which = 0; which < nw; ++which) {
        // dK (which 0; with shared K = V, dK + dV in dV's columns) and dV (which 1), rows scaled by r
        const uint32_t tsrc = a.shared_kv ? t_dv + db * 64 : (which == 0 ? t_dk : t_dv) + db * 64;
        const int gcol = which == 0 ? colk : colv;
        uint32_t v0[32], v1[32];
        tmem_ld_32x32b_x32(tsrc + lane_off, v0);
        tmem_ld_32x32b_x32(tsrc + 32 + lane_off, v1);
        tmem_ld_wait();
        if (which == nw - 1) {  // this TMEM buffer may take block blk + 2
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dvk_empty[db]);
        }
        if (full_slice) {  // the staging's previous stores have read it
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t* v = c < 4 ? v0 + 8 * c : v1 + 8 * (c - 4);
          uint32_t h[4], l[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            split2(__uint_as_float(v[2 * j]) * rs, __uint_as_float(v[2 * j + 1]) * rs, h[j], l[j]);
          if (full_slice) {  // 128-byte-swizzled rows of the staging (hi, lo)
            const uint32_t off = ((uint32_t)c ^ sw) * 16;
            *reinterpret_cast<uint4*>(rowp + off) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(rowp + 4096 + off) = make_uint4(l[0], l[1], l[2], l[3]);
          } else if (row_ok) {
            reinterpret_cast<uint4*>(a.dkv + row * a.kvw + gcol)[c] = make_uint4(h[0], h[1], h[2], h[3]);
            reinterpret_cast<uint4*>(a.dkv_lo + row * a.kvw + gcol)[c] = make_uint4(l[0], l[1], l[2], l[3]);
          }
        }
        if (full_slice) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmDKV, dst, gcol, (int)slice0);
            tma_store_2d(&tmDKVlo, dst + 4096, gcol, (int)slice0);
            bulk_commit();
          }
        }
      }
      done = blk + 1;
    }
    if (lane == 0) bulk_wait<0>();  // this warp's tensor stores are complete: its staging is free
    __syncwarp();
    // dq += this chunk's share once the last block's MMAs are complete (its dvk_full, waited above):
    // quadrant qd holds d_h indices 32 (qd % 2) + lane of K hi (qd < 2) or K lo (qd >= 2); columns
    // 0..31 are the dS hi products of queries 0..31, columns 32..63 the dS lo ones. Quadrants 2 and 3
    // hand their sums to quadrants 0 and 1 through their staging; those add them to dq.
    const bool ok_dq = done == nblk && *abort_flag == 0;
    float* xch = reinterpret_cast<float*>(smem + L::OFF_DST + ((qd & 1) + 2) * 8192);  // [32 queries][32 lanes]
    int* xok = reinterpret_cast<int*>(xch + 32 * 32);
    float sum[32];
    if (ok_dq) {
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld_32x32b_x32(t_dq + lane_off, v0);
      tmem_ld_32x32b_x32(t_dq + 32 + lane_off, v1);
      tmem_ld_wait();
#pragma unroll
      for (int n = 0; n < 32; ++n) sum[n] = __uint_as_float(v0[n]) + __uint_as_float(v1[n]);
    }
    if (qd >= 2) {
      if (ok_dq) {
#pragma unroll
        for (int n = 0; n < 32; ++n) xch[n * 32 + lane] = sum[n];
      }
      if (lane == 0) *xok = ok_dq ? 1 : 0;
    }
    named_bar_sync(2, 128);  // the four drain warps (every one reaches it)
    if (qd < 2 && ok_dq && *xok) {
      const int m = qd * 32 + lane;  // d_h index
#pragma unroll
      for (int n = 0; n < 32; ++n)
        if (n < a.N) atomicAdd(a.dq + ((long long)b * a.N + n) * a.d + colk + m, sum[n] + xch[n * 32 + lane]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace whale
