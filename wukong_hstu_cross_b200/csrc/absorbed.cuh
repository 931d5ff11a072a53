// absorbed.cuh — Eq. (4) of WHALE with the key and value projections folded into the queries
// (gist.science technical summary of WHALE, section 2.1 "Core Architecture", Attention-Based
// Fusion Module; pith.science verdict, "key_machinery"). For query q = (head j, token n) of
// example b and history row t with RMSNorm row factor r_t = 1/sqrt(mean(H_t^2) + eps):
//
//   q_j . K_{t,j} / sqrt(d_h) = r_t * (H_t . qa_q),     qa_q = diag(g_kv) W_K,j^T q_j / sqrt(d_h)
//   sum_t p_{q,t} V_{t,j}     = (sum_t p_{q,t} r_t H_t) . diag(g_kv) W_V,j^T = z_q W'_V,j^T
//
// which is exact algebra. Per history row this costs 2 * (N h) * d multiply-adds instead of the
// 2 d^2 of projecting K and V (and no K|V tensor is written or re-read), so it is the path taken
// when N h <= d. Work is done in units of 256 history rows of one example by a CTA pair (cluster
// of two, cta_group::2 MMAs; CTA r holds queries [128 r, 128 r + 128) of the example's 256):
//
//   pass A  S = qa H_u^T (M = 256 queries, N = 256 rows, K = d), r_t applied per column, online
//           softmax per query in base 2 with a lazy reference (raised only when a tile maximum
//           exceeds it by kAbsLazy): writes pw = p * r_t (bf16), the reference of every unit, and
//           (m, l) of every segment.
//   pass B  z += pw_u H_u (M = 256 queries, N = d, K = 256 rows; H as an MN-major operand),
//           rescaling the TMEM accumulator whenever pass A raised a reference; writes z / l of
//           examples held by one pair, or an unnormalised partial.
//   merge   combines the partials of examples split across pairs (log-sum-exp weights).
//
// The weights pw are stored tiled: the 64 history rows c of unit u form tile 4u + c, rows
// (4u + c) * 256 + query, 64 columns, so every TMA box of them is one contiguous block.
// Both passes give the P pairs contiguous ranges of the flattened unit index (units of example b
// are [ustart[b], ustart[b+1])); a range cut inside an example makes a partial segment, stored
// in slot 2p (the range's first segment) or 2p + 1 (its last).
#pragma once

#include <type_traits>

#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace whale {

constexpr int kAbsRows = 256;      // history rows per unit
constexpr int kAbsQ = 256;         // absorbed queries per example (N * h)
constexpr int kAbsMaxPairs = 74;   // CTA pairs of one launch (one CTA per SM)
constexpr float kAbsLazy = 8.0f;   // log2 headroom before the softmax reference is raised
constexpr float kAbsRedo = 64.0f;  // log2 excess above which a unit's weights are rewritten

struct AbsArgs {
  const int* offsets;       // [B+1]
  const int* ustart;        // [B+1] first unit of each example; ustart[B] = number of units
  int B, N, d;              // examples, tokens per example, width
  int n_pairs;
  long long total_L;
  float inv_d, eps;
  float* mref;              // [units_max, 256] softmax reference of each unit (log2 units)
  float* stats_whole;       // [B, 256] (m, l) of examples held by one pair
  float* stats_part;        // [2 * n_pairs, 256] (m, l) of partial segments
  __nv_bfloat16* part_z;    // [2 * n_pairs, 256, d] unnormalised z of partial segments (bf16)
  __nv_bfloat16* z_hi;      // [h, B*N, d] z / l, bf16 (row j*B*N + b*N + n)
  const int* pstart;        // [n_pairs][8]: u0, u1, b, ub, ub1 of each pair's range (null: searched)
  // [2 + n_pairs]: pairs of pass A in the order they finished (p + 1; 0 = not yet) after two counters
  // (entries published, entries taken). Null: pass B waits for the whole of pass A instead.
  int* pq;
};

__device__ __forceinline__ long long abs_off(const AbsArgs& a, int b) {
  long long o = a.offsets[b];
  return o < 0 ? 0 : (o > a.total_L ? a.total_L : o);
}

// U * p < 2^31: units_max < 2^31 / 256 (checked on the host) and P <= kAbsMaxPairs.
__device__ __forceinline__ int abs_range_start(int U, int P, int p) { return (int)(((unsigned)U * (unsigned)p) / (unsigned)P); }

// Pair whose range holds unit u (0 <= u < U).
__device__ __forceinline__ int abs_pair_of(int u, int U, int P) {
  int p = (int)(((long long)u * P) / U);
  if (p > P - 1) p = P - 1;
  while (p + 1 < P && abs_range_start(U, P, p + 1) <= u) ++p;
  while (p > 0 && abs_range_start(U, P, p) > u) --p;
  return p;
}

// Walk over the units [u0, u1) of one pair, tracking the example they belong to.
struct AbsWalk {
  int u, u0, u1, p;
  int b, ub, ub1;  // example of u and its unit range
  __device__ __forceinline__ void init(const AbsArgs& a, int p_) {
    p = p_;
    if (a.pstart != nullptr) {  // tabulated once per forward by abs_units_kernel
      const int4 e = *reinterpret_cast<const int4*>(a.pstart + 8 * p);
      u0 = e.x;
      u1 = e.y;
      b = e.z;
      ub = e.w;
      ub1 = a.pstart[8 * p + 4];
      u = u0;
      return;
    }
    const int U = a.ustart[a.B];
    u0 = abs_range_start(U, a.n_pairs, p);
    u1 = abs_range_start(U, a.n_pairs, p + 1);
    u = u0;
    b = 0;
    ub = ub1 = 0;
    if (u < u1) {
      int lo = 0, hi = a.B - 1;  // largest b with ustart[b] <= u (non-empty since u < ustart[B])
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.ustart[mid] <= u) lo = mid;
        else hi = mid - 1;
      }
      b = lo;
      ub = a.ustart[b];
      ub1 = a.ustart[b + 1];
    }
  }
  __device__ __forceinline__ bool valid() const { return u < u1; }
  __device__ __forceinline__ void next(const AbsArgs& a) {
    ++u;
    if (u < u1 && u >= ub1) {
      do {
        ++b;
      } while (a.ustart[b + 1] <= u);
      ub = a.ustart[b];
      ub1 = a.ustart[b + 1];
    }
  }
};

struct AbsUnit {
  int b, t, nvalid, ptile0, slot;  // ptile0: first 64-row weight tile of the unit (4 per unit)
  long long row0;            // first history row of the unit
  bool first, last, whole;   // first / last unit of its segment; segment = the whole example
};

__device__ __forceinline__ AbsUnit abs_unit(const AbsArgs& a, const AbsWalk& w) {
  AbsUnit un;
  un.b = w.b;
  un.t = w.u - w.ub;
  const long long lo = abs_off(a, w.b);
  long long hi = abs_off(a, w.b + 1);
  if (hi < lo) hi = lo;
  un.row0 = lo + (long long)kAbsRows * un.t;
  const long long nv = hi - un.row0;
  un.nvalid = nv > kAbsRows ? kAbsRows : (nv < 1 ? 1 : (int)nv);
  un.ptile0 = w.u * (kAbsRows / 64);
  un.first = (w.u == w.u0) || (un.t == 0);
  un.last = (w.u == w.u1 - 1) || (w.u == w.ub1 - 1);
  un.whole = (w.u0 <= w.ub) && (w.u1 >= w.ub1);
  un.slot = (w.u0 >= w.ub) ? 2 * w.p : 2 * w.p + 1;
  return un;
}

// ustart[b] = sum_{b' < b} ceil(L_b' / 256), capped at units_max (only inconsistent offsets reach
// the cap; they lose rows, never index past the buffers). One block of 1024 threads.
// With P > 0 it also tabulates each of the P pairs' starting state for AbsWalk (pstart[p][0..4] =
// u0, u1, the example b of unit u0, ustart[b], ustart[b + 1]), so the passes start without a search,
// and clears pq, the order in which the pairs of pass A finish.
__global__ void __launch_bounds__(1024) abs_units_kernel(const int* __restrict__ offsets, int B, long long total_L,
                                                         int units_max, int* __restrict__ ustart, int P,
                                                         int* __restrict__ pstart, int* __restrict__ pq) {
  pdl_wait();
  pdl_trigger();
  __shared__ int part[1024];
  const int per = (B + 1023) / 1024;
  const int b0 = threadIdx.x * per, b1 = min(B, b0 + per);
  auto clampo = [&](int b) -> long long {
    long long o = offsets[b];
    return o < 0 ? 0 : (o > total_L ? total_L : o);
  };
  long long sum = 0;
  for (int b = b0; b < b1; ++b) {
    const long long L = clampo(b + 1) - clampo(b);
    if (L > 0) sum += (L + kAbsRows - 1) / kAbsRows;
  }
  part[threadIdx.x] = (int)(sum < units_max ? sum : units_max);
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {  // inclusive scan (values capped, no overflow)
    const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] = min(part[threadIdx.x] + v, units_max);
    __syncthreads();
  }
  long long run = threadIdx.x > 0 ? part[threadIdx.x - 1] : 0;
  for (int b = b0; b < b1; ++b) {
    ustart[b] = (int)run;
    const long long L = clampo(b + 1) - clampo(b);
    if (L > 0) run += (L + kAbsRows - 1) / kAbsRows;
    if (run > units_max) run = units_max;
  }
  if (threadIdx.x == 1023) ustart[B] = part[1023];
  if (P <= 0) return;
  // The finishing order of pass A (ordering: this clear -> pass A, which waits on its predecessor,
  // so on this kernel transitively -> pass A publishes -> pass B acquires -> the merge clears again).
  for (int i = threadIdx.x; i < 2 + P; i += blockDim.x) pq[i] = 0;
  __syncthreads();  // ustart written by this block is visible to it
  const int U = __ldcg(ustart + B);
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const int u0 = abs_range_start(U, P, p), u1 = abs_range_start(U, P, p + 1);
    int b = 0, ub = 0, ub1 = 0;
    if (u0 < u1) {
      int lo = 0, hi = B - 1;  // largest b with ustart[b] <= u0
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldcg(ustart + mid) <= u0) lo = mid;
        else hi = mid - 1;
      }
      b = lo;
      ub = __ldcg(ustart + b);
      ub1 = __ldcg(ustart + b + 1);
    }
    int* e = pstart + 8 * p;
    e[0] = u0;
    e[1] = u1;
    e[2] = b;
    e[3] = ub;
    e[4] = ub1;
  }
}

// ================================================================================================
// pass A: S = qa H^T, online softmax, pw = p * r
// ================================================================================================
// Columns of one weight store (the staging tile of an epilogue warp is 32 queries x kAbsEpiCols):
// 64 (128-byte rows, 128-byte swizzle), 32 (64-byte rows, 64-byte swizzle) or 16 (32-byte rows,
// 32-byte swizzle). Each halving of the staging memory leaves room for more stages of history rows
// at d = 512 (3, 4, 5) at the price of twice the stores and proxy fences; 32 measured fastest
// (4 us per layer ahead of 16, 9 us ahead of 64).
constexpr int kAbsEpiCols = 32;
// The softmax of full 32-column chunks in packed f32x2 arithmetic (scale, shift, sums and weights of
// two scores per instruction) with 3-input maxima: fewer issue slots in the epilogue that bounds
// pass A.
constexpr bool kAbsPackedSoftmax = true;
// Pass A prefetches history rows into L2 this many 64-column blocks ahead of its stage loads (one
// prefetch per load): lookahead beyond what the shared-memory ring holds. 0 disables it.
constexpr int kAbsPrefetchKb = 4;
// Pass B: the same, in 64-row chunks (weights tile and this CTA's columns of the history rows).
constexpr int kAbsBPrefetchCh = 1;

template <int E>  // d = 256 E
struct AbsASmem {
  static constexpr int BK = 64;
  static constexpr int KB = 4 * E;                     // 64-column blocks of d
  static constexpr uint32_t BLK_BYTES = 128 * BK * 2;  // 128 rows x 64 columns
  static constexpr uint32_t QA_BYTES = KB * BLK_BYTES; // this CTA's 128 absorbed queries, all of d
  static constexpr uint32_t STAGE_BYTES = BLK_BYTES;   // this CTA's 128 history rows, one column block
  static constexpr uint32_t EPI_WARP = 32 * kAbsEpiCols * 2;
  static constexpr uint32_t EPI_BYTES = 8 * EPI_WARP;
  static constexpr int XCH = 2 * 256 * 4 + 2 * 2 * 128 * 4 + 2 * 128 * 4;  // r[2][256], max[2][2][128], l[2][128]
  static constexpr int FIXED = 1024 + QA_BYTES + EPI_BYTES + XCH + 512;
  static constexpr int STAGES = (232448 - FIXED) / (int)STAGE_BYTES > 8 ? 8 : (232448 - FIXED) / (int)STAGE_BYTES;
  static constexpr size_t BYTES = FIXED + STAGES * (size_t)STAGE_BYTES;
  static_assert(STAGES >= 3, "at least three stages of history rows");
  // full/ready/empty per stage; tfull, tempty, nfull, edone, eloc [2]; xbar [8]; lbar [4]; qfull,
  // qempty; then the TMEM address slot and the abort flag
  static_assert(3 * STAGES * 8 + 24 * 8 + 8 <= 512, "barriers fit their area");
};
constexpr int kAbsAThreads = 512;

// The absorbed queries of the example (the MMA's A operand, 128 per CTA) stay resident in shared
// memory for the pair's whole segment of that example: the stage ring carries history rows only,
// which halves the operand bytes streamed per MMA (TMA ingest bounds the loop, not the tensor pipe).
// warps: 0 TMA producer (both CTAs), 1 TMEM (2 x 256 columns) + MMA issue (even CTA), 2..9 softmax
// epilogue (two warps per lane quadrant, 128 columns each), 10..13 row statistics of this CTA's 128
// history rows (r of all 256 columns reaches both CTAs through distributed shared memory), 14 relay
// of "stage landed" (even CTA) as in the 2-SM projection GEMM, 15 forwarder of "epilogue done with
// the unit's row factors" to the peer CTA: a cluster-scope release costs about 0.7 us, so the
// epilogue warps arrive locally (CTA scope) and this warp issues the cluster-scope arrive.
template <int E>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAbsAThreads, 1)
    abs_scores_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmH,
                      const __grid_constant__ CUtensorMap tmP, const AbsArgs a) {
  using L = AbsASmem<E>;
  constexpr int ST = L::STAGES;
  constexpr int KB = L::KB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qsm = smem;                      // [KB][128 queries][64 columns], 128-byte swizzle
  uint8_t* stages = smem + L::QA_BYTES;     // [ST][128 history rows][64 columns]
  uint8_t* epi = stages + ST * L::STAGE_BYTES;
  float* rbuf = reinterpret_cast<float*>(epi + L::EPI_BYTES);  // [2][256]
  float* xmax = rbuf + 2 * 256;                                // [2 acc][2 half][128]
  float* xsum = xmax + 2 * 2 * 128;                            // [2 half][128]
  uint64_t* full = reinterpret_cast<uint64_t*>(xsum + 2 * 128);
  uint64_t* ready = full + ST;
  uint64_t* empty = ready + ST;
  uint64_t* tfull = empty + ST;   // [2]
  uint64_t* tempty = tfull + 2;   // [2] (even CTA: 8 + 8 epilogue warps)
  uint64_t* nfull = tempty + 2;   // [2] 4 local + 4 peer statistic warps
  uint64_t* edone = nfull + 2;    // [2] 8 local + 8 peer epilogue warps
  uint64_t* xbar = edone + 2;     // [4 quadrants][2 acc] tile maxima of both half-warps written
  uint64_t* lbar = xbar + 8;      // [4 quadrants] segment sums of both half-warps written
  uint64_t* qfull = lbar + 4;     // the segment's queries landed (both CTAs' copies, even CTA)
  uint64_t* qempty = qfull + 1;   // the segment's last MMAs are done (commit to both CTAs)
  uint64_t* eloc = qempty + 1;    // [2] the 8 local epilogue warps are done with the row factors
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(eloc + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 1);
      mbar_init(&empty[s], 1 + 4);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 16);
      mbar_init(&nfull[i], 8);
      mbar_init(&edone[i], 2);  // the forwarders of both CTAs
      mbar_init(&eloc[i], 8);
    }
    for (int i = 0; i < 8; ++i) mbar_init(&xbar[i], 2);
    for (int i = 0; i < 4; ++i) mbar_init(&lbar[i], 2);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmP);
  }
  if (warp == 1) {
    tmem_alloc_cg2(tmem_slot, 512);
    tmem_relinquish_cg2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  AbsWalk wk;
  wk.init(a, pair);

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int kg = 0, nseg = 0;
      bool stop = false;
      const uint32_t qbar = mapa_shared(smem_u32(qfull), 0);
      // prefetch cursor (unit pf, block pkb), kAbsPrefetchKb blocks ahead of the loads
      AbsWalk pf = wk;
      int pkb = 0, prow = pf.valid() ? (int)abs_unit(a, pf).row0 : 0;
      auto pf_advance = [&]() {
        if (++pkb == KB) {
          pkb = 0;
          pf.next(a);
          if (pf.valid()) prow = (int)abs_unit(a, pf).row0;
        }
      };
      for (int i = 0; i < kAbsPrefetchKb && pf.valid(); ++i) pf_advance();
      for (; wk.valid() && !stop; wk.next(a)) {
        const AbsUnit un = abs_unit(a, wk);
        if (un.first) {
          // a new segment: its queries replace the previous segment's once those MMAs are done
          if (nseg > 0 && !mbar_wait(qempty, (nseg - 1) & 1, abort_flag)) break;
          if (leader) mbar_arrive_expect_tx(qfull, 2 * L::QA_BYTES);
          const int qrow = un.b * kAbsQ + (int)rank * 128;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) tma_load_2d_cg2(qsm + kb * L::BLK_BYTES, &tmQ, kb * L::BK, qrow, qbar);
          ++nseg;
        }
        const int hrow = (int)un.row0 + (int)rank * 128;
        for (int kb = 0; kb < KB; ++kb, ++kg) {
          const int s = kg % ST, u = kg / ST;
          if (kg >= ST && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag)) {
            stop = true;
            break;
          }
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * L::STAGE_BYTES);
          tma_load_2d_cg2(stages + s * L::STAGE_BYTES, &tmH, kb * L::BK, hrow, bar);
          if (kAbsPrefetchKb > 0 && pf.valid()) {
            tma_prefetch_l2_2d(&tmH, pkb * L::BK, prow + (int)rank * 128);
            pf_advance();
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (even CTA) ----------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256);
      int kg = 0, it = 0, nseg = 0;
      bool stop = false;
      for (; wk.valid() && !stop; wk.next(a), ++it) {
        const AbsUnit un = abs_unit(a, wk);
        const int acc = it & 1, ua = it >> 1;
        if (un.first) {
          if (!mbar_wait(qfull, nseg & 1, abort_flag)) break;
          ++nseg;
        }
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
          const uint32_t a_base = smem_u32(qsm + kb * L::BLK_BYTES);
          const uint32_t b_base = smem_u32(stages + s * L::STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < L::BK / 16; ++kk)
            umma_f16_cg2(d_tmem, sdesc_k_sw128(a_base + kk * 32), sdesc_k_sw128(b_base + kk * 32), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_cg2_mc(&empty[s], 0x3);
        }
        umma_commit_cg2_mc(&tfull[acc], 0x3);
        if (un.last) umma_commit_cg2_mc(qempty, 0x3);  // also on abort: arrives once issued MMAs are done
      }
    }
  } else if (warp == 15) {
    // ---------------- forwarder (both CTAs): local epilogue done -> both CTAs' edone ----------------
    if (lane == 0) {
      const uint32_t edone_peer0 = mapa_shared(smem_u32(&edone[0]), rank ^ 1);
      int it = 0;
      for (; wk.valid(); wk.next(a), ++it) {
        const int acc = it & 1, ua = it >> 1;
        if (!mbar_wait(&eloc[acc], ua & 1, abort_flag)) break;
        mbar_arrive(&edone[acc]);
        mbar_arrive_cluster_release(edone_peer0 + acc * 8);
      }
    }
  } else if (warp == 14) {
    // ---------------- relay (even CTA) ----------------
    if (leader && lane == 0) {
      const uint32_t peer_ready0 = mapa_shared(smem_u32(&ready[0]), 1);
      const int total = (wk.u1 - wk.u0) * KB;
      for (int kg = 0; kg < total; ++kg) {
        const int s = kg % ST, u = kg / ST;
        if (!mbar_wait(&full[s], u & 1, abort_flag)) break;
        mbar_arrive(&ready[s]);
        mbar_arrive_cluster(peer_ready0 + s * 8);
      }
    }
  } else if (warp >= 10) {
    // ---------------- row statistics of this CTA's 128 history rows (both CTAs) ----------------
    const int row = (warp & 3) * 32 + lane;
    const uint32_t rb_peer = mapa_shared(smem_u32(rbuf), rank ^ 1);
    const uint32_t nfull_peer0 = mapa_shared(smem_u32(&nfull[0]), rank ^ 1);
    int kg = 0, it = 0;
    for (; wk.valid(); wk.next(a), ++it) {
      const int acc = it & 1, ua = it >> 1;
      float ss = 0.f;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++kg) {
        const int s = kg % ST, u = kg / ST;
        if (!mbar_wait(&ready[s], u & 1, abort_flag)) {
          ok = false;
          break;
        }
        const uint4* rp = reinterpret_cast<const uint4*>(stages + s * L::STAGE_BYTES + row * 128);
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
      // both CTAs' epilogues must be done with this buffer before either side rewrites it
      if (it >= 2 && !mbar_wait_cluster(&edone[acc], (ua - 1) & 1, abort_flag)) break;
      const float rv = rsqrtf(ss * a.inv_d + a.eps);
      const int idx = acc * 256 + (int)rank * 128 + row;
      rbuf[idx] = rv;
      st_shared_cluster_f32(rb_peer + idx * 4, rv);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&nfull[acc]);
        mbar_arrive_cluster_release(nfull_peer0 + acc * 8);
      }
    }
  } else {
    // ---------------- softmax epilogue (warps 2..9, both CTAs) ----------------
    // The first unit of a segment takes its reference from its own tile maximum (a pass over TMEM
    // and an exchange with the partner half-warp). Later units write their weights with the
    // current reference in one pass and exchange the tile maximum afterwards: above the lazy
    // headroom the reference is raised for the following units (never at a segment's last unit,
    // whose reference is the segment's), and above kAbsRedo the unit is rewritten with the new
    // maximum so no weight exceeds 2^kAbsRedo.
    const int qd = warp & 3;
    const int hf = (warp - 2) >> 2;  // columns [128 hf, 128 hf + 128) of the unit
    const int row = qd * 32 + lane;
    const int qg = (int)rank * 128 + row;
    uint8_t* sbuf = epi + (warp - 2) * L::EPI_WARP;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);

    // maximum of r_t * s over the valid columns of this half
    auto tile_max = [&](uint32_t t0, const float* r, int nv) -> float {
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t0 + c * 32, v);
        tmem_ld_wait();
        const float4* r4 = reinterpret_cast<const float4*>(r + c * 32);
        const bool masked = c * 32 + 32 > nv;
        if (!masked) {  // four independent chains
          float m4[4] = {mx, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 rr = r4[i];
            m4[0] = fmaxf(m4[0], __uint_as_float(v[4 * i]) * rr.x);
            m4[1] = fmaxf(m4[1], __uint_as_float(v[4 * i + 1]) * rr.y);
            m4[2] = fmaxf(m4[2], __uint_as_float(v[4 * i + 2]) * rr.z);
            m4[3] = fmaxf(m4[3], __uint_as_float(v[4 * i + 3]) * rr.w);
          }
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          continue;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 rr = r4[i];
          const float x0 = __uint_as_float(v[4 * i]) * rr.x, x1 = __uint_as_float(v[4 * i + 1]) * rr.y;
          const float x2 = __uint_as_float(v[4 * i + 2]) * rr.z, x3 = __uint_as_float(v[4 * i + 3]) * rr.w;
          {
            const int col = c * 32 + 4 * i;
            if (col < nv) mx = fmaxf(mx, x0);
            if (col + 1 < nv) mx = fmaxf(mx, x1);
            if (col + 2 < nv) mx = fmaxf(mx, x2);
            if (col + 3 < nv) mx = fmaxf(mx, x3);
          }
        }
      }
      return mx;
    };
    // p = 2^(r s - m) over the valid columns (0 elsewhere): returns the local maximum of r s, adds
    // sum(p) to lsum, and stores pw = p * r (bf16) through the staging tile into the 64-column
    // tiles of the tiled weight layout (kAbsEpiCols columns per store).
    auto write_weights = [&](uint32_t t0, const float* r, int nv, float m, float& lsum, int tile_row0) -> float {
      float mx = -INFINITY;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
          const int c0 = cc * 64 + h2 * 32;
          // the packed path of 32-column stores waits for the staging buffer only once its
          // weights are in registers (the previous store's read then overlaps the arithmetic)
          const bool late_wait = kAbsPackedSoftmax && kAbsEpiCols == 32 && c0 + 32 <= nv;
          if (!late_wait && (kAbsEpiCols == 32 || (kAbsEpiCols == 64 && h2 == 0))) {
            if (lane == 0) bulk_wait_read<0>();  // the previous store from this buffer has read it
            __syncwarp();
          }
          uint32_t v[32];
          tmem_ld_32x32b_x32(t0 + c0, v);
          tmem_ld_wait();
          const float4* r4 = reinterpret_cast<const float4*>(r + c0);
          // Full 32-column chunks (all but the last of a ragged unit) skip the column test; four
          // independent maximum / sum chains per chunk.
          auto packed_chunk = [&]() {
            const uint64_t nm2 = f2pack(-m, -m);
            uint64_t lsa = f2pack(0.f, 0.f), lsb = lsa;
            float mxa = mx, mxb = -INFINITY;
            uint4 pks[4];
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
              uint32_t wpk[4];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const float4 rr = r4[2 * j8 + h];
                const int j = 8 * j8 + 4 * h;
                const uint64_t r01 = f2pack(rr.x, rr.y), r23 = f2pack(rr.z, rr.w);
                const uint64_t xr01 = fmul2(f2pack(__uint_as_float(v[j]), __uint_as_float(v[j + 1])), r01);
                const uint64_t xr23 = fmul2(f2pack(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3])), r23);
                float x0, x1, x2, x3, t0, t1, t2, t3;
                f2unpack(xr01, x0, x1);
                f2unpack(xr23, x2, x3);
                mxa = fmax3(mxa, x0, x1);
                mxb = fmax3(mxb, x2, x3);
                f2unpack(fadd2(xr01, nm2), t0, t1);
                f2unpack(fadd2(xr23, nm2), t2, t3);
                const uint64_t p01 = f2pack(fast_exp2(t0), fast_exp2(t1));
                const uint64_t p23 = f2pack(fast_exp2(t2), fast_exp2(t3));
                lsa = fadd2(lsa, p01);
                lsb = fadd2(lsb, p23);
                float w0, w1, w2, w3;
                f2unpack(fmul2(p01, r01), w0, w1);
                f2unpack(fmul2(p23, r23), w2, w3);
                wpk[2 * h] = pack_bf16x2(w0, w1);
                wpk[2 * h + 1] = pack_bf16x2(w2, w3);
              }
              pks[j8] = make_uint4(wpk[0], wpk[1], wpk[2], wpk[3]);
            }
            if (kAbsEpiCols == 32) {
              if (lane == 0) bulk_wait_read<0>();  // the previous store from this buffer has read it
              __syncwarp();
            }
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
              if (kAbsEpiCols == 64)
                reinterpret_cast<uint4*>(sbuf + lane * 128)[(h2 * 4 + j8) ^ (lane & 7)] = pks[j8];
              else
                reinterpret_cast<uint4*>(sbuf + lane * 64)[j8 ^ ((lane >> 1) & 3)] = pks[j8];
            }
            mx = fmaxf(mxa, mxb);
            float l0, l1, l2, l3;
            f2unpack(lsa, l0, l1);
            f2unpack(lsb, l2, l3);
            lsum += (l0 + l1) + (l2 + l3);
          };
          auto chunk = [&](auto masked_t) {
            constexpr bool kMasked = decltype(masked_t)::value;
            float mx4[4] = {mx, -INFINITY, -INFINITY, -INFINITY}, ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
              float w[8];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const float4 rr = r4[2 * j8 + h];
                const float rv[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const int j = 8 * j8 + 4 * h + k;
                  const float x = __uint_as_float(v[j]);
                  const float pexp = fast_exp2(fmaf(x, rv[k], -m));
                  if (!kMasked) {
                    mx4[k] = fmaxf(mx4[k], x * rv[k]);
                    ls4[k] += pexp;
                    w[4 * h + k] = pexp * rv[k];
                  } else {
                    const bool ok = c0 + j < nv;
                    mx4[k] = ok ? fmaxf(mx4[k], x * rv[k]) : mx4[k];
                    const float pv = ok ? pexp : 0.f;
                    ls4[k] += pv;
                    w[4 * h + k] = pv * (ok ? rv[k] : 0.f);
                  }
                }
              }
              uint4 pk;
              pk.x = pack_bf16x2(w[0], w[1]);
              pk.y = pack_bf16x2(w[2], w[3]);
              pk.z = pack_bf16x2(w[4], w[5]);
              pk.w = pack_bf16x2(w[6], w[7]);
              // row = lane; 16-byte chunk positions follow the store's swizzle (128-, 64- or 32-byte)
              if (kAbsEpiCols == 64) {
                reinterpret_cast<uint4*>(sbuf + lane * 128)[(h2 * 4 + j8) ^ (lane & 7)] = pk;
              } else if (kAbsEpiCols == 32) {
                reinterpret_cast<uint4*>(sbuf + lane * 64)[j8 ^ ((lane >> 1) & 3)] = pk;
              } else {
                if ((j8 & 1) == 0) {  // the previous store from this buffer has read it
                  if (lane == 0) bulk_wait_read<0>();
                  __syncwarp();
                }
                reinterpret_cast<uint4*>(sbuf + lane * 32)[(j8 & 1) ^ ((lane >> 2) & 1)] = pk;
                if (j8 & 1) {
                  fence_proxy_async_smem();
                  __syncwarp();
                  if (lane == 0) {
                    tma_store_2d(&tmP, sbuf, h2 * 32 + (j8 >> 1) * 16,
                                 (tile_row0 + hf * 2 + cc) * kAbsQ + (int)rank * 128 + qd * 32);
                    bulk_commit();
                  }
                }
              }
            }
            mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            lsum += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
          };
          if (c0 + 32 > nv) chunk(std::true_type{});
          else if (kAbsPackedSoftmax && kAbsEpiCols != 16) packed_chunk();
          else chunk(std::false_type{});
          if (kAbsEpiCols == 32 || (kAbsEpiCols == 64 && h2 == 1)) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmP, sbuf, kAbsEpiCols == 32 ? h2 * 32 : 0,
                           (tile_row0 + hf * 2 + cc) * kAbsQ + (int)rank * 128 + qd * 32);
              bulk_commit();
            }
          }
        }
      }
      return mx;
    };

    float m_run = 0.f, l_part = 0.f;
    int it = 0, nseg = 0;
    bool ok = true;
    for (; wk.valid() && ok; wk.next(a), ++it) {
      const AbsUnit un = abs_unit(a, wk);
      const int acc = it & 1, ua = it >> 1;
      if (!mbar_wait(&tfull[acc], ua & 1, abort_flag)) break;
      if (!mbar_wait_cluster(&nfull[acc], ua & 1, abort_flag)) break;
      tc_fence_after();
      const float* r = rbuf + acc * 256 + hf * 128;
      const uint32_t t0 = tmem_base + acc * 256 + hf * 128 + ((uint32_t)(qd * 32) << 16);
      const int nv = un.nvalid - hf * 128;  // valid columns of this half (may be <= 0)
      // tile maximum of both halves, through the quadrant's exchange barrier (bounded wait)
      auto exchange = [&](float mine) -> float {
        xmax[(acc * 2 + hf) * 128 + row] = mine;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xbar[qd * 2 + acc]);
        if (!mbar_wait(&xbar[qd * 2 + acc], ua & 1, abort_flag)) {
          ok = false;
          return mine;
        }
        return fmaxf(xmax[(acc * 2) * 128 + row], xmax[(acc * 2 + 1) * 128 + row]);
      };
      float m_use, l_unit = 0.f;
      if (un.first) {
        m_use = exchange(tile_max(t0, r, nv));
        if (!ok) break;
        l_part = 0.f;
        write_weights(t0, r, nv, m_use, l_unit, un.ptile0);
        m_run = m_use;
        l_part = l_unit;
      } else {
        m_use = m_run;
        const float mt = exchange(write_weights(t0, r, nv, m_use, l_unit, un.ptile0));
        if (!ok) break;
        if (mt > m_use + kAbsRedo) {
          // rewrite this unit with the new maximum (after the stores already issued completed)
          if (lane == 0) bulk_wait<0>();
          __syncwarp();
          l_unit = 0.f;
          write_weights(t0, r, nv, mt, l_unit, un.ptile0);
          l_part = l_part * fast_exp2(m_use - mt) + l_unit;
          m_use = m_run = mt;
        } else if (mt > m_use + kAbsLazy && !un.last) {
          l_part = (l_part + l_unit) * fast_exp2(m_use - mt);  // the following units use mt
          m_run = mt;
        } else {
          l_part += l_unit;
        }
      }
      float l_seg = 0.f;
      if (un.last) {
        xsum[hf * 128 + row] = l_part;
        __syncwarp();
        if (lane == 0) mbar_arrive(&lbar[qd]);
        if (!mbar_wait(&lbar[qd], nseg & 1, abort_flag)) break;
        ++nseg;
        l_seg = xsum[row] + xsum[128 + row];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(tempty0 + acc * 8);  // the even CTA's MMA may reuse this accumulator
        mbar_arrive(&eloc[acc]);                 // forwarded to both CTAs' edone by warp 15
      }
      // The unit's reference and the segment's (m, l) are for pass B and the merge (later kernels):
      // stored after the arrives, so the cluster-scope release above does not wait for them.
      if (hf == 0) {
        a.mref[(size_t)wk.u * kAbsQ + qg] = m_use;
        if (un.last) {
          float2* st = un.whole ? reinterpret_cast<float2*>(a.stats_whole) + (size_t)un.b * kAbsQ + qg
                                : reinterpret_cast<float2*>(a.stats_part) + (size_t)un.slot * kAbsQ + qg;
          *st = make_float2(m_use, l_seg);
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  if (a.pq != nullptr) {  // weights (bulk stores, complete above), references, statistics: to gpu scope
    fence_proxy_async_all();
    __threadfence();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_cg2(tmem_base, 512);
  }
  // Pass B reads only this pair's outputs: publish the pair as finished (both CTAs are past the
  // cluster barrier, so their writes are ordered before the release). The queue was cleared by a
  // kernel this one waited for (the unit starts, or the previous layer's merge), and pass B can only
  // have started after this grid's trigger, which follows its dependency wait.
  if (a.pq != nullptr && leader && threadIdx.x == 0) {
    __threadfence();
    st_release_gpu(a.pq + 2 + atomicAdd(a.pq, 1), pair + 1);
  }
}


// 32 fp32 values scaled by `s` -> 32 bf16 at `dst` (16-byte aligned): four 16-byte stores.
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const uint32_t (&v)[32], float s) {
  uint32_t w[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * s, __uint_as_float(v[2 * j + 1]) * s);
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

// ================================================================================================
// pass B: z += pw H
// ================================================================================================
template <int E>  // d = 256 E
struct AbsBSmem {
  static constexpr uint32_t A_BYTES = 128 * 64 * 2;       // pw: this CTA's 128 queries x 64 rows
  static constexpr uint32_t BOX_BYTES = 64 * 64 * 2;      // 64 rows x 64 columns of H
  static constexpr uint32_t B_BYTES = E * 2 * BOX_BYTES;  // this CTA's 128 columns of each 256-column half
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int FIXED = 1024 + 512;
  static constexpr int STAGES = (232448 - FIXED) / (int)STAGE_BYTES > 8 ? 8 : (232448 - FIXED) / (int)STAGE_BYTES;
  static constexpr size_t BYTES = FIXED + STAGES * (size_t)STAGE_BYTES;
};
constexpr int kAbsBThreads = 320;

// warps: 0 TMA producer (both CTAs), 1 TMEM (256 E columns: z of this CTA's 128 queries) + MMA issue
// (even CTA), 2..9 correction and drain (two warps per lane quadrant, half of the columns each).
// Per unit: the correction warps compare pass A's references of consecutive units; where one
// was raised they wait for the previous unit's MMAs, scale their rows of z in TMEM and only then
// release the unit to the MMA issuer (`cready`, 8 + 8 warps). They run at most two units ahead
// (`udone` of unit - 2), so the two `cready` phases never alias.
template <int E>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAbsBThreads, 1)
    abs_values_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmH,
                      const AbsArgs a) {
  using L = AbsBSmem<E>;
  constexpr int ST = L::STAGES;
  constexpr uint32_t TMEM_COLS = 256 * E;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * L::STAGE_BYTES);
  uint64_t* empty = full + ST;
  uint64_t* udone = empty + ST;   // [2] MMAs of a unit complete (commit to both CTAs)
  uint64_t* cready = udone + 2;   // [2] even CTA: unit released by 8 + 8 correction warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cready + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* ticket = reinterpret_cast<int*>(tmem_slot + 2);  // even CTA: this pair's place in pass A's order
  int* src_slot = ticket + 1;                           // the pass A pair taken (+ 1; 0 = none)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&udone[i], 1);
      mbar_init(&cready[i], 16);
    }
    *abort_flag = 0;
    // The ticket counter is read without a dependency wait: pass B launches only after pass A's
    // trigger, which pass A issues after its own wait, so the clear of the queue (a kernel before
    // pass A) has completed; the atomic is performed at L2, where that completed clear is.
    if (a.pq != nullptr && leader) *ticket = atomicAdd(a.pq + 1, 1);
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmH);
  }
  if (warp == 1) {
    tmem_alloc_cg2(tmem_slot, TMEM_COLS);
    tmem_relinquish_cg2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  int src = pair;  // the pass A pair whose units (weights, references, statistics) this pair reduces
  if (a.pq != nullptr) {
    // Pass A pairs are taken in the order they finish (the ticket drawn by the even CTA), each as
    // soon as its outputs are published: no wait for the rest of pass A.
    if (threadIdx.x == 0) {
      const int t = leader ? *ticket : ld_shared_cluster_s32(mapa_shared(smem_u32(ticket), 0));
      const int v = (t >= 0 && t < a.n_pairs) ? wait_nonzero_gpu(a.pq + 2 + t) : 0;
      fence_proxy_async_all();  // the weights are read by TMA below
      if (v == 0) *abort_flag = 1;
      *src_slot = v;
    }
    __syncthreads();
    src = *src_slot - 1;
  } else {
    pdl_wait();
  }
  pdl_trigger();

  AbsWalk wk;
  wk.init(a, src < 0 ? pair : src);
  if (src < 0) wk.u = wk.u1;  // nothing taken (timed out): no units

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs): only the 64-row chunks holding valid rows ----------
    if (lane == 0) {
      int kg = 0;
      bool stop = false;
      // prefetch cursor (unit pf, chunk pc), kAbsBPrefetchCh valid chunks ahead of the loads
      AbsWalk pf = wk;
      int pc = 0;
      AbsUnit pu{};
      if (pf.valid()) pu = abs_unit(a, pf);
      auto pf_advance = [&]() {
        if (++pc == (pu.nvalid + 63) / 64) {
          pc = 0;
          pf.next(a);
          if (pf.valid()) pu = abs_unit(a, pf);
        }
      };
      for (int i = 0; i < kAbsBPrefetchCh && pf.valid(); ++i) pf_advance();
      for (; wk.valid() && !stop; wk.next(a)) {
        const AbsUnit un = abs_unit(a, wk);
        const int nch = (un.nvalid + 63) / 64;
        for (int c = 0; c < nch; ++c, ++kg) {
          const int s = kg % ST, u = kg / ST;
          if (kg >= ST && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag)) {
            stop = true;
            break;
          }
          uint8_t* st = smem + s * L::STAGE_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * L::STAGE_BYTES);
          tma_load_2d_cg2(st, &tmP, 0, (un.ptile0 + c) * kAbsQ + (int)rank * 128, bar);
          const int hrow = (int)un.row0 + 64 * c;
#pragma unroll
          for (int e = 0; e < E; ++e)
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d_cg2(st + L::A_BYTES + (e * 2 + j) * L::BOX_BYTES, &tmH, e * 256 + (int)rank * 128 + j * 64,
                              hrow, bar);
          if (kAbsBPrefetchCh > 0 && pf.valid()) {
            tma_prefetch_l2_2d(&tmP, 0, (pu.ptile0 + pc) * kAbsQ + (int)rank * 128);
#pragma unroll
            for (int e = 0; e < E; ++e)
#pragma unroll
              for (int j = 0; j < 2; ++j)
                tma_prefetch_l2_2d(&tmH, e * 256 + (int)rank * 128 + j * 64, (int)pu.row0 + 64 * pc);
            pf_advance();
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (even CTA) ----------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256) | kIdescBMnMajor;
      int kg = 0, it = 0;
      bool stop = false;
      for (; wk.valid() && !stop; wk.next(a), ++it) {
        const AbsUnit un = abs_unit(a, wk);
        if (!mbar_wait_cluster(&cready[it & 1], (it >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const int nch = (un.nvalid + 63) / 64;
        for (int c = 0; c < nch; ++c, ++kg) {
          const int s = kg % ST, u = kg / ST;
          if (!mbar_wait(&full[s], u & 1, abort_flag)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * L::STAGE_BYTES);
          const uint32_t b_base = a_base + L::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int e = 0; e < E; ++e)
              umma_f16_cg2(tmem_base + e * 256, sdesc_k_sw128(a_base + kk * 32),
                           sdesc_mn_sw128(b_base + e * 2 * L::BOX_BYTES + kk * 2048, L::BOX_BYTES, 1024), idesc,
                           (un.first && c == 0 && kk == 0) ? 0u : 1u);
          umma_commit_cg2_mc(&empty[s], 0x3);
        }
        umma_commit_cg2_mc(&udone[it & 1], 0x3);
      }
    }
  } else {
    // ---------------- correction and drain (warps 2..9, both CTAs) ----------------
    const int qd = warp & 3;
    const int hf = (warp - 2) >> 2;
    constexpr int NC = E * 128;  // z columns of this warp: [NC hf, NC hf + NC)
    const int row = qd * 32 + lane;
    const int qg = (int)rank * 128 + row;
    const int head = qg / a.N, n = qg % a.N;
    const uint32_t cready0 = mapa_shared(smem_u32(&cready[0]), 0);
    const uint32_t t0 = tmem_base + hf * NC + ((uint32_t)(qd * 32) << 16);
    int it = 0;
    for (; wk.valid(); wk.next(a), ++it) {
      const AbsUnit un = abs_unit(a, wk);
      if (it >= 2 && !mbar_wait(&udone[it & 1], ((it - 2) >> 1) & 1, abort_flag)) break;
      if (!un.first) {
        const float mp = a.mref[(size_t)(wk.u - 1) * kAbsQ + qg];
        const float mc = a.mref[(size_t)wk.u * kAbsQ + qg];
        if (__any_sync(0xffffffffu, mc != mp)) {
          if (!mbar_wait(&udone[(it - 1) & 1], ((it - 1) >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          const float f = mc != mp ? fast_exp2(mp - mc) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < NC / 32; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(t0 + c * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
            tmem_st_32x32b_x32(t0 + c * 32, v);
          }
          tmem_st_wait();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&cready[it & 1]);
        else mbar_arrive_cluster_release(cready0 + (it & 1) * 8);
      }
      if (un.last) {
        if (!mbar_wait(&udone[it & 1], (it >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        // whole example: z / l; partial segment: unnormalised z (merged by abs_merge_kernel)
        const float inv = un.whole
                              ? 1.0f / reinterpret_cast<const float2*>(a.stats_whole)[(size_t)un.b * kAbsQ + qg].y
                              : 1.0f;
        __nv_bfloat16* dz = un.whole ? a.z_hi + (((size_t)head * a.B + un.b) * a.N + n) * a.d + hf * NC
                                     : a.part_z + ((size_t)un.slot * kAbsQ + qg) * a.d + hf * NC;
#pragma unroll 1
        for (int c = 0; c < NC / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t0 + c * 32, v);
          tmem_ld_wait();
          store_bf16x32(dz + c * 32, v, inv);
        }
        tc_fence_before();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_cg2(tmem_base, TMEM_COLS);
  }
}

// ================================================================================================
// merge of examples split across pairs; zero z for empty histories
// ================================================================================================
// grid (B, 256 / 8), 256 threads: one warp per absorbed query. The lanes first gather the
// (slot, weight) list of the example's partials (one pair each), then stream the partial z rows.
// (Four queries per warp, with a quarter of the warps per SM, measured slower.)
__global__ void __launch_bounds__(256) abs_merge_kernel(const AbsArgs a) {
  pdl_wait();
  pdl_trigger();
  // Pass B is complete (this kernel waited for it), and with it every pass A pair it acquired, so
  // every pass A pair has published: the queue can be reset for the next layer's passes.
  if (a.pq != nullptr && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < 2 + a.n_pairs; i += blockDim.x) a.pq[i] = 0;
  __shared__ int s_slot[8][kAbsMaxPairs];
  __shared__ float s_w[8][kAbsMaxPairs];
  __shared__ float s_l[8][kAbsMaxPairs];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int q = blockIdx.y * 8 + warp;
  if (q >= kAbsQ) return;
  const int U = a.ustart[a.B];
  const int ub = a.ustart[b], ub1 = a.ustart[b + 1];
  const int head = q / a.N, n = q % a.N;
  const size_t zrow = ((size_t)head * a.B + b) * a.N + n;
  uint2* zh = reinterpret_cast<uint2*>(a.z_hi + zrow * a.d);
  if (ub >= ub1) {  // empty history: the attention output is the empty sum
    for (int c = lane; c < a.d / 4; c += 32) zh[c] = make_uint2(0u, 0u);
    return;
  }
  const int P = a.n_pairs;
  const int p0 = abs_pair_of(ub, U, P), p1 = abs_pair_of(ub1 - 1, U, P);
  if (p0 == p1) return;  // finished by pass B
  const int cnt = p1 - p0 + 1;  // <= n_pairs <= kAbsMaxPairs
  const float2* st = reinterpret_cast<const float2*>(a.stats_part);
  float M = -INFINITY;
  for (int j = lane; j < cnt; j += 32) {
    const int p = p0 + j;
    const int r0 = abs_range_start(U, P, p), r1 = abs_range_start(U, P, p + 1);
    const int slot = r0 < r1 ? (r0 >= ub ? 2 * p : 2 * p + 1) : -1;
    s_slot[warp][j] = slot;
    const float2 ml = slot >= 0 ? st[(size_t)slot * kAbsQ + q] : make_float2(-INFINITY, 0.f);  // (m, l) at once
    s_w[warp][j] = ml.x;
    s_l[warp][j] = ml.y;
    M = fmaxf(M, ml.x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float l = 0.f;
  for (int j = lane; j < cnt; j += 32) {
    const int slot = s_slot[warp][j];
    const float w = slot >= 0 ? fast_exp2(s_w[warp][j] - M) : 0.f;
    s_w[warp][j] = w;
    if (slot >= 0) l += w * s_l[warp][j];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  __syncwarp();
  const float inv = 1.0f / l;
  // Lane c holds columns [8c, 8c + 8) and, at d = 512, [256 + 8c, 256 + 8c + 8): one 16-byte
  // load per chunk and partial, the loads of a partial issued together.
  const int nch = a.d / 256;
  float acc[2][8];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[i][k] = 0.f;
#pragma unroll 2
  for (int j = 0; j < cnt; ++j) {
    const int slot = s_slot[warp][j];
    const float w = s_w[warp][j];  // 0 for an empty range
    uint4 v[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    if (slot >= 0) {
      const uint4* src = reinterpret_cast<const uint4*>(a.part_z + ((size_t)slot * kAbsQ + q) * a.d);
      v[0] = __ldcg(src + lane);
      if (nch == 2) v[1] = __ldcg(src + 32 + lane);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (i >= nch) break;
      float f[8];
      bf16x8_to_f32(v[i], f);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[i][k] = fmaf(w, f[k], acc[i][k]);
    }
  }
  uint4* zh16 = reinterpret_cast<uint4*>(a.z_hi + zrow * a.d);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (i >= nch) break;
    zh16[i * 32 + lane] = make_uint4(pack_bf16x2(acc[i][0] * inv, acc[i][1] * inv),
                                     pack_bf16x2(acc[i][2] * inv, acc[i][3] * inv),
                                     pack_bf16x2(acc[i][4] * inv, acc[i][5] * inv),
                                     pack_bf16x2(acc[i][6] * inv, acc[i][7] * inv));
  }
}

}  // namespace whale
