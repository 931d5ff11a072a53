// absorbed_fused.cuh — the two passes of the absorbed cross-attention (absorbed.cuh: Eq. (4) of
// WHALE with W_K and W_V folded into the queries) in one kernel, so that every history row leaves
// HBM once per layer and the softmax weights never leave the SMs.
//
// A cluster of four CTAs walks one contiguous range of 256-row units (the ranges, segments and
// partial slots of absorbed.cuh, with one range per cluster):
//
//   scorer pair, ranks 0 and 1 (pass A): S = qa H_u^T on the 2-SM tensor cores, the RMSNorm row
//     factor r_t, and the online softmax. For every unit it first takes the tile maximum, moves the
//     reference to it when it exceeds the current one by more than 2^kAbsLazy (so every weight is
//     below 2^kAbsLazy and nothing is ever rewritten), then writes pw = 2^(r s - m) * r of each
//     64-row chunk straight into the shared memory of the value CTA that holds the same 128 queries
//     (rank + 2), together with the unit's reference and, at a segment's end, its softmax sum.
//   value pair, ranks 2 and 3 (pass B): z += pw_chunk H_chunk on the 2-SM tensor cores (H as the
//     MN-major operand, read from L2 right after the scorer's read of the same rows), rescaling z in
//     TMEM where the reference moved, and draining z / l (or an unnormalised partial) at segment ends.
//
// Hand-off: a ring of kFuRing weight-chunk slots (128 queries x 64 rows, K-major, 128-byte swizzle)
// in each value CTA. A scorer epilogue warp writes its 32 x 64 tile of a chunk into a local staging
// ring of kFuStg chunks (plain shared stores), fences them towards the async proxy, and one lane
// hands the 4 KB tile to the copy engine (cp.async.bulk shared::cta -> shared::cluster), which
// counts the bytes on the value CTA's `pw_full` barrier (armed by the value CTA's producer). The
// warps never store across the cluster themselves and issue no cluster-scope fence. The value
// leader's MMA thread waits for its own slot and, through a relay warp of rank 3, for rank 3's;
// it then frees the scorer's staging chunk (`stg_free`, rank 0; the relay does it for rank 1), and
// its MMA commit frees the slot (`pw_empty`, multicast to ranks 0 and 1). A unit's softmax
// references travel by st.async into the reference row of its first chunk's slot (`mref_full`,
// counted in bytes; the slot's `pw_empty` guards the row as it guards the weights). A segment's
// softmax sums travel by st.async into a one-entry mailbox (`lseg_full`), which the value CTA hands
// back (`lbox_free`) once its eight correction warps have read it.
#pragma once

#include "absorbed.cuh"

namespace whale {

constexpr int kFuRing = 9;   // weight chunks in flight per value CTA (2.25 units)
constexpr int kFuStg = 4;    // staged weight chunks per scorer CTA (one unit)
constexpr int kFuPrefetch = 2;  // units of history rows the scorer prefetches into L2 ahead of its loads
constexpr int kFuThreads = 480;
constexpr int kFuMaxClusters = 37;  // 148 SMs / 4

template <int E>  // d = 256 E
struct FuSmem {
  // common header: the same offsets in all four CTAs (multicast commits and remote arrivals
  // address a barrier by its offset)
  static constexpr int PW_EMPTY = 0;                        // [kFuRing] scorer CTAs: slot consumed (MMA commit)
  static constexpr int PW_FULL = PW_EMPTY + kFuRing * 8;    // [kFuRing] value CTAs: own slot landed (bytes)
  static constexpr int PW_PEER = PW_FULL + kFuRing * 8;     // [kFuRing] rank 2: rank 3's slot landed (relay)
  static constexpr int MREF_FULL = PW_PEER + kFuRing * 8;   // [kFuRing] value CTAs: slot's references landed
  static constexpr int LSEG_FULL = MREF_FULL + kFuRing * 8; // value CTAs: segment sums landed (bytes)
  static constexpr int LBOX_FREE = LSEG_FULL + 8;           // scorer CTAs: segment sums read
  static constexpr int STG_FREE = LBOX_FREE + 8;            // [kFuStg] scorer CTAs: staged chunk landed
  static constexpr int MREF = STG_FREE + kFuStg * 8;        // [kFuRing][128] f32, value CTAs
  static constexpr int LSEG = MREF + kFuRing * 128 * 4;     // [128] f32, value CTAs
  static constexpr int HEADER = (LSEG + 128 * 4 + 1023) / 1024 * 1024;
  // scorer region: stages of (qa box | H box), staging ring, exchange arrays, local barriers
  static constexpr uint32_t SA_BYTES = 128 * 64 * 2;
  static constexpr uint32_t S_STAGE = 2 * SA_BYTES;
  static constexpr int S_ST = 4;
  static constexpr uint32_t PW_SLOT = 128 * 64 * 2;  // one chunk of this CTA's 128 queries
  static constexpr int S_STG = HEADER + S_ST * (int)S_STAGE;
  static constexpr int S_XCH = S_STG + kFuStg * (int)PW_SLOT;  // rbuf[2][256], xmax[2][2][128], xsum[2][128]
  static constexpr int S_BAR = S_XCH + (2 * 256 + 2 * 2 * 128 + 2 * 128) * 4;
  static constexpr int S_END = S_BAR + (3 * S_ST + 8 + 8 + 4) * 8 + 16;  // + tmem slot, abort flag
  // value region: weight ring, H stages (E x 2 boxes of 64 rows x 64 columns), local barriers
  static constexpr uint32_t BOX = 64 * 64 * 2;
  static constexpr uint32_t V_STAGE = E * 2 * BOX;
  static constexpr int V_ST = 2;
  static constexpr int V_PW = HEADER;
  static constexpr int V_H = V_PW + kFuRing * (int)PW_SLOT;
  static constexpr int V_BAR = V_H + V_ST * (int)V_STAGE;
  static constexpr int V_END = V_BAR + (2 * V_ST + 5) * 8 + 16;
  static constexpr int END = S_END > V_END ? S_END : V_END;
  static constexpr size_t BYTES = 1024 + (size_t)END;
  static_assert(BYTES <= 232448, "shared memory of one CTA");
  // the producer arms a slot's reference barrier when it loads the slot's chunk; the unit that used
  // the slot before (at most 4 chunks, kFuRing chunks back) must have passed its correction by then
  static_assert(kFuRing - 4 >= V_ST, "weight ring deeper than the H stages plus one unit");
  static_assert(HEADER % 1024 == 0 && V_H % 1024 == 0 && S_STG % 1024 == 0 && S_XCH % 1024 == 0,
                "swizzled tiles need 1 KB alignment");
};

// ------------------------------------------------------------------------------------------------
// scorer epilogue (warps 2..9 of ranks 0, 1): softmax and the hand-off of the weights
// ------------------------------------------------------------------------------------------------
// Warp (quadrant qd, half hf) owns queries 32 qd .. 32 qd + 31 of this CTA and unit rows
// 128 hf .. 128 hf + 127, i.e. weight chunks 2 hf and 2 hf + 1 of the unit.
template <int E>
__device__ __forceinline__ void fu_scorer_epilogue(uint8_t* smem, uint32_t rank, const AbsArgs& a, AbsWalk wk,
                                                   uint32_t tmem_base, const float* rbuf, float* xmax, float* xsum,
                                                   uint64_t* tfull, uint64_t* tempty, uint64_t* nfull, uint64_t* edone,
                                                   uint64_t* xbar, uint64_t* lbar, volatile int* abort_flag) {
  using L = FuSmem<E>;
  uint64_t* pw_empty = reinterpret_cast<uint64_t*>(smem + L::PW_EMPTY);
  uint64_t* stg_free = reinterpret_cast<uint64_t*>(smem + L::STG_FREE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qd = warp & 3;
  const int hf = (warp - 2) >> 2;
  const int row = qd * 32 + lane;
  const int qg = (int)rank * 128 + row;
  const uint32_t vrank = rank + 2;  // value CTA holding the same 128 queries
  const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
  const uint32_t edone_peer0 = mapa_shared(smem_u32(&edone[0]), rank ^ 1);
  const uint32_t tile_off = (uint32_t)(qd * 4096);  // this warp's 32 rows of a chunk slot
  uint8_t* stg_tile0 = smem + L::S_STG + tile_off;
  uint8_t* stg_row0 = stg_tile0 + lane * 128;
  const uint32_t pw_dst0 = mapa_shared(smem_u32(smem + L::V_PW), vrank) + tile_off;
  const uint32_t pw_full0 = mapa_shared(smem_u32(smem + L::PW_FULL), vrank);
  uint64_t* lbox_free = reinterpret_cast<uint64_t*>(smem + L::LBOX_FREE);
  const uint32_t mref_dst = mapa_shared(smem_u32(smem + L::MREF), vrank) + (uint32_t)(row * 4);
  const uint32_t lseg_dst = mapa_shared(smem_u32(smem + L::LSEG), vrank) + (uint32_t)(row * 4);
  const uint32_t mref_full0 = mapa_shared(smem_u32(smem + L::MREF_FULL), vrank);
  const uint32_t lseg_full = mapa_shared(smem_u32(smem + L::LSEG_FULL), vrank);

  // 32 consecutive row factors (the same for every lane: broadcast shared-memory loads)
  auto load_r32 = [&](const float* r, float (&rr)[32]) {
    const float4* r4 = reinterpret_cast<const float4*>(r);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 x = r4[i];
      rr[4 * i] = x.x;
      rr[4 * i + 1] = x.y;
      rr[4 * i + 2] = x.z;
      rr[4 * i + 3] = x.w;
    }
  };
  // maximum of r_t * s over the valid columns of this half
  auto tile_max = [&](uint32_t t0, const float* r, int nv) -> float {
    float mx = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float rr[32];
      load_r32(r + c * 32, rr);
      uint32_t v[32];
      tmem_ld_32x32b_x32(t0 + c * 32, v);
      tmem_ld_wait();
      if (c * 32 + 32 <= nv) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          mx = fmaxf(mx, fmaxf(fmaxf(__uint_as_float(v[j]) * rr[j], __uint_as_float(v[j + 1]) * rr[j + 1]),
                               fmaxf(__uint_as_float(v[j + 2]) * rr[j + 2], __uint_as_float(v[j + 3]) * rr[j + 3])));
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c * 32 + j < nv) mx = fmaxf(mx, __uint_as_float(v[j]) * rr[j]);
      }
    }
    return mx;
  };
  // pw = 2^(r s - m) * r over the valid columns of one 64-row chunk (0 elsewhere) into this lane's
  // row of the staging tile at `row_ptr` (128-byte swizzled K-major layout, as the MMA reads it).
  auto stage_chunk = [&](uint32_t t0, const float* r, int nv, float m, float& lsum, uint8_t* row_ptr) {
#pragma unroll 1
    for (int h2 = 0; h2 < 2; ++h2) {
      const int c0 = h2 * 32;
      float rr[32];
      load_r32(r + c0, rr);
      uint32_t v[32];
      tmem_ld_32x32b_x32(t0 + c0, v);
      tmem_ld_wait();
      uint32_t pk[16];
      float ls = 0.f;
      if (c0 + 32 <= nv) {
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(v[j]), rr[j], -m));
          const float p1 = fast_exp2(fmaf(__uint_as_float(v[j + 1]), rr[j + 1], -m));
          ls += p0 + p1;
          pk[j / 2] = pack_bf16x2(p0 * rr[j], p1 * rr[j + 1]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const bool ok0 = c0 + j < nv, ok1 = c0 + j + 1 < nv;
          const float p0 = ok0 ? fast_exp2(fmaf(__uint_as_float(v[j]), rr[j], -m)) : 0.f;
          const float p1 = ok1 ? fast_exp2(fmaf(__uint_as_float(v[j + 1]), rr[j + 1], -m)) : 0.f;
          ls += p0 + p1;
          pk[j / 2] = pack_bf16x2(p0 * rr[j], p1 * rr[j + 1]);
        }
      }
      lsum += ls;
      uint4* dst = reinterpret_cast<uint4*>(row_ptr);
#pragma unroll
      for (int j8 = 0; j8 < 4; ++j8)
        dst[(h2 * 4 + j8) ^ (lane & 7)] = make_uint4(pk[4 * j8], pk[4 * j8 + 1], pk[4 * j8 + 2], pk[4 * j8 + 3]);
    }
  };

  float m_run = 0.f, l_part = 0.f;
  int it = 0, nseg = 0;
  long long kch = 0;  // weight chunks of the earlier units of the range
  bool ok = true;
  for (; wk.valid() && ok; wk.next(a), ++it) {
    const AbsUnit un = abs_unit(a, wk);
    const int acc = it & 1, ua = it >> 1;
    if (!mbar_wait(&tfull[acc], ua & 1, abort_flag)) break;
    if (!mbar_wait_cluster(&nfull[acc], ua & 1, abort_flag)) break;
    tc_fence_after();
    const float* r = rbuf + acc * 256 + hf * 128;
    const uint32_t t0 = tmem_base + acc * 256 + hf * 128 + ((uint32_t)(qd * 32) << 16);
    const int nv = un.nvalid - hf * 128;  // valid rows of this half (may be <= 0)
    const int nch = (un.nvalid + 63) / 64;
    // tile maximum of both halves, through the quadrant's exchange barrier
    xmax[(acc * 2 + hf) * 128 + row] = tile_max(t0, r, nv);
    __syncwarp();
    if (lane == 0) mbar_arrive(&xbar[qd * 2 + acc]);
    if (!mbar_wait(&xbar[qd * 2 + acc], ua & 1, abort_flag)) break;
    const float mt = fmaxf(xmax[(acc * 2) * 128 + row], xmax[(acc * 2 + 1) * 128 + row]);
    float m_use;
    if (un.first) {
      m_use = mt;
      l_part = 0.f;
    } else if (mt > m_run + kAbsLazy) {
      m_use = mt;
      l_part *= fast_exp2(m_run - mt);
    } else {
      m_use = m_run;
    }
    m_run = m_use;
    // this warp's chunks 2 hf, 2 hf + 1 that hold valid rows: wait until the value CTA's slot is
    // consumed and the staging chunk's previous copy has landed, stage, then hand both to the copy
    // engine
    const int ncc = nch - hf * 2 < 0 ? 0 : (nch - hf * 2 > 2 ? 2 : nch - hf * 2);
    float l_unit = 0.f;
#pragma unroll 1
    for (int cc = 0; cc < ncc; ++cc) {
      const long long k = kch + hf * 2 + cc;
      if (k >= kFuRing &&
          !mbar_wait_cluster(&pw_empty[k % kFuRing], (uint32_t)((k / kFuRing - 1) & 1), abort_flag)) {
        ok = false;
        break;
      }
      // the unit's references go to the reference row of its first chunk's slot, free now
      if (hf == 0 && cc == 0) {
        const int g0 = (int)(k % kFuRing);
        st_async_f32(mref_dst + (uint32_t)(g0 * 512), m_use, mref_full0 + g0 * 8);
      }
      if (k >= kFuStg && !mbar_wait_cluster(&stg_free[k % kFuStg], (uint32_t)((k / kFuStg - 1) & 1), abort_flag)) {
        ok = false;
        break;
      }
      stage_chunk(t0 + cc * 64, r + cc * 64, nv - cc * 64, m_use, l_unit,
                  stg_row0 + (k % kFuStg) * L::PW_SLOT);
    }
    if (!ok) break;
    if (ncc > 0) {
      fence_proxy_async_smem();  // the staged tiles are read by the copy engine (async proxy)
      __syncwarp();
      if (lane == 0)
        for (int cc = 0; cc < ncc; ++cc) {
          const long long k = kch + hf * 2 + cc;
          const int g = (int)(k % kFuRing);
          bulk_copy_to_peer(pw_dst0 + (uint32_t)g * L::PW_SLOT, stg_tile0 + (k % kFuStg) * L::PW_SLOT, 4096,
                            pw_full0 + g * 8);
        }
    }
    kch += nch;
    l_part += l_unit;
    if (un.last) {
      xsum[hf * 128 + row] = l_part;
      __syncwarp();
      if (lane == 0) mbar_arrive(&lbar[qd]);
      if (!mbar_wait(&lbar[qd], nseg & 1, abort_flag)) break;
      if (hf == 0) {
        const float lseg = xsum[row] + xsum[128 + row];
        float2* st = un.whole ? reinterpret_cast<float2*>(a.stats_whole) + (size_t)un.b * kAbsQ + qg
                              : reinterpret_cast<float2*>(a.stats_part) + (size_t)un.slot * kAbsQ + qg;
        *st = make_float2(m_use, lseg);
        // the mailbox holds one segment: wait until the value CTA has read the previous one
        if (nseg >= 1 && !mbar_wait_cluster(lbox_free, (uint32_t)((nseg - 1) & 1), abort_flag)) break;
        st_async_f32(lseg_dst, lseg, lseg_full);
      }
      ++nseg;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_cluster(tempty0 + acc * 8);  // rank 0's MMA may reuse this accumulator
      // rbuf[acc] may be rewritten: its reads above have completed (their values are used), so a
      // plain arrival orders them before the statistic warps' writes
      mbar_arrive(&edone[acc]);
      mbar_arrive_cluster(edone_peer0 + acc * 8);
    }
  }
  // Before the CTA may leave, the value CTAs' last remote arrivals on this CTA's barriers must have
  // landed: wait for the consumption of every slot's last chunk and the landing of every staged one.
  if (ok && warp == 2 && lane == 0) {
    for (long long k = (kch > kFuRing ? kch - kFuRing : 0); k < kch; ++k)
      if (!mbar_wait_cluster(&pw_empty[k % kFuRing], (uint32_t)((k / kFuRing) & 1), abort_flag)) break;
    for (long long k = (kch > kFuStg ? kch - kFuStg : 0); k < kch; ++k)
      if (!mbar_wait_cluster(&stg_free[k % kFuStg], (uint32_t)((k / kFuStg) & 1), abort_flag)) break;
  }
}

// ------------------------------------------------------------------------------------------------
// scorer pair (ranks 0, 1)
// ------------------------------------------------------------------------------------------------
// warps: 0 TMA producer, 1 TMEM (2 x 256 columns) + MMA issue (rank 0), 2..9 softmax and hand-off
// (two warps per lane quadrant, 128 unit rows each), 10..13 row statistics, 14 relay (rank 0).
template <int E>
__device__ __forceinline__ void fu_scorer(uint8_t* smem, uint32_t rank, int cl, const AbsArgs& a,
                                          const CUtensorMap* tmQ, const CUtensorMap* tmH, uint32_t& tmem_cols,
                                          uint32_t& tmem_addr) {
  using L = FuSmem<E>;
  constexpr int ST = L::S_ST;
  uint64_t* pw_empty = reinterpret_cast<uint64_t*>(smem + L::PW_EMPTY);
  uint64_t* stg_free = reinterpret_cast<uint64_t*>(smem + L::STG_FREE);
  float* rbuf = reinterpret_cast<float*>(smem + L::S_XCH);  // [2][256]
  float* xmax = rbuf + 2 * 256;                              // [2 acc][2 half][128]
  float* xsum = xmax + 2 * 2 * 128;                          // [2 half][128]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::S_BAR);
  uint64_t* ready = full + ST;
  uint64_t* empty = ready + ST;
  uint64_t* tfull = empty + ST;  // [2]
  uint64_t* tempty = tfull + 2;  // [2]
  uint64_t* nfull = tempty + 2;  // [2]
  uint64_t* edone = nfull + 2;   // [2]
  uint64_t* xbar = edone + 2;    // [8]
  uint64_t* lbar = xbar + 8;     // [4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lbar + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool leader = rank == 0;
  const int KB = a.d / 64;

  if (threadIdx.x == 0) {
    for (int g = 0; g < kFuRing; ++g) mbar_init(&pw_empty[g], 1);
    for (int b = 0; b < kFuStg; ++b) mbar_init(&stg_free[b], 1);
    mbar_init(reinterpret_cast<uint64_t*>(smem + L::LBOX_FREE), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 1);
      mbar_init(&empty[s], 1 + 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 16);
      mbar_init(&nfull[i], 8);
      mbar_init(&edone[i], 16);
    }
    for (int i = 0; i < 8; ++i) mbar_init(&xbar[i], 2);
    for (int i = 0; i < 4; ++i) mbar_init(&lbar[i], 2);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(tmQ);
    tma_prefetch_desc(tmH);
  }
  if (warp == 1) {
    tmem_alloc_cg2(tmem_slot, 512);
    tmem_relinquish_cg2();
  }
  tmem_cols = 512;
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // every barrier of the cluster is initialised before anyone arrives remotely
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  tmem_addr = tmem_base;
  pdl_wait();
  pdl_trigger();

  AbsWalk wk;
  wk.init(a, cl);

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      // The history rows of unit u + kFuPrefetch are prefetched into L2 while unit u loads, so the
      // stage loads below are L2 hits (four stages of lookahead do not cover HBM latency).
      AbsWalk pf = wk;
      for (int i = 0; i < kFuPrefetch && pf.valid(); ++i) {
        const AbsUnit pu = abs_unit(a, pf);
        for (int kb = 0; kb < KB; ++kb) tma_prefetch_l2_2d(tmH, kb * 64, (int)pu.row0 + (int)rank * 128);
        pf.next(a);
      }
      int kg = 0;
      bool stop = false;
      for (; wk.valid() && !stop; wk.next(a)) {
        const AbsUnit un = abs_unit(a, wk);
        const int qrow = un.b * kAbsQ + (int)rank * 128;
        const int hrow = (int)un.row0 + (int)rank * 128;
        if (pf.valid()) {
          const AbsUnit pu = abs_unit(a, pf);
          for (int kb = 0; kb < KB; ++kb) tma_prefetch_l2_2d(tmH, kb * 64, (int)pu.row0 + (int)rank * 128);
          pf.next(a);
        }
        for (int kb = 0; kb < KB; ++kb, ++kg) {
          const int s = kg % ST, u = kg / ST;
          if (kg >= ST && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag)) {
            stop = true;
            break;
          }
          uint8_t* st = smem + L::HEADER + s * L::S_STAGE;
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * L::S_STAGE);
          tma_load_2d_cg2(st, tmQ, kb * 64, qrow, bar);
          tma_load_2d_cg2(st + L::SA_BYTES, tmH, kb * 64, hrow, bar);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (rank 0) ----------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256);
      int kg = 0, it = 0;
      bool stop = false;
      for (; wk.valid() && !stop; wk.next(a), ++it) {
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
          const uint32_t a_base = smem_u32(smem + L::HEADER + s * L::S_STAGE);
          const uint32_t b_base = a_base + L::SA_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16_cg2(d_tmem, sdesc_k_sw128(a_base + kk * 32), sdesc_k_sw128(b_base + kk * 32), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_cg2_mc(&empty[s], 0x3);
        }
        umma_commit_cg2_mc(&tfull[acc], 0x3);
      }
    }
  } else if (warp == 14) {
    // ---------------- relay of "stage landed" to rank 1's statistic warps (rank 0) ----------------
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
        const uint4* rp = reinterpret_cast<const uint4*>(smem + L::HEADER + s * L::S_STAGE + L::SA_BYTES + row * 128);
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
    fu_scorer_epilogue<E>(smem, rank, a, wk, tmem_base, rbuf, xmax, xsum, tfull, tempty, nfull, edone, xbar, lbar,
                          abort_flag);
  }
}


// ------------------------------------------------------------------------------------------------
// value pair (ranks 2, 3)
// ------------------------------------------------------------------------------------------------
// warps: 0 TMA producer (H of every chunk; arms the weight slot of each chunk), 1 TMEM (256 E
// columns: z of this CTA's 128 queries) + MMA issue (rank 2), 2..9 correction and drain (two warps
// per lane quadrant, half of the columns each), 10 relay (this CTA's slot landed -> the partner
// scorer CTA's stg_free, and on rank 3 rank 2's pw_peer), 11..14 idle.
template <int E>
__device__ __forceinline__ void fu_value(uint8_t* smem, uint32_t rank, int cl, const AbsArgs& a,
                                         const CUtensorMap* tmH64, uint32_t& tmem_cols, uint32_t& tmem_addr) {
  using L = FuSmem<E>;
  constexpr int ST = L::V_ST;
  constexpr uint32_t TMEM_COLS = 256 * E;
  uint64_t* pw_empty = reinterpret_cast<uint64_t*>(smem + L::PW_EMPTY);
  uint64_t* pw_full = reinterpret_cast<uint64_t*>(smem + L::PW_FULL);
  uint64_t* pw_peer = reinterpret_cast<uint64_t*>(smem + L::PW_PEER);
  uint64_t* mref_full = reinterpret_cast<uint64_t*>(smem + L::MREF_FULL);
  uint64_t* lseg_full = reinterpret_cast<uint64_t*>(smem + L::LSEG_FULL);
  const uint32_t stg_free0 = mapa_shared(smem_u32(smem + L::STG_FREE), rank - 2);  // the partner scorer CTA
  const float* mref = reinterpret_cast<const float*>(smem + L::MREF);
  const float* lseg = reinterpret_cast<const float*>(smem + L::LSEG);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::V_BAR);
  uint64_t* empty = full + ST;
  uint64_t* udone = empty + ST;  // [2] MMAs of a unit complete (commit to ranks 2 and 3)
  uint64_t* cready = udone + 2;  // [2] rank 2: unit released by 8 + 8 correction warps
  uint64_t* lread = cready + 2;  // the 8 correction warps have read the segment-sum mailbox
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lread + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t vr = rank - 2;  // 0 or 1 within the pair
  const bool leader = vr == 0;

  if (threadIdx.x == 0) {
    for (int g = 0; g < kFuRing; ++g) {
      mbar_init(&pw_full[g], 1);    // the producer's arm + 4 x 4 KB from the copy engine
      mbar_init(&pw_peer[g], 1);
      mbar_init(&mref_full[g], 1);  // the producer's arm + 512 B by st.async
    }
    mbar_init(lseg_full, 1);        // warp 2's arm + 512 B by st.async
    mbar_init(lread, 8);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&udone[i], 1);
      mbar_init(&cready[i], 16);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(tmH64);
  if (warp == 1) {
    tmem_alloc_cg2(tmem_slot, TMEM_COLS);
    tmem_relinquish_cg2();
  }
  tmem_cols = TMEM_COLS;
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  tmem_addr = tmem_base;
  pdl_wait();
  pdl_trigger();

  AbsWalk wk;
  wk.init(a, cl);

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs): H rows of the chunks holding valid rows ----------
    if (lane == 0) {
      int kg = 0;
      bool stop = false;
      for (; wk.valid() && !stop; wk.next(a)) {
        const AbsUnit un = abs_unit(a, wk);
        const int nch = (un.nvalid + 63) / 64;
        for (int c = 0; c < nch; ++c, ++kg) {
          const int s = kg % ST, u = kg / ST;
          if (kg >= ST && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag)) {
            stop = true;
            break;
          }
          uint8_t* st = smem + L::V_H + s * L::V_STAGE;
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 2);
          // The slot of chunk kg - kFuRing was consumed before the MMA waited for stage s of chunk
          // kg - ST (kFuRing > ST), so its phase has completed: arm the slot's next phase.
          mbar_arrive_expect_tx(&pw_full[kg % kFuRing], L::PW_SLOT);
          if (c == 0) mbar_arrive_expect_tx(&mref_full[kg % kFuRing], 128 * 4);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * L::V_STAGE);
          const int hrow = (int)un.row0 + 64 * c;
#pragma unroll
          for (int e = 0; e < E; ++e)
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d_cg2(st + (e * 2 + j) * L::BOX, tmH64, e * 256 + (int)vr * 128 + j * 64, hrow, bar);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (rank 2) ----------------
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256) | kIdescBMnMajor;
      int kg = 0, it = 0;
      long long kp = 0;
      bool stop = false;
      for (; wk.valid() && !stop; wk.next(a), ++it) {
        const AbsUnit un = abs_unit(a, wk);
        if (!mbar_wait_cluster(&cready[it & 1], (it >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const int nch = (un.nvalid + 63) / 64;
        for (int c = 0; c < nch; ++c, ++kg, ++kp) {
          const int s = kg % ST, u = kg / ST;
          const int g = (int)(kp % kFuRing);
          const uint32_t ph = (uint32_t)((kp / kFuRing) & 1);
          if (!mbar_wait(&full[s], u & 1, abort_flag) || !mbar_wait_cluster(&pw_full[g], ph, abort_flag) ||
              !mbar_wait_cluster(&pw_peer[g], ph, abort_flag)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + L::V_PW + g * L::PW_SLOT);
          const uint32_t b_base = smem_u32(smem + L::V_H + s * L::V_STAGE);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int e = 0; e < E; ++e)
              umma_f16_cg2(tmem_base + e * 256, sdesc_k_sw128(a_base + kk * 32),
                           sdesc_mn_sw128(b_base + e * 2 * L::BOX + kk * 2048, L::BOX, 1024), idesc,
                           (un.first && c == 0 && kk == 0) ? 0u : 1u);
          umma_commit_cg2_mc(&empty[s], 0xC);
          umma_commit_cg2_mc(&pw_empty[g], 0x3);
        }
        umma_commit_cg2_mc(&udone[it & 1], 0xC);
      }
    }
  } else if (warp == 10) {
    // ---------------- relay (both CTAs): this CTA's weight slot landed ----------------
    // frees the partner scorer CTA's staging chunk at once (not when the MMA reaches the chunk), and
    // on rank 3 tells rank 2's MMA thread that rank 3's slot is complete
    if (lane == 0) {
      const uint32_t peer0 = mapa_shared(smem_u32(&pw_peer[0]), 2);
      long long kp = 0;
      bool stop = false;
      for (; wk.valid() && !stop; wk.next(a)) {
        const AbsUnit un = abs_unit(a, wk);
        const int nch = (un.nvalid + 63) / 64;
        for (int c = 0; c < nch; ++c, ++kp) {
          const int g = (int)(kp % kFuRing);
          if (!mbar_wait_cluster(&pw_full[g], (uint32_t)((kp / kFuRing) & 1), abort_flag)) {
            stop = true;
            break;
          }
          mbar_arrive_cluster_release(stg_free0 + (uint32_t)(kp % kFuStg) * 8);
          if (!leader) mbar_arrive_cluster_release(peer0 + g * 8);
        }
      }
    }
  } else if (warp < 10) {
    // ---------------- correction and drain (warps 2..9, both CTAs) ----------------
    const int qd = warp & 3;
    const int hf = (warp - 2) >> 2;
    constexpr int NC = E * 128;  // z columns of this warp: [NC hf, NC hf + NC)
    const int row = qd * 32 + lane;
    const int qg = (int)vr * 128 + row;
    const int head = qg / a.N, n = qg % a.N;
    const uint32_t cready0 = mapa_shared(smem_u32(&cready[0]), 2);
    const uint32_t t0 = tmem_base + hf * NC + ((uint32_t)(qd * 32) << 16);
    if (warp == 2 && lane == 0 && wk.valid()) mbar_arrive_expect_tx(lseg_full, 128 * 4);
    float m_prev = 0.f;
    uint32_t mphase = 0;  // phase bit of each slot's reference barrier
    int it = 0, nseg = 0;
    long long kch = 0;
    for (; wk.valid(); wk.next(a), ++it) {
      const AbsUnit un = abs_unit(a, wk);
      const int g0 = (int)(kch % kFuRing);  // slot of the unit's first chunk: holds its references
      kch += (un.nvalid + 63) / 64;
      if (it >= 2 && !mbar_wait(&udone[it & 1], ((it - 2) >> 1) & 1, abort_flag)) break;
      if (!mbar_wait_cluster(&mref_full[g0], (mphase >> g0) & 1u, abort_flag)) break;
      mphase ^= 1u << g0;
      const float mc = mref[g0 * 128 + row];
      if (!un.first && __any_sync(0xffffffffu, mc != m_prev)) {
        if (!mbar_wait(&udone[(it - 1) & 1], ((it - 1) >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const float f = mc != m_prev ? fast_exp2(m_prev - mc) : 1.0f;
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
      m_prev = mc;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&cready[it & 1]);
        else mbar_arrive_cluster_release(cready0 + (it & 1) * 8);
      }
      if (un.last) {
        if (!mbar_wait(&udone[it & 1], (it >> 1) & 1, abort_flag)) break;
        if (!mbar_wait_cluster(lseg_full, (uint32_t)(nseg & 1), abort_flag)) break;
        const float lsg = lseg[row];
        // once all eight correction warps have read the mailbox, warp 2 hands it back to the scorer
        __syncwarp();
        if (lane == 0) mbar_arrive(lread);
        if (warp == 2 && wk.u + 1 < wk.u1) {
          if (!mbar_wait(lread, (uint32_t)(nseg & 1), abort_flag)) break;
          if (lane == 0) {
            mbar_arrive_expect_tx(lseg_full, 128 * 4);
            mbar_arrive_cluster_release(mapa_shared(smem_u32(smem + L::LBOX_FREE), rank - 2));
          }
        }
        ++nseg;
        tc_fence_after();
        const float inv = un.whole ? 1.0f / lsg : 1.0f;
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
}

// ------------------------------------------------------------------------------------------------
// the fused kernel: grid = 4 x clusters, one CTA per SM
// ------------------------------------------------------------------------------------------------
template <int E>
__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(kFuThreads, 1)
    abs_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmH,
                     const __grid_constant__ CUtensorMap tmH64, const AbsArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t rank = cluster_ctarank();
  const int cl = blockIdx.x >> 2;
  uint32_t tmem_cols = 0, tmem_addr = 0;
  if (rank < 2) fu_scorer<E>(smem, rank, cl, a, &tmQ, &tmH, tmem_cols, tmem_addr);
  else fu_value<E>(smem, rank, cl, a, &tmH64, tmem_cols, tmem_addr);
  // no CTA leaves while a peer may still access its shared memory or arrive on its barriers
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc_cg2(tmem_addr, tmem_cols);
  }
}

}  // namespace whale
