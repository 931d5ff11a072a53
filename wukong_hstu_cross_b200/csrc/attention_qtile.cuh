// attention_qtile.cuh — Eq. (4) of WHALE (gist.science technical summary, section 2.1, Attention-
// Based Fusion Module) for many queries per history: the serving shape, where the tokens of every
// candidate of one request attend to the request's one long history (pith.science verdict, the
// amortisation of footnote 1). A query-tiled online-softmax attention on the tcgen05 tensor cores.
//
// One CTA per (example b, tile of 128 queries, box of HB = 64 / d_h heads). The history is walked
// in blocks of 128 rows; per block and head h of the box:
//   S_h = Q_h K_h^T   (M = 128 queries, N = 128 rows, K = d_h) into TMEM,
//   the softmax warps of head h (one thread per query row, the row's 128 scores in registers) free
//   S_h at once, keep a lazy reference (raised only when a block maximum exceeds it by 2^8, with
//   the O rescale in TMEM then), and write P_h = 2^(s - m) as bf16 into shared memory,
//   O_h += P_h V  (M = 128, N = 64: the box's 64 value columns, K = 128 rows; V as the MN-major
//   operand) into TMEM; only head h's d_h columns of O_h are kept.
// Q, K and V come by TMA in 64-column boxes (128-byte swizzle); K and V of a block share a stage.
// The output is O / l as a bf16 pair (hi, lo), like the split-L kernel's.
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace whale {

struct QtArgs {
  const int* offsets;     // [B+1]
  __nv_bfloat16* out;     // A hi [B*N, d]
  __nv_bfloat16* out_lo;  // A lo (may be null)
  int B, N, d;
  int n_qt;               // query tiles per example, ceil(N / 128)
  int n_hb;               // head boxes, n_heads / HB
  int v_col0;             // first value column of the K|V tensor (d; 0 with shared K = V)
  long long total_L;
  float scale_log2;       // log2(e) / sqrt(d_h)
};

template <int DH>
struct QtSmem {
  static constexpr int HB = 64 / DH;                      // heads per 64-column box
  static constexpr uint32_t BOX = 128 * 64 * 2;           // 128 rows x 64 columns
  static constexpr uint32_t STAGE = 2 * BOX;              // K box | V box
  static constexpr int ST = 3;
  static constexpr uint32_t P_HEAD = 2 * 128 * 64 * 2;    // 128 queries x 128 rows: two 64-row blocks
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + (int)BOX;
  static constexpr int OFF_P = OFF_KV + ST * (int)STAGE;
  static constexpr int OFF_BAR = OFF_P + HB * (int)P_HEAD;
  // qfull, kvfull[ST], kvempty[ST], sfull[HB], sfree[HB], pfull[HB], pfree[HB], tmem slot, abort flag
  static constexpr int USED = OFF_BAR + (1 + 2 * ST + 4 * HB) * 8 + 16;
  static constexpr size_t BYTES = 1024 + (size_t)USED;
  static constexpr uint32_t TMEM_COLS = HB == 2 ? 512 : 256;  // S: HB x 128, O: HB x 64
  static_assert(BYTES <= 232448, "shared memory of one CTA");
};
constexpr int kQtThreads = 320;
constexpr float kQtLazy = 8.0f;  // log2 headroom before the softmax reference is raised

// 2^x on the FMA pipe, for x <= kQtLazy: Cody-Waite reduction x = n + f with n = round(x) (the
// 1.5 * 2^23 rounding trick) and f in [-1/2, 1/2]; 2^f by a degree-3 polynomial fitted to minimise
// the relative error on that interval (max relative error 7.51e-5, below the 2^-9 of the bf16
// weights it produces); 2^n added to the exponent bits. Arguments below -125 give 2^-125 (no
// denormals or exponent wrap; used only for blocks without masked rows). Takes a share of the
// exponentials off the MUFU unit.
__device__ __forceinline__ float exp2_fma(float x) {
  const float xc = fmaxf(x, -125.0f);
  const float big = 12582912.0f;  // 1.5 * 2^23
  const float t = xc + big;
  const float f = xc - (t - big);
  const float p = fmaf(fmaf(fmaf(0.05517113208770752f, f, 0.24261008203029633f), f, 0.6932609677314758f), f,
                       0.9999281167984009f);
  return __int_as_float(__float_as_int(p) + ((__float_as_int(t) - __float_as_int(big)) << 23));
}

template <int DH>
__global__ void __launch_bounds__(kQtThreads, 1)
    attn_qtile_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
                      const QtArgs a) {
  using L = QtSmem<DH>;
  constexpr int HB = L::HB, ST = L::ST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kvfull = qfull + 1;
  uint64_t* kvempty = kvfull + ST;
  uint64_t* sfull = kvempty + ST;  // [HB] S_h in TMEM (MMA commit)
  uint64_t* sfree = sfull + HB;    // [HB] S_h read by the 4 softmax warps of head h
  uint64_t* pfull = sfree + HB;    // [HB] P_h written by the 4 softmax warps of head h
  uint64_t* pfree = pfull + HB;    // [HB] P_h read by the MMA (commit after O_h += P_h V)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pfree + HB);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hb = blockIdx.x % a.n_hb;
  const int qt = (blockIdx.x / a.n_hb) % a.n_qt;
  const int b = blockIdx.x / (a.n_hb * a.n_qt);

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&kvfull[s], 1);
      mbar_init(&kvempty[s], 1);
    }
    for (int h = 0; h < HB; ++h) {
      mbar_init(&sfull[h], 1);
      mbar_init(&sfree[h], 4);
      mbar_init(&pfull[h], 4);
      mbar_init(&pfree[h], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  long long lo = a.offsets[b], hi = a.offsets[b + 1];
  lo = lo < 0 ? 0 : (lo > a.total_L ? a.total_L : lo);
  hi = hi < lo ? lo : (hi > a.total_L ? a.total_L : hi);
  const long long len = hi - lo;
  const int nblk = (int)((len + 127) / 128);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && nblk > 0) {
      mbar_arrive_expect_tx(qfull, L::BOX);
      tma_load_2d(smem + L::OFF_Q, &tmQ, hb * 64, b * a.N + qt * 128, qfull);
      for (int i = 0; i < nblk; ++i) {
        const int s = i % ST;
        if (i >= ST && !mbar_wait(&kvempty[s], (i / ST - 1) & 1, abort_flag)) break;
        uint8_t* st = smem + L::OFF_KV + s * L::STAGE;
        mbar_arrive_expect_tx(&kvfull[s], L::STAGE);
        const int row = (int)(lo + 128ll * i);
        tma_load_2d(st, &tmKV, hb * 64, row, &kvfull[s]);
        tma_load_2d(st + L::BOX, &tmKV, a.v_col0 + hb * 64, row, &kvfull[s]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && nblk > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 64) | kIdescBMnMajor;
      const uint32_t q_base = smem_u32(smem + L::OFF_Q);
      auto issue_s = [&](int i, int h) {
        const uint32_t k_base = smem_u32(smem + L::OFF_KV + (i % ST) * L::STAGE);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
          umma_f16(tmem_base + h * 128, sdesc_k_sw128(q_base + h * DH * 2 + kk * 32),
                   sdesc_k_sw128(k_base + h * DH * 2 + kk * 32), idesc_s, kk > 0 ? 1u : 0u);
        umma_commit(&sfull[h]);
      };
      bool ok = mbar_wait(qfull, 0, abort_flag) && mbar_wait(&kvfull[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int h = 0; h < HB; ++h) issue_s(0, h);
      }
      for (int i = 0; i < nblk && ok; ++i) {
        const bool more = i + 1 < nblk;
        if (more && !mbar_wait(&kvfull[(i + 1) % ST], ((i + 1) / ST) & 1, abort_flag)) break;
        const uint32_t v_base = smem_u32(smem + L::OFF_KV + (i % ST) * L::STAGE + L::BOX);
        for (int h = 0; h < HB; ++h) {
          // S_h of the next block as soon as the softmax warps have read this one
          if (more) {
            if (!mbar_wait(&sfree[h], i & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(i + 1, h);
          }
          if (!mbar_wait(&pfull[h], i & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t p_base = smem_u32(smem + L::OFF_P + h * L::P_HEAD);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16(tmem_base + HB * 128 + h * 64, sdesc_k_sw128(p_base + (kk >> 2) * 16384 + (kk & 3) * 32),
                     sdesc_mn_sw128(v_base + kk * 2048, L::BOX, 1024), idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&pfree[h]);
        }
        umma_commit(&kvempty[i % ST]);
      }
    }
  } else if (warp < 2 + 4 * HB) {
    // ---------------- softmax and output (warps 2.., 4 per head: one thread per query row) ----------
    const int q4 = warp & 3;
    const int h = (warp - 2) >> 2;
    const int row = q4 * 32 + lane;
    const int qrow = qt * 128 + row;                           // query within the example
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t s_tm = tmem_base + h * 128 + lane_off;
    const uint32_t o_tm = tmem_base + HB * 128 + h * 64 + lane_off;
    uint8_t* p_row = smem + L::OFF_P + h * L::P_HEAD + row * 128;
    float m_run = 0.f, l = 0.f;
    bool ok = true;
    for (int i = 0; i < nblk && ok; ++i) {
      if (!mbar_wait(&sfull[h], i & 1, abort_flag)) break;
      tc_fence_after();
      uint32_t v[128];
      tmem_ld_32x32b_x32(s_tm + 0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld_32x32b_x32(s_tm + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_ld_32x32b_x32(s_tm + 64, *reinterpret_cast<uint32_t(*)[32]>(&v[64]));
      tmem_ld_32x32b_x32(s_tm + 96, *reinterpret_cast<uint32_t(*)[32]>(&v[96]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sfree[h]);  // the MMA may write the next block's S_h
      const long long rem = len - 128ll * i;
      const int nv = rem > 128 ? 128 : (int)rem;
      // block maximum over the raw scores (the scale is positive), eight independent chains
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
      if (nv == 128) {
#pragma unroll
        for (int j = 0; j < 128; ++j) mx[j & 7] = fmaxf(mx[j & 7], __uint_as_float(v[j]));
      } else {
#pragma unroll
        for (int j = 0; j < 128; ++j) {
          if (j >= nv) v[j] = __float_as_uint(-INFINITY);
          mx[j & 7] = fmaxf(mx[j & 7], __uint_as_float(v[j]));
        }
      }
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * a.scale_log2;
      float m_new = m_run;
      if (i == 0 || mt > m_run + kQtLazy) m_new = mt;
      // P_h of the previous block has been read and O_h updated: P_h may be rewritten, O_h rescaled
      if (i > 0 && !mbar_wait(&pfree[h], (i - 1) & 1, abort_flag)) break;
      if (i > 0 && __any_sync(0xffffffffu, m_new != m_run)) {
        tc_fence_after();
        const float f = fast_exp2(m_run - m_new);
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(o_tm + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
          tmem_st_32x32b_x32(o_tm + c * 32, o);
        }
        tmem_st_wait();
        l *= f;
      }
      m_run = m_new;
      // p = 2^(s * scale - m): in full blocks 5 of every 16 eight-row chunks take the FMA-pipe
      // polynomial, the rest (and every block with masked rows) MUFU; the choice is made per block
      // so that inside the loop it is a compile-time constant
      float lsum = 0.f;
      auto exp_pass = [&](auto full_tag) {
        constexpr bool kFull = decltype(full_tag)::value;
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 16; ++c) {  // 16 chunks of 8 rows: blocks of 64 rows, 128-byte swizzle
          uint32_t pk[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float x0 = fmaf(__uint_as_float(v[8 * c + 2 * k]), a.scale_log2, -m_run);
            const float x1 = fmaf(__uint_as_float(v[8 * c + 2 * k + 1]), a.scale_log2, -m_run);
            float p0, p1;
            if (kFull && (c % 3) == 1) {
              p0 = exp2_fma(x0);
              p1 = exp2_fma(x1);
            } else {
              p0 = fast_exp2(x0);
              p1 = fast_exp2(x1);
            }
            ls[k] += p0 + p1;
            pk[k] = pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(p_row + (c >> 3) * 16384 + (((c & 7) ^ (row & 7)) * 16)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      };
      if (nv == 128) exp_pass(std::true_type{});
      else exp_pass(std::false_type{});
      l += lsum;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pfull[h]);
    }
    // output: O_h / l for this head's d_h columns of the box (empty history: A = 0)
    bool have = nblk > 0 && ok;
    if (have && !mbar_wait(&pfree[h], (nblk - 1) & 1, abort_flag)) have = false;
    // tcgen05.ld is warp-collective: every lane loads, only rows inside the example are stored
    const bool store = qrow < a.N;
    const size_t orow = (size_t)b * a.N + (store ? qrow : 0);
    const int col0 = (hb * HB + h) * DH;
    const float inv = have && l > 0.f ? 1.0f / l : 0.f;
    if (have) tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < DH / 32; ++c) {
      uint32_t o[32];
      if (have) {
        tmem_ld_32x32b_x32(o_tm + h * DH + c * 32, o);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0u;
      }
      if (!store) continue;
      uint32_t hi[16], lo16[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float x0 = __uint_as_float(o[2 * j]) * inv, x1 = __uint_as_float(o[2 * j + 1]) * inv;
        const __nv_bfloat162 hv = __floats2bfloat162_rn(x0, x1);
        hi[j] = *reinterpret_cast<const uint32_t*>(&hv);
        const float2 hf2 = __bfloat1622float2(hv);
        lo16[j] = pack_bf16x2(x0 - hf2.x, x1 - hf2.y);
      }
      uint4* dh = reinterpret_cast<uint4*>(a.out + orow * a.d + col0 + c * 32);
#pragma unroll
      for (int k = 0; k < 4; ++k) dh[k] = make_uint4(hi[4 * k], hi[4 * k + 1], hi[4 * k + 2], hi[4 * k + 3]);
      if (a.out_lo) {
        uint4* dl = reinterpret_cast<uint4*>(a.out_lo + orow * a.d + col0 + c * 32);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          dl[k] = make_uint4(lo16[4 * k], lo16[4 * k + 1], lo16[4 * k + 2], lo16[4 * k + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

}  // namespace whale
