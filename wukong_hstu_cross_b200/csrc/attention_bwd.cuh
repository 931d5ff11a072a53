// attention_bwd.cuh — backward of Eq. (4) on the warp-level tensor cores (bf16 mode).
//
// For example b, head j (s = q k^T / sqrt(d_h), p = softmax over the example's history rows,
// a = p v), with the upstream gradient da:
//   dp = da v^T,  delta_n = sum_t p_nt dp_nt = da_n . a_n,  ds = p (dp - delta),
//   dv = p^T da,  dk = ds^T q / sqrt(d_h),  dq = ds k / sqrt(d_h).
// p is recomputed from the forward's log-sum-exp (the split-L kernel exports it), in base 2:
// p_nt = 2^(s_nt log2(e) / sqrt(d_h) - lse_n).
//
// Schedule: KV-parallel (gist.science technical summary of WHALE, section 2.2, Asymmetric Backward
// Variants). The pages' shapes have few queries per example (N <= 32) against thousands of history
// rows: a CTA owns a chunk of up to 1024 history rows of one example and a group of heads, keeps
// all of the example's queries (q, da, lse, delta) in shared memory, and streams the chunk's K|V
// rows in blocks of 64 (cp.async double buffer). dK and dV of those rows are then complete inside
// the CTA (no reduction over queries, stored once); only dq, a sum over history rows, is
// split across the example's chunks: each CTA adds its chunk's share with fp32 atomics into a dq
// buffer zeroed before the launch (N d values per chunk). The Q-parallel order would split the
// other way (dK, dV reduced across query blocks, L d values per block) and only pays with many
// queries per history.
//
// Per warp: one head, 16 of the block's 64 rows, all NQ (16 or 32) queries:
//   S^T = K Q^T and dP^T = V dA^T (mma.sync m16n8k16, K/V rows as A, Q/dA rows as B),
//   P^T, dS^T in registers, re-packed as A fragments (rows = history rows, k = queries),
//   dV = P^T dA, dK = dS^T Q (B fragments of dA / Q by transposing ldmatrix),
//   dQ^T += K^T dS^T (K^T by transposing ldmatrix, dS^T staged in shared memory per warp).
// Precision: every operand is a bf16 hi/lo pair (K, V, Q from the recomputed projections, dA, and P
// and dS split in registers) and every product takes three MMAs (hi hi, lo hi, hi lo), so the
// contractions carry about 16 significant bits: bf16 storage of K and V alone put the weight
// gradients' worst elements near the parity bound. dK and dV are stored as pairs.
#pragma once

#include "ptx.cuh"

namespace whale {

constexpr int kBwdChunk = 1024;  // history rows per CTA of the attention backward

struct AttnBwdArgs {
  // every operand is a bf16 pair (hi, lo: about 16 significant bits); the lo pointers are required
  const __nv_bfloat16 *q, *q_lo;    // [B*N, d]
  const __nv_bfloat16 *kv, *kv_lo;  // [total_L, kvw]
  const __nv_bfloat16 *da, *da_lo;  // [B*N, d] dLoss/dA
  const float* lse;          // [B*N, h] log2 softmax denominators (scaled units)
  const float* delta;        // [B*N, h]
  const int* offsets;        // [B+1]
  const int* cstart;         // [B+1] first chunk of each example; cstart[B] = number of chunks
  int chunk;                 // history rows per chunk (the tensor-core kernel; the other takes kBwdChunk)
  float* dq;                 // [B*N, d] fp32, zero at launch (atomics)
  __nv_bfloat16 *dkv, *dkv_lo;  // [total_L, kvw]: dK in columns [0, d), dV from v_col0 (shared K = V: dK + dV)
  const float* row_scale;     // [total_L] or null: dK and dV of history row t are stored times row_scale[t]
  int B, N, d, n_heads, kvw, v_col0, shared_kv;
  long long total_L;
  float scale_log2;          // log2(e) / sqrt(d_h)
  float scale;               // 1 / sqrt(d_h)
};

// CTA: a head group of HG heads (HG d_h = 128 columns), blocks of 64 history rows; per head four
// warps of 16 rows each.
template <int DH, int NQ>
struct AttnBwdCfg {
  static constexpr int HG = 128 / DH;
  static constexpr int KB = 64;                 // history rows per block
  static constexpr int WPH = 4;                 // warps per head (16 rows each)
  static constexpr int WARPS = WPH * HG;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int COLS = HG * DH;          // 128 columns of the head group
  static constexpr int ROWB = COLS * 2 + 16;    // padded row (bytes): conflict-free ldmatrix
  static constexpr int QBYTES = NQ * ROWB;      // one of q, q_lo, da, da_lo
  static constexpr int KVBYTES = KB * ROWB;     // one of k, k_lo, v, v_lo for one block
  static constexpr int DSROW = NQ * 2 + 16;     // dS^T staging row (bytes), per warp [16][NQ] hi and lo
  static constexpr int DSBYTES = 2 * 16 * DSROW;
  static constexpr int OFF_Q = 0;                           // q, q_lo, da, da_lo
  static constexpr int OFF_KV = 4 * QBYTES;                 // [2 buffers][k, k_lo, v, v_lo]
  static constexpr int OFF_DS = OFF_KV + 8 * KVBYTES;
  static constexpr int OFF_LSE = OFF_DS + WARPS * DSBYTES;
  static constexpr int OFF_DEL = OFF_LSE + NQ * HG * 4;
  static constexpr int BYTES = OFF_DEL + NQ * HG * 4;
  static_assert(DH % 16 == 0 && NQ % 16 == 0 && COLS == 128, "tile shape");
  static_assert(BYTES <= 232448, "shared memory");
};

// cstart[b] = sum_{b' < b} ceil(L_b' / rows), capped at cmax; one block of 1024 threads.
__global__ void __launch_bounds__(1024) chunk_starts_kernel(const int* __restrict__ offsets, int B, long long total_L,
                                                            int rows, int cmax, int* __restrict__ cstart) {
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
    if (L > 0) sum += (L + rows - 1) / rows;
  }
  part[threadIdx.x] = (int)(sum < cmax ? sum : cmax);
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] = min(part[threadIdx.x] + v, cmax);
    __syncthreads();
  }
  long long run = threadIdx.x > 0 ? part[threadIdx.x - 1] : 0;
  for (int b = b0; b < b1; ++b) {
    cstart[b] = (int)run;
    const long long L = clampo(b + 1) - clampo(b);
    if (L > 0) run += (L + rows - 1) / rows;
    if (run > cmax) run = cmax;
  }
  if (threadIdx.x == 1023) cstart[B] = part[1023];
}

// delta[row, j] = sum over head j's columns of da * a (a = a_hi + a_lo, the forward's output as a
// bf16 pair), and da as a bf16 pair: da32 fp32 with row stride ld_da. A thread takes 8 consecutive
// columns; the d_h / 8 threads of one (row, head) are consecutive lanes of one warp (d_h / 8 a power
// of two dividing 32) and add their partial sums with shuffles.
__global__ void attn_bwd_prep_kernel(const float* __restrict__ da32, long long ld_da, const __nv_bfloat16* __restrict__ a_hi,
                                     const __nv_bfloat16* __restrict__ a_lo, long long rows, int d, int n_heads,
                                     float* __restrict__ delta, __nv_bfloat16* __restrict__ da_hi,
                                     __nv_bfloat16* __restrict__ da_lo) {
  pdl_wait();
  pdl_trigger();
  const int gph = (d / n_heads) >> 3;  // threads per (row, head)
  const int cg = d >> 3;
  const long long n = rows * cg;
  const int lane = threadIdx.x & 31;
  const long long stride = (long long)gridDim.x * blockDim.x;
  // warp-uniform trip count: every lane of a warp takes part in the shuffles
  for (long long base = (long long)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < n; base += stride) {
    const long long i = base + lane;
    const bool act = i < n;
    float s = 0.f;
    long long r = 0;
    int c = 0;
    if (act) {
      r = n < (1ll << 31) ? (long long)((unsigned)i / (unsigned)cg) : i / cg;
      c = (int)(i - r * cg) * 8;
      const float4 g0 = *reinterpret_cast<const float4*>(da32 + r * ld_da + c);
      const float4 g1 = *reinterpret_cast<const float4*>(da32 + r * ld_da + c + 4);
      const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      const uint4 ah = *reinterpret_cast<const uint4*>(a_hi + r * d + c);
      const uint4 al = a_lo ? *reinterpret_cast<const uint4*>(a_lo + r * d + c) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t wh[4] = {ah.x, ah.y, ah.z, ah.w}, wl[4] = {al.x, al.y, al.z, al.w};
      uint32_t h[4], l[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // bf16 -> fp32: the bf16 bits are the high half of the fp32 word
        const float a0 = __uint_as_float(wh[j] << 16) + __uint_as_float(wl[j] << 16);
        const float a1 = __uint_as_float(wh[j] & 0xffff0000u) + __uint_as_float(wl[j] & 0xffff0000u);
        s = fmaf(g[2 * j], a0, s);
        s = fmaf(g[2 * j + 1], a1, s);
        const __nv_bfloat162 gh = __floats2bfloat162_rn(g[2 * j], g[2 * j + 1]);
        h[j] = *reinterpret_cast<const uint32_t*>(&gh);
        const float2 gf = __bfloat1622float2(gh);
        l[j] = pack_bf16x2(g[2 * j] - gf.x, g[2 * j + 1] - gf.y);
      }
      *reinterpret_cast<uint4*>(da_hi + r * d + c) = make_uint4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<uint4*>(da_lo + r * d + c) = make_uint4(l[0], l[1], l[2], l[3]);
    }
    for (int o = gph >> 1; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (act && (lane & (gph - 1)) == 0) delta[r * n_heads + c / (d / n_heads)] = s;
  }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// (a_hi + a_lo)(b_hi + b_lo) without the lo * lo term (below 2^-16 of the product): three MMAs.
__device__ __forceinline__ void mma3(float (&c)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4], uint32_t bh0,
                                     uint32_t bh1, uint32_t bl0, uint32_t bl1) {
  mma_bf16_16816(c, ah[0], ah[1], ah[2], ah[3], bh0, bh1);
  mma_bf16_16816(c, al[0], al[1], al[2], al[3], bh0, bh1);
  mma_bf16_16816(c, ah[0], ah[1], ah[2], ah[3], bl0, bl1);
}

// hi and lo bf16 halves of two fp32 values, packed as two bf16x2 words
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  const float2 hf = __bfloat1622float2(h);
  lo = pack_bf16x2(x0 - hf.x, x1 - hf.y);
}

template <int DH, int NQ>
__global__ void __launch_bounds__(AttnBwdCfg<DH, NQ>::THREADS, 1) attn_bwd_kernel(const AttnBwdArgs a) {
  using C = AttnBwdCfg<DH, NQ>;
  constexpr int HG = C::HG;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x, hg = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const int U = a.cstart[a.B];
  if (chunk >= U) return;
  // example of this chunk: largest b with cstart[b] <= chunk
  int lo = 0, hi = a.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.cstart[mid] <= chunk) lo = mid;
    else hi = mid - 1;
  }
  const int b = lo;
  auto clampo = [&](int e) -> long long {
    long long o = a.offsets[e];
    return o < 0 ? 0 : (o > a.total_L ? a.total_L : o);
  };
  const long long lo_b = clampo(b);
  long long hi_b = clampo(b + 1);
  if (hi_b < lo_b) hi_b = lo_b;
  const long long k0 = lo_b + (long long)(chunk - a.cstart[b]) * kBwdChunk;
  const long long k1 = min(hi_b, k0 + kBwdChunk);
  if (k0 >= k1) return;  // uniform across the CTA
  const int col0 = hg * C::COLS;
  const uint32_t sbase = smem_u32(smem);
  float* lse_s = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* del_s = reinterpret_cast<float*>(smem + C::OFF_DEL);

  // ---- the example's queries: q, da as pairs (zero past N), lse (+inf past N: p = 0), delta ----
  {
    const __nv_bfloat16* src[4] = {a.q, a.q_lo, a.da, a.da_lo};
    for (int i = threadIdx.x; i < 4 * NQ * (C::COLS / 8); i += C::THREADS) {
      const int t = i / (NQ * (C::COLS / 8)), rem = i % (NQ * (C::COLS / 8));
      const int n = rem / (C::COLS / 8), c8 = rem % (C::COLS / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (n < a.N) v = *reinterpret_cast<const uint4*>(src[t] + ((long long)b * a.N + n) * a.d + col0 + 8 * c8);
      *reinterpret_cast<uint4*>(smem + C::OFF_Q + t * C::QBYTES + n * C::ROWB + c8 * 16) = v;
    }
  }
  for (int i = threadIdx.x; i < NQ * HG; i += C::THREADS) {
    const int n = i / HG, hl = i % HG;
    const long long idx = ((long long)b * a.N + n) * a.n_heads + hg * HG + hl;
    lse_s[i] = n < a.N ? a.lse[idx] : INFINITY;
    del_s[i] = n < a.N ? a.delta[idx] : 0.f;
  }

  // ---- K|V block loader (hi and lo halves): rows [r0, r0 + 64) of the chunk, zero past k1 ----
  const int nblk = (int)((k1 - k0 + C::KB - 1) / C::KB);
  auto kv_tile = [&](int buf, int which) -> uint32_t {  // which: 0 k, 1 k_lo, 2 v, 3 v_lo
    return sbase + C::OFF_KV + (buf * 4 + which) * C::KVBYTES;
  };
  auto load_block = [&](int blk) {
    const int buf = blk & 1;
    const long long r0 = k0 + (long long)blk * C::KB;
    const int nt = a.shared_kv ? 2 : 4;
    for (int i = threadIdx.x; i < nt * C::KB * (C::COLS / 8); i += C::THREADS) {
      const int which = i / (C::KB * (C::COLS / 8)), rem = i % (C::KB * (C::COLS / 8));
      const int r = rem / (C::COLS / 8), c8 = rem % (C::COLS / 8);
      const long long row = r0 + r;
      const bool ok = row < k1;
      const long long srow = ok ? row : lo_b;  // a valid address even when nothing is read
      const __nv_bfloat16* base = (which & 1) ? a.kv_lo : a.kv;
      const int col = col0 + 8 * c8 + ((which >> 1) ? a.v_col0 : 0);
      cp_async16(kv_tile(buf, which) + r * C::ROWB + c8 * 16, base + srow * a.kvw + col, ok ? 16u : 0u);
    }
  };

  const int hl = warp / C::WPH, kq = warp % C::WPH;
  const int hc = hl * DH;    // head's first column inside the group tile
  const int kr0 = 16 * kq;   // this warp's first row inside the block
  const int g = lane >> 2, qd = lane & 3, mi = lane >> 3, r8 = lane & 7;
  const uint32_t q_s = sbase + C::OFF_Q, ql_s = q_s + C::QBYTES;
  const uint32_t da_s = q_s + 2 * C::QBYTES, dal_s = q_s + 3 * C::QBYTES;
  uint8_t* ds_p = smem + C::OFF_DS + warp * C::DSBYTES;  // [16][NQ] hi, then [16][NQ] lo
  const uint32_t ds_s = smem_u32(ds_p), dsl_s = ds_s + 16 * C::DSROW;

  float qacc[DH / 16][NQ / 8][4];  // dQ^T of this warp's head: [d_h rows][queries]
#pragma unroll
  for (int i = 0; i < DH / 16; ++i)
#pragma unroll
    for (int j = 0; j < NQ / 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) qacc[i][j][e] = 0.f;

  load_block(0);
  cp_async_commit();
  for (int blk = 0; blk < nblk; ++blk) {
    if (blk + 1 < nblk) {
      load_block(blk + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // block blk landed (and, on the first pass, the query tiles)
    const int buf = blk & 1;
    const uint32_t k_s = kv_tile(buf, 0), kl_s = kv_tile(buf, 1);
    const uint32_t v_s = a.shared_kv ? k_s : kv_tile(buf, 2), vl_s = a.shared_kv ? kl_s : kv_tile(buf, 3);
    const long long row0 = k0 + (long long)blk * C::KB + kr0;  // history row of this warp's tile row 0

    // ---- S^T = K Q^T, dP^T = V dA^T: [16 rows] x [NQ queries], pairs on both sides ----
    float st[NQ / 8][4], dpt[NQ / 8][4];
#pragma unroll
    for (int nt = 0; nt < NQ / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[nt][e] = dpt[nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < DH / 16; ++ks) {
      uint32_t akh[4], akl[4], avh[4], avl[4];
      {
        const int row = kr0 + r8 + 8 * (mi & 1);
        const int colb = (hc + 16 * ks + 8 * (mi >> 1)) * 2;
        ldsm_x4(k_s + row * C::ROWB + colb, akh[0], akh[1], akh[2], akh[3]);
        ldsm_x4(kl_s + row * C::ROWB + colb, akl[0], akl[1], akl[2], akl[3]);
        ldsm_x4(v_s + row * C::ROWB + colb, avh[0], avh[1], avh[2], avh[3]);
        ldsm_x4(vl_s + row * C::ROWB + colb, avl[0], avl[1], avl[2], avl[3]);
      }
#pragma unroll
      for (int np = 0; np < NQ / 16; ++np) {
        const int qrow = 16 * np + 8 * (mi >> 1) + r8;
        const int colb = (hc + 16 * ks + 8 * (mi & 1)) * 2;
        uint32_t qh[4], qlw[4], eh[4], el[4];
        ldsm_x4(q_s + qrow * C::ROWB + colb, qh[0], qh[1], qh[2], qh[3]);
        ldsm_x4(ql_s + qrow * C::ROWB + colb, qlw[0], qlw[1], qlw[2], qlw[3]);
        ldsm_x4(da_s + qrow * C::ROWB + colb, eh[0], eh[1], eh[2], eh[3]);
        ldsm_x4(dal_s + qrow * C::ROWB + colb, el[0], el[1], el[2], el[3]);
        mma3(st[2 * np], akh, akl, qh[0], qh[1], qlw[0], qlw[1]);
        mma3(st[2 * np + 1], akh, akl, qh[2], qh[3], qlw[2], qlw[3]);
        mma3(dpt[2 * np], avh, avl, eh[0], eh[1], el[0], el[1]);
        mma3(dpt[2 * np + 1], avh, avl, eh[2], eh[3], el[2], el[3]);
      }
    }

    // ---- P^T, dS^T (rows past the chunk and queries past N give 0): A fragments (pairs) and the
    // dS^T staging (pairs) ----
    uint32_t pah[NQ / 16][4], pal[NQ / 16][4], dsh[NQ / 16][4], dsl[NQ / 16][4];
#pragma unroll
    for (int nt = 0; nt < NQ / 8; ++nt) {
      float pv[4], dsv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int rloc = g + 8 * (e >> 1);
        const int n = 8 * nt + 2 * qd + (e & 1);
        const bool ok = row0 + rloc < k1;
        const float p = ok ? fast_exp2(fmaf(st[nt][e], a.scale_log2, -lse_s[n * HG + hl])) : 0.f;
        pv[e] = p;
        dsv[e] = p * (dpt[nt][e] - del_s[n * HG + hl]);
      }
      uint32_t h0, l0, h1, l1;
      split2(dsv[0], dsv[1], h0, l0);
      split2(dsv[2], dsv[3], h1, l1);
      // dS^T staging [row][query] (unscaled; dQ^T is scaled once at the end)
      *reinterpret_cast<uint32_t*>(ds_p + g * C::DSROW + (8 * nt + 2 * qd) * 2) = h0;
      *reinterpret_cast<uint32_t*>(ds_p + (g + 8) * C::DSROW + (8 * nt + 2 * qd) * 2) = h1;
      *reinterpret_cast<uint32_t*>(ds_p + (16 + g) * C::DSROW + (8 * nt + 2 * qd) * 2) = l0;
      *reinterpret_cast<uint32_t*>(ds_p + (16 + g + 8) * C::DSROW + (8 * nt + 2 * qd) * 2) = l1;
      const int kt = nt >> 1, hi8 = nt & 1;
      split2(pv[0], pv[1], pah[kt][2 * hi8], pal[kt][2 * hi8]);
      split2(pv[2], pv[3], pah[kt][2 * hi8 + 1], pal[kt][2 * hi8 + 1]);
      // dK = (dS^T / sqrt(d_h)) Q: the scale folded into the A fragments
      split2(dsv[0] * a.scale, dsv[1] * a.scale, dsh[kt][2 * hi8], dsl[kt][2 * hi8]);
      split2(dsv[2] * a.scale, dsv[3] * a.scale, dsh[kt][2 * hi8 + 1], dsl[kt][2 * hi8 + 1]);
    }
    __syncwarp();

    // ---- dV = P^T dA and dK = dS^T Q / sqrt(d_h): [16 rows] x [d_h] ----
    float acc[DH / 8][4];
    auto zero_acc = [&]() {
#pragma unroll
      for (int nt = 0; nt < DH / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    };
    auto mul_acc = [&](const uint32_t (&afh)[NQ / 16][4], const uint32_t (&afl)[NQ / 16][4], uint32_t src_s,
                       uint32_t srcl_s) {
#pragma unroll
      for (int kt = 0; kt < NQ / 16; ++kt) {
#pragma unroll
        for (int cp = 0; cp < DH / 16; ++cp) {
          const int qrow = 16 * kt + 8 * (mi & 1) + r8;
          const int colb = (hc + 16 * cp + 8 * (mi >> 1)) * 2;
          uint32_t bh[4], bl[4];
          ldsm_x4_t(src_s + qrow * C::ROWB + colb, bh[0], bh[1], bh[2], bh[3]);
          ldsm_x4_t(srcl_s + qrow * C::ROWB + colb, bl[0], bl[1], bl[2], bl[3]);
          mma3(acc[2 * cp], afh[kt], afl[kt], bh[0], bh[1], bl[0], bl[1]);
          mma3(acc[2 * cp + 1], afh[kt], afl[kt], bh[2], bh[3], bl[2], bl[3]);
        }
      }
    };
    auto store_acc = [&](int col) {  // col: first column of this head in the dkv row
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const long long row = row0 + g + 8 * hr;
        if (row >= k1) continue;
        __nv_bfloat16* dst = a.dkv + row * a.kvw + col;
        __nv_bfloat16* dstl = a.dkv_lo + row * a.kvw + col;
        const float rs = a.row_scale ? a.row_scale[row] : 1.0f;
#pragma unroll
        for (int nt = 0; nt < DH / 8; ++nt) {
          uint32_t h, l;
          split2(acc[nt][2 * hr] * rs, acc[nt][2 * hr + 1] * rs, h, l);
          *reinterpret_cast<uint32_t*>(dst + 8 * nt + 2 * qd) = h;
          *reinterpret_cast<uint32_t*>(dstl + 8 * nt + 2 * qd) = l;
        }
      }
    };
    zero_acc();
    mul_acc(pah, pal, da_s, dal_s);
    if (!a.shared_kv) {
      store_acc(a.v_col0 + col0 + hc);
      zero_acc();
    }
    mul_acc(dsh, dsl, q_s, ql_s);
    store_acc(col0 + hc);  // dK (plus dV with shared K = V)

    // ---- dQ^T += K^T dS^T: [d_h] x [NQ queries], contracting this warp's 16 rows ----
#pragma unroll
    for (int mt2 = 0; mt2 < DH / 16; ++mt2) {
      const int krow = kr0 + r8 + 8 * (mi >> 1);
      const int colb = (hc + 16 * mt2 + 8 * (mi & 1)) * 2;
      uint32_t ah[4], al[4];
      ldsm_x4_t(k_s + krow * C::ROWB + colb, ah[0], ah[1], ah[2], ah[3]);
      ldsm_x4_t(kl_s + krow * C::ROWB + colb, al[0], al[1], al[2], al[3]);
#pragma unroll
      for (int np = 0; np < NQ / 16; ++np) {
        const int srow = 8 * (mi & 1) + r8;
        const int scolb = (16 * np + 8 * (mi >> 1)) * 2;
        uint32_t bh[4], bl[4];
        ldsm_x4_t(ds_s + srow * C::DSROW + scolb, bh[0], bh[1], bh[2], bh[3]);
        ldsm_x4_t(dsl_s + srow * C::DSROW + scolb, bl[0], bl[1], bl[2], bl[3]);
        mma3(qacc[mt2][2 * np], ah, al, bh[0], bh[1], bl[0], bl[1]);
        mma3(qacc[mt2][2 * np + 1], ah, al, bh[2], bh[3], bl[2], bl[3]);
      }
    }
    __syncthreads();  // every warp is done with buffer `buf` (and its dS^T staging) before it refills
  }

  // ---- dq += this chunk's share (scaled by 1/sqrt(d_h)); rows are queries, columns the head's ----
#pragma unroll
  for (int mt2 = 0; mt2 < DH / 16; ++mt2) {
#pragma unroll
    for (int nt = 0; nt < NQ / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = 16 * mt2 + g + 8 * (e >> 1);
        const int n = 8 * nt + 2 * qd + (e & 1);
        if (n < a.N) atomicAdd(a.dq + ((long long)b * a.N + n) * a.d + col0 + hc + m, qacc[mt2][nt][e] * a.scale);
      }
    }
  }
}

}  // namespace whale
