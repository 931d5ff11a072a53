// gemm_tc.cuh — bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
//   out[M, N'] = epilogue( sum_k A[m, k] * W[n, k] ),  A = [A0 | A1] (two K sources),
//   W row-major [N, K0 + K1] (nn.Linear layout), fp32 accumulation in tensor memory.
//
// Operand precision. With SPLIT, each A source is given as a pair of bf16 tensors (hi, lo)
// with A = hi + lo (about 16 mantissa bits), and every k-step issues two MMAs, hi*W and lo*W,
// into the same accumulator. The weights are bf16 values, so the product is then as precise
// as an fp32 activation times the weight. The token-side (residual-stream) GEMMs use this;
// the history-side K|V projection reads bf16 states directly.
//
// Operand layouts. An operand is K-major (rows of the operand along M or N, K contiguous: the
// nn.Linear layout of W, and the activations of the forward) or, with A_MN / B_MN, MN-major (stored
// [K, M] or [K, N] row-major: M or N contiguous). MN-major tiles are loaded as 64-element-wide TMA
// boxes of 64 K rows (128-byte swizzle) and described to the MMA with the transpose bit of the
// instruction descriptor; they let the backward pass contract over the token or history rows
// (weight gradients dW = dY^T X: both operands MN-major) and multiply by an untransposed weight
// (dX = dY W: W [K, N] is an MN-major B) without transposing anything in memory.
//
// Persistent: CTA c walks the 128 x BN tiles c, c + gridDim.x, ... (N-tiles of a row block are
// adjacent, so A is re-read from L2, not HBM). Warp roles (192 threads, 320 with ROWNORM):
//   warp 0      TMA producer: A (hi, lo) and W tiles (64 columns = 128 B, 128-byte swizzle)
//               into a STAGES-deep ring of shared-memory stages, completion on `full[s]`.
//   warp 1      allocates 2 x BN TMEM columns (two accumulators: tile i uses buffer i % 2, so the
//               epilogue of tile i overlaps the MMAs of tile i+1); one thread issues tcgen05.mma
//               (M=128, N=BN, K=16 per instruction) and commits each stage back to `empty[s]`.
//   warps 2..5  epilogue: thread i of the warp with quadrant q = warp % 4 owns output row
//               32q + i (= TMEM lane).
//   warps 6..9  (ROWNORM) read their row of every A stage from shared memory while the MMAs run
//               and accumulate sum(x^2), so RMSNorm's row factor r = 1/sqrt(mean(x^2) + eps)
//               costs no extra pass over A: RMSNorm(x; g) W^T = r * (x (W diag(g))^T), with
//               diag(g) folded into W beforehand.
// Epilogue value per element (fp32): STORE r*acc; SILU silu(acc); RESID acc + resid32;
// SWIGLU (W rows packed in blocks of 32 = 16 up rows then the 16 matching gate rows)
// silu(r*gate) * r*up; SWIGLU_TIED (W_gate = W_up) silu(r*u) * r*u; QABS acc, written to a
// per-head row order (see GemmArgs). It is then written to any of: out32 (fp32), out_hi (bf16
// rounding), out_lo (bf16 of the rounding residue).
#pragma once

#include "ptx.cuh"

namespace whale {

enum GemmEpi : int { EPI_STORE = 0, EPI_SILU = 1, EPI_RESID = 2, EPI_SWIGLU = 3, EPI_SWIGLU_TIED = 4, EPI_QABS = 5 };

struct GemmArgs {
  int M;                       // rows of A and of the output
  int N;                       // accumulator columns (rows of W), multiple of 32
  int kb0;                     // 64-column K blocks taken from A0
  int kb1;                     // 64-column K blocks taken from A1 (0: single source)
  int tiles_n;                 // N / BN
  int num_tiles;               // ceil(M / 128) * tiles_n (CTAs walk tiles blockIdx.x + i * gridDim.x)
  float inv_k;                 // 1 / (K of the normalised source), ROWNORM only
  float eps;                   // RMSNorm epsilon, ROWNORM only
  __nv_bfloat16* out_hi;       // bf16 output (may be null)
  __nv_bfloat16* out_lo;       // bf16 residue of out_hi (may be null)
  float* out32;                // fp32 output (may be null)
  long long ldo;               // output row stride (elements), shared by the three outputs
  const float* resid32;        // EPI_RESID: fp32 residual [M, N]
  long long ldr;
  // Per-head GEMMs in one launch (head_tiles > 0): output columns come in head blocks of
  // head_tiles n-tiles; the tiles of head j read A from K block j * a_kb_step (block-diagonal W)
  // and from row j * a_row_step (a stack of per-head A matrices).
  int head_tiles;
  int a_kb_step;
  long long a_row_step;
  // EPI_QABS: the accumulator row m = b * qabs_N + n of head block j (qabs_d columns) is written to
  // row b * qabs_rows + j * qabs_N + n, columns relative to the head block.
  int qabs_N, qabs_d, qabs_rows;
  // Split-K (ksplit > 1, one K source): tile t of num_tiles = ksplit * tiles_m * tiles_n takes K blocks
  // [s kb_split, (s + 1) kb_split) of split s = t / (tiles_m tiles_n) and writes its fp32 partial at
  // out32 + s * split_stride (a later pass sums the partials in split order).
  int ksplit, kb_split;
  long long split_stride;
  // ROWNORM: the row factors r are also written here (by the tiles of the first output columns; may be null).
  float* rows_r;
  // SPLIT, K-major A: tmA0 and tmA1 each cover both halves of their pair as two planes (3-D with one
  // K block per stage, 4-D with two), so one copy per source and stage brings hi and lo (in either
  // order: the kernel only ever sums the two halves' products and squares).
  int a_planes;
};


// A pipeline stage holds KPS consecutive 64-column K blocks: [A hi: KPS blocks][A lo: KPS blocks]
// [W: KPS blocks][W lo: KPS blocks], each block a 128-byte-swizzled [rows][64] tile.
template <int BN, bool SPLIT, bool SPLIT_B = false, int KPS = 1, bool TST = false>
struct GemmSmem {
  static constexpr int BM = 128, BK = 64;
  static constexpr uint32_t A_BYTES = BM * BK * 2;  // one K block of A (hi or lo)
  static constexpr uint32_t A_ALL = (SPLIT ? 2 : 1) * KPS * A_BYTES;
  static constexpr uint32_t B_BYTES = BN * BK * 2;  // one K block of W
  static constexpr uint32_t STAGE_BYTES = A_ALL + (SPLIT_B ? 2 : 1) * KPS * B_BYTES;
  // stages fill what the 227 KB of shared memory leaves (one CTA per SM either way): five 40 KB
  // stages for the 64-column hi/lo tiles, two 80 KB ones when a stage holds two K blocks
  // TST: the epilogue's staging buffers for tensor stores, 8 KB per epilogue warp (after the stages)
  static constexpr int STG_BYTES = TST ? 4 * 8192 : 0;
  static constexpr int FIXED = 1024 /*alignment slack*/ + STG_BYTES + 2 * 128 * 4 /*row factors*/ + 256 /*barriers*/;
  static constexpr int STAGES =
      ((232448 - FIXED) / (int)STAGE_BYTES) > 8 ? 8 : ((232448 - FIXED) / (int)STAGE_BYTES);
  static constexpr size_t BYTES = FIXED + STAGES * (size_t)STAGE_BYTES;
};

// silu(x) = x / (1 + e^-x) with the fast (approximate-reciprocal) divide: a few ulp of fp32, far below
// the 16 bits the hi/lo outputs keep; 0 once the denominator passes 2^126 (silu there is below 2^-119).
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word (integer-pipe shift
// and mask, no conversion instruction). The first element of each pair is the low half.
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Write NV consecutive fp32 values (NV multiple of 8) of one row to the requested outputs.
template <int NV>
__device__ __forceinline__ void store_row_chunk(const GemmArgs& g, long long off, const float* x,
                                                long long off32 = 0) {
  if (g.out32) {
    float4* d = reinterpret_cast<float4*>(g.out32 + off32 + off);
#pragma unroll
    for (int i = 0; i < NV / 4; ++i) d[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
  }
  if (g.out_hi) {
    uint32_t hi[NV / 2], lo[NV / 2];
#pragma unroll
    for (int j = 0; j < NV / 2; ++j) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
      hi[j] = *reinterpret_cast<const uint32_t*>(&h);
      const float2 hf = __bfloat1622float2(h);
      lo[j] = pack_bf16x2(x[2 * j] - hf.x, x[2 * j + 1] - hf.y);
    }
    uint4* dh = reinterpret_cast<uint4*>(g.out_hi + off);
#pragma unroll
    for (int i = 0; i < NV / 8; ++i) dh[i] = make_uint4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]);
    if (g.out_lo) {
      uint4* dl = reinterpret_cast<uint4*>(g.out_lo + off);
#pragma unroll
      for (int i = 0; i < NV / 8; ++i) dl[i] = make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]);
    }
  }
}

template <bool ROWNORM>
constexpr int gemm_threads() {
  return ROWNORM ? 320 : 192;
}

// ---- epilogue of one 128-row accumulator tile (shared by the one-CTA and the CTA-pair kernels) ----
// Thread i of TMEM lane quadrant q owns output row 32q + i. Residual tiles of 64 columns: the row's
// residual is loaded into registers before the accumulator is waited for, so its DRAM latency
// overlaps the MMAs.
template <int BN, int EPI>
struct EpiPre {
  static constexpr bool kOn = EPI == EPI_RESID && BN <= 64;
  static constexpr int kN = kOn ? BN / 4 : 1;
};

template <int BN, int EPI>
__device__ __forceinline__ void epi_load_resid(const GemmArgs& args, long long gm, bool row_ok, int n0,
                                               float4 (&pre)[EpiPre<BN, EPI>::kN]) {
  if (EpiPre<BN, EPI>::kOn && row_ok) {
    const float4* rp = reinterpret_cast<const float4*>(args.resid32 + gm * args.ldr + n0);
#pragma unroll
    for (int i = 0; i < EpiPre<BN, EPI>::kN; ++i)
      if (n0 + 4 * i < args.N) pre[i] = rp[i];
  }
}

// t_row: TMEM address of this thread's lane at column 0 of the accumulator; r: row factor.
// off32: extra offset of the fp32 output (a split-K partial's place).
template <int BN, int EPI>
__device__ __forceinline__ void epi_tile(const GemmArgs& args, uint32_t t_row, float r, long long gm, bool row_ok,
                                         int n0, const float4 (&pre)[EpiPre<BN, EPI>::kN], long long off32 = 0) {
  constexpr bool kPre = EpiPre<BN, EPI>::kOn;
  auto chunk = [&](const int c, const uint32_t (&v)[32]) {
    const int col = n0 + c * 32;
    if (!row_ok || col >= args.N) return;
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(v[j]) * r;
    if (EPI == EPI_SWIGLU) {
      float h[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) h[j] = silu_f(x[16 + j]) * x[j];
      store_row_chunk<16>(args, gm * args.ldo + col / 2, h);
    } else {
      if (EPI == EPI_RESID) {
        const float4* rp = reinterpret_cast<const float4*>(args.resid32 + gm * args.ldr + col);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 t = kPre ? pre[(c * 8 + i) % EpiPre<BN, EPI>::kN] : rp[i];
          x[4 * i] += t.x;
          x[4 * i + 1] += t.y;
          x[4 * i + 2] += t.z;
          x[4 * i + 3] += t.w;
        }
      } else if (EPI == EPI_SILU) {
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = silu_f(x[j]);
      } else if (EPI == EPI_SWIGLU_TIED) {
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = silu_f(x[j]) * x[j];
      }
      if (EPI == EPI_QABS) {
        const int head = col / args.qabs_d;
        const long long orow =
            (gm / args.qabs_N) * args.qabs_rows + (long long)head * args.qabs_N + gm % args.qabs_N;
        store_row_chunk<32>(args, orow * args.ldo + (col - head * args.qabs_d), x);
      } else {
        store_row_chunk<32>(args, gm * args.ldo + col, x, off32);
      }
    }
  };
  // Two 32-column accumulator chunks per TMEM wait (BN / 32 is even); the loads are warp-collective,
  // so every lane issues them. Fully unrolled for the register-held residual, whose chunks need
  // constant indices.
#pragma unroll (kPre ? BN / 64 : 1)
  for (int c = 0; c < BN / 32; c += 2) {
    uint32_t va[32], vb[32];
    tmem_ld_32x32b_x32(t_row + c * 32, va);
    tmem_ld_32x32b_x32(t_row + (c + 1) * 32, vb);
    tmem_ld_wait();
    chunk(c, va);
    chunk(c + 1, vb);
  }
}

// The epilogue through shared memory (TST): each 32-column chunk of the warp's 32 rows is staged in
// the warp's 8 KB buffer (fp32: 128-byte rows, 128-byte swizzle; bf16 hi and lo: 64-byte rows,
// 64-byte swizzle) and written by one lane with tensor stores: whole lines per copy, where direct
// stores write 32 rows' 16-byte pieces per instruction. Rows past M are clipped by the tensor maps.
struct EpiStage {
  uint8_t* buf;
  const CUtensorMap *o32, *ohi, *olo;
  int orow;   // first output row of this warp
  int split;  // split-K range of the tile (the fp32 output's third coordinate)
  int lane;
};

template <int BN, int EPI>
__device__ __forceinline__ void epi_tile_tma(const GemmArgs& args, uint32_t t_row, float r, long long gm, bool row_ok,
                                             int n0, const float4 (&pre)[EpiPre<BN, EPI>::kN], const EpiStage& es) {
  constexpr bool kPre = EpiPre<BN, EPI>::kOn;
  const int lane = es.lane;
  uint8_t* s32 = es.buf;
  uint8_t* shi = es.buf + 4096;
  uint8_t* slo = es.buf + 6144;
  // stage 32 values of this lane's row (all lanes) and store them at output column ocol
  auto emit = [&](const float (&x)[32], int ocol, int orow) {
    if (lane == 0) bulk_wait_read<0>();  // the previous chunk's stores have read the buffer
    __syncwarp();
    if (args.out32) {
      uint4* d = reinterpret_cast<uint4*>(s32 + lane * 128);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        d[j ^ (lane & 7)] = make_uint4(__float_as_uint(x[4 * j]), __float_as_uint(x[4 * j + 1]),
                                       __float_as_uint(x[4 * j + 2]), __float_as_uint(x[4 * j + 3]));
    }
    if (args.out_hi) {
      uint32_t hi[16], lo[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
        hi[j] = *reinterpret_cast<const uint32_t*>(&h);
        const float2 hf = __bfloat1622float2(h);
        lo[j] = pack_bf16x2(x[2 * j] - hf.x, x[2 * j + 1] - hf.y);
      }
      uint4* dh = reinterpret_cast<uint4*>(shi + lane * 64);
      uint4* dl = reinterpret_cast<uint4*>(slo + lane * 64);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        dh[j ^ ((lane >> 1) & 3)] = make_uint4(hi[4 * j], hi[4 * j + 1], hi[4 * j + 2], hi[4 * j + 3]);
        if (args.out_lo) dl[j ^ ((lane >> 1) & 3)] = make_uint4(lo[4 * j], lo[4 * j + 1], lo[4 * j + 2], lo[4 * j + 3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (args.out32) tma_store_3d(es.o32, s32, ocol, orow, es.split);
      if (args.out_hi) tma_store_2d(es.ohi, shi, ocol, orow);
      if (args.out_hi && args.out_lo) tma_store_2d(es.olo, slo, ocol, orow);
      bulk_commit();
    }
  };
  // the 32 values of accumulator chunk c (all epilogues but SwiGLU)
  auto values = [&](const int c, const uint32_t (&v)[32], float (&x)[32]) {
    const int col = n0 + c * 32;
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(v[j]) * r;
    if (EPI == EPI_RESID) {
      if (row_ok) {
        const float4* rp = reinterpret_cast<const float4*>(args.resid32 + gm * args.ldr + col);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 t = kPre ? pre[(c * 8 + i) % EpiPre<BN, EPI>::kN] : rp[i];
          x[4 * i] += t.x;
          x[4 * i + 1] += t.y;
          x[4 * i + 2] += t.z;
          x[4 * i + 3] += t.w;
        }
      }
    } else if (EPI == EPI_SILU) {
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] = silu_f(x[j]);
    } else if (EPI == EPI_SWIGLU_TIED) {
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] = silu_f(x[j]) * x[j];
    }
  };
#pragma unroll (kPre ? BN / 64 : 1)
  for (int c = 0; c < BN / 32; c += 2) {
    uint32_t va[32], vb[32];
    tmem_ld_32x32b_x32(t_row + c * 32, va);
    tmem_ld_32x32b_x32(t_row + (c + 1) * 32, vb);
    tmem_ld_wait();
    if (EPI == EPI_SWIGLU) {  // 16 up and 16 gate columns per chunk: the pair gives 32 outputs
      float h[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        h[j] = silu_f(__uint_as_float(va[16 + j]) * r) * (__uint_as_float(va[j]) * r);
        h[16 + j] = silu_f(__uint_as_float(vb[16 + j]) * r) * (__uint_as_float(vb[j]) * r);
      }
      emit(h, (n0 + c * 32) / 2, es.orow);
    } else if (EPI == EPI_QABS) {  // head block j of the warp's example: rows b qabs_rows + j qabs_N + n
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int col = n0 + (c + h2) * 32;
        const int head = col / args.qabs_d;
        const int orow = (es.orow / args.qabs_N) * args.qabs_rows + head * args.qabs_N + es.orow % args.qabs_N;
        float x[32];
        values(c + h2, h2 ? vb : va, x);
        emit(x, col - head * args.qabs_d, orow);
      }
    } else {
      float x[32];
      values(c, va, x);
      emit(x, n0 + c * 32, es.orow);
      values(c + 1, vb, x);
      emit(x, n0 + (c + 1) * 32, es.orow);
    }
  }
}

// Instruction-descriptor bit selecting an MN-major A operand.
constexpr uint32_t kIdescAMnMajor = 1u << 15;

// SPLIT_B: B is a hi/lo pair too (single A source: tmA1 then holds B's lo half), and every k-step
// issues A_hi B_hi, A_lo B_hi and A_hi B_lo (the A_lo B_lo term is below 2^-16 of the product):
// the weight gradients of the token side, whose sums over rows cancel, need both operands at ~16 bits.
// With an exact bf16 A (SPLIT off) it issues A B_hi and A B_lo: the backward's recompute of the
// history-side projection multiplies the raw states by W diag(g) carried as a pair.
//
// KPS = 2: each stage carries two K blocks, loaded with 3-D tensor maps (the view {64 columns, rows,
// K / 64 blocks} of each K-major operand, box {64, rows, 2}), so a stage costs three copies instead of
// six. The K blocks of every tile, of A0 and of each split-K range are then even in number.
//
// TST: the epilogue writes through shared memory with tensor stores (maps tmO32, tmOhi, tmOlo over
// the fp32 output {columns, rows, split} and the bf16 hi and lo outputs, boxes of 32 x 32). The QABS
// row scatter takes it when a warp's 32 rows stay within one example (qabs_N a multiple of 32).
template <int BN, int EPI, bool ROWNORM, bool SPLIT, bool A_MN = false, bool B_MN = false, bool SPLIT_B = false,
          int KPS = 1, bool TST = false>
__global__ void __launch_bounds__(gemm_threads<ROWNORM>(), 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA0lo,
                   const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmA1lo,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmO32,
                   const __grid_constant__ CUtensorMap tmOhi, const __grid_constant__ CUtensorMap tmOlo,
                   const GemmArgs args) {
  using L = GemmSmem<BN, SPLIT, SPLIT_B, KPS, TST>;
  constexpr int STAGES = L::STAGES;
  constexpr uint32_t TMEM_COLS = 2 * BN;  // two accumulators: 128, 256 or 512 columns
  static_assert(!(ROWNORM && A_MN), "row statistics read K-major A rows");
  static_assert(KPS == 1 || (KPS == 2 && !A_MN && !B_MN && !SPLIT_B), "two-block stages: K-major operands");
  static_assert(STAGES >= 2, "pipeline depth");
  constexpr uint32_t MN_BOX = 64 * 64 * 2;  // one MN-major box: 64 K rows x 64 elements
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: [A hi | A lo (SPLIT) | W]; then the epilogue staging (TST); row factors [2][128]; barriers
  uint8_t* stg = smem + STAGES * L::STAGE_BYTES;
  float* rbuf = reinterpret_cast<float*>(stg + L::STG_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(rbuf + 2 * 128);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;  // [2] accumulator ready (MMA commit)
  uint64_t* tempty = tfull + 2;      // [2] accumulator drained (4 epilogue warps)
  uint64_t* nfull = tempty + 2;      // [2] row factors ready (4 statistic warps)
  uint64_t* edone = nfull + 2;       // [2] row factors consumed (4 epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(edone + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = args.kb0 + args.kb1;
  const int nsplit = args.ksplit > 1 ? args.ksplit : 1;
  const int tiles_mn = args.num_tiles / nsplit;
  // tile -> (split, m0, n0) and the split's K blocks [kb_lo, kb_hi)
  auto tile_of = [&](int tile, int& m0, int& n0, int& kb_lo, int& kb_hi, int& split) {
    split = tile / tiles_mn;
    const int tmn = tile - split * tiles_mn;
    m0 = (tmn / args.tiles_n) * L::BM;
    n0 = (tmn % args.tiles_n) * BN;
    kb_lo = nsplit > 1 ? split * args.kb_split : 0;
    kb_hi = nsplit > 1 ? min(KB, kb_lo + args.kb_split) : KB;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + (ROWNORM ? 4 : 0));
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
      mbar_init(&nfull[i], 4);
      mbar_init(&edone[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB);
    if (SPLIT) tma_prefetch_desc(&tmA0lo);
    if (SPLIT_B) tma_prefetch_desc(&tmA1);
    if (args.kb1 > 0) {
      tma_prefetch_desc(&tmA1);
      if (SPLIT) tma_prefetch_desc(&tmA1lo);
    }
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
    // ---------------- TMA producer: every K block of every tile of this CTA ----------------
    if (lane == 0) {
      auto load_b = [&](uint8_t* st, int kb, int n0, uint64_t* bar) {
        if (B_MN) {
#pragma unroll
          for (int i = 0; i < BN / 64; ++i) {
            tma_load_2d(st + L::A_ALL + i * MN_BOX, &tmB, n0 + 64 * i, kb * L::BK, bar);
            if (SPLIT_B) tma_load_2d(st + L::A_ALL + L::B_BYTES + i * MN_BOX, &tmA1, n0 + 64 * i, kb * L::BK, bar);
          }
        } else if (KPS == 1) {
          tma_load_2d(st + L::A_ALL, &tmB, kb * L::BK, n0, bar);
          if (SPLIT_B) tma_load_2d(st + L::A_ALL + L::B_BYTES, &tmA1, kb * L::BK, n0, bar);
        } else {
          tma_load_3d(st + L::A_ALL, &tmB, 0, n0, kb, bar);
        }
      };
      int kg = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < args.num_tiles && !stop; tile += gridDim.x) {
        int m0, n0, kb_lo, kb_hi, split;
        tile_of(tile, m0, n0, kb_lo, kb_hi, split);
        for (int kb = kb_lo; kb < kb_hi; kb += KPS, ++kg) {
          const int s = kg % STAGES, u = kg / STAGES;
          if (kg >= STAGES && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag)) {
            stop = true;
            break;
          }
          uint8_t* st = smem + s * L::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], L::STAGE_BYTES);
          const bool first = kb < args.kb0;
          int kc = (first ? kb : kb - args.kb0) * L::BK, ma = m0;
          if (args.head_tiles > 0) {
            const int head = (tile % args.tiles_n) / args.head_tiles;
            kc += head * args.a_kb_step * L::BK;
            ma += (int)(head * args.a_row_step);
          }
          if (A_MN) {
#pragma unroll
            for (int i = 0; i < L::BM / 64; ++i) {
              tma_load_2d(st + i * MN_BOX, first ? &tmA0 : &tmA1, ma + 64 * i, kc, &full[s]);
              if (SPLIT) tma_load_2d(st + L::A_BYTES + i * MN_BOX, first ? &tmA0lo : &tmA1lo, ma + 64 * i, kc, &full[s]);
            }
          } else if (SPLIT && args.a_planes) {
            if (KPS == 1) tma_load_3d(st, first ? &tmA0 : &tmA1, kc, ma, 0, &full[s]);
            else tma_load_4d(st, first ? &tmA0 : &tmA1, 0, ma, kc / L::BK, 0, &full[s]);
          } else if (KPS == 1) {
            tma_load_2d(st, first ? &tmA0 : &tmA1, kc, ma, &full[s]);
            if (SPLIT) tma_load_2d(st + L::A_BYTES, first ? &tmA0lo : &tmA1lo, kc, ma, &full[s]);
          } else {
            tma_load_3d(st, first ? &tmA0 : &tmA1, 0, ma, kc / L::BK, &full[s]);
            if (SPLIT) tma_load_3d(st + KPS * L::A_BYTES, first ? &tmA0lo : &tmA1lo, 0, ma, kc / L::BK, &full[s]);
          }
          load_b(st, kb, n0, &full[s]);
        }
      }
      if (*abort_flag) {
        // Unwinding after a timeout: let the copies this thread started land before the CTA exits.
        volatile int quiet = 0;
        for (int k = (kg > STAGES ? kg - STAGES : 0); k < kg; ++k)
          mbar_wait(&full[k % STAGES], (k / STAGES) & 1, &quiet);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: tile i accumulates into buffer i % 2 ----------------
    if (lane == 0) {
      constexpr uint32_t idesc =
          idesc_bf16_f32(128, BN) | (A_MN ? kIdescAMnMajor : 0u) | (B_MN ? kIdescBMnMajor : 0u);
      int kg = 0, it = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < args.num_tiles && !stop; tile += gridDim.x, ++it) {
        const int acc = it & 1, ua = it >> 1;
        if (it >= 2 && !mbar_wait(&tempty[acc], (ua - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        int m0, n0, kb_lo, kb_hi, split;
        tile_of(tile, m0, n0, kb_lo, kb_hi, split);
        for (int kb = kb_lo; kb < kb_hi; kb += KPS, ++kg) {
          const int s = kg % STAGES, u = kg / STAGES;
          if (!mbar_wait(&full[s], u & 1, abort_flag)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t st_base = smem_u32(smem + s * L::STAGE_BYTES);
#pragma unroll
          for (int j = 0; j < KPS; ++j) {
            const uint32_t a_base = st_base + j * L::A_BYTES;
            const uint32_t b_base = st_base + L::A_ALL + j * L::B_BYTES;
#pragma unroll
            for (int kk = 0; kk < L::BK / 16; ++kk) {
              // MN-major: 16 K rows of 128 bytes per k-step; 64-element MN groups one box apart
              auto bd = [&](uint32_t base) {
                return B_MN ? sdesc_mn_sw128(base + kk * 2048, MN_BOX, 1024) : sdesc_k_sw128(base + kk * 32);
              };
              auto ad = [&](uint32_t base) {
                return A_MN ? sdesc_mn_sw128(base + kk * 2048, MN_BOX, 1024) : sdesc_k_sw128(base + kk * 32);
              };
              const uint64_t bdesc = bd(b_base), adesc = ad(a_base);
              umma_f16(d_tmem, adesc, bdesc, idesc, (kb > kb_lo || j > 0 || kk > 0) ? 1u : 0u);
              if (SPLIT) umma_f16(d_tmem, ad(a_base + KPS * L::A_BYTES), bdesc, idesc, 1u);
              if (SPLIT_B) umma_f16(d_tmem, adesc, bd(b_base + KPS * L::B_BYTES), idesc, 1u);
            }
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&tfull[acc]);  // also on abort: arrives once all issued MMAs are done
      }
    }
  } else if (warp >= 6) {
    // ---------------- row statistics (ROWNORM): sum of squares of each A row ----------------
    if (ROWNORM) {
      const int row = (warp & 3) * 32 + lane;
      int kg = 0, it = 0;
      for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1, ua = it >> 1;
        float ss = 0.f;
        bool ok = true;
        for (int kb = 0; kb < KB; kb += KPS, ++kg) {
          const int s = kg % STAGES, u = kg / STAGES;
          if (!mbar_wait(&full[s], u & 1, abort_flag)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int jb = 0; jb < KPS; ++jb) {
            if (kb + jb < args.kb0) {
              // The row's 128 bytes are contiguous; the 128-byte swizzle stores its logical 16-byte
              // chunk c at position c ^ (row % 8) (identically in the hi and lo tiles). Summing in
              // logical order keeps the row factor independent of the row's position in the tile.
              const uint8_t* st = smem + s * L::STAGE_BYTES + jb * L::A_BYTES + row * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const int pc = c ^ (row & 7);
                float f[8];
                bf16x8_to_f32(reinterpret_cast<const uint4*>(st)[pc], f);
                if (SPLIT) {
                  float fl[8];
                  bf16x8_to_f32(reinterpret_cast<const uint4*>(st + KPS * L::A_BYTES)[pc], fl);
#pragma unroll
                  for (int j = 0; j < 8; ++j) f[j] += fl[j];
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) ss = fmaf(f[j], f[j], ss);
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
    }
  } else {
    // ---------------- epilogue (warps 2..5): thread i of quadrant q owns row 32q + i ----------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    float4 pre[EpiPre<BN, EPI>::kN];
    int it = 0;
    for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1, ua = it >> 1;
      int m0, n0, kb_lo, kb_hi, split;
      tile_of(tile, m0, n0, kb_lo, kb_hi, split);
      const long long gm = (long long)m0 + row;
      const bool row_ok = gm < args.M;
      epi_load_resid<BN, EPI>(args, gm, row_ok, n0, pre);
      if (!mbar_wait(&tfull[acc], ua & 1, abort_flag)) break;
      if (ROWNORM && !mbar_wait(&nfull[acc], ua & 1, abort_flag)) break;
      tc_fence_after();
      const float r = ROWNORM ? rbuf[acc * 128 + row] : 1.0f;
      if (ROWNORM && args.rows_r && n0 == 0 && row_ok) args.rows_r[gm] = r;
      if constexpr (TST) {
        const int orow = m0 + q * 32;
        const EpiStage es{stg + (warp - 2) * 8192, &tmO32, &tmOhi, &tmOlo, orow, nsplit > 1 ? split : 0, lane};
        epi_tile_tma<BN, EPI>(args, tmem_base + acc * BN + ((uint32_t)(q * 32) << 16), r, gm, row_ok, n0, pre, es);
      } else {
        epi_tile<BN, EPI>(args, tmem_base + acc * BN + ((uint32_t)(q * 32) << 16), r, gm, row_ok, n0, pre,
                          nsplit > 1 ? split * args.split_stride : 0ll);
      }
      // this accumulator buffer and its row factors may be reused
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[acc]);
        mbar_arrive(&edone[acc]);
      }
    }
    if (TST && lane == 0) bulk_wait<0>();  // this warp's tensor stores are complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Residual-stream tensor from a bf16 input: x32 = x, lo = 0 (x itself serves as hi).
__global__ void pair_from_bf16_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ x32,
                                      __nv_bfloat16* __restrict__ lo, long long n) {
  pdl_wait();
  pdl_trigger();
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    if (x32) x32[i] = __bfloat162float(x[i]);
    if (lo) lo[i] = __float2bfloat16_rn(0.f);
  }
}

// The same, 8 values per thread and step (x, x32 and lo 16-byte aligned); the last n % 8 values by
// the first threads.
__global__ void pair_from_bf16_8_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ x32,
                                        __nv_bfloat16* __restrict__ lo, long long n) {
  pdl_wait();
  pdl_trigger();
  const long long n8 = n >> 3, t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long long i = t0; i < n8; i += (long long)gridDim.x * blockDim.x) {
    if (x32) {
      float f[8];
      bf16x8_to_f32(reinterpret_cast<const uint4*>(x)[i], f);
      float4* d = reinterpret_cast<float4*>(x32 + 8 * i);
      d[0] = make_float4(f[0], f[1], f[2], f[3]);
      d[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    if (lo) reinterpret_cast<uint4*>(lo)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (t0 < n - 8 * n8) {
    const long long i = 8 * n8 + t0;
    if (x32) x32[i] = __bfloat162float(x[i]);
    if (lo) lo[i] = __float2bfloat16_rn(0.f);
  }
}

}  // namespace whale
