// backward.cuh — the element-wise, row-wise and reduction kernels of the fusion layer's backward
// pass (the vector-Jacobian product of the forward for an upstream gradient dY = dLoss/dH_f), and
// the SIMT kernels of its fp32 (correctness) mode. The dense contractions of the bf16 mode run on
// the tcgen05 GEMM (gemm_tc.cuh, MN-major operands and split-K) and the attention's backward on
// attention_bwd.cuh.
//
// The derivatives are the forward's steps differentiated one by one (gist.science technical summary
// of WHALE, section 2.2 "Efficiency Optimizations", Asymmetric Backward Variants, names the
// backward's schedules; the formulas follow from the forward of section 2.1):
//   RMSNorm  n = r x g, r = (mean(x^2) + eps)^-1/2:  dx = r (dn g) - x r^3 / d * sum(dn g x),
//                                                    dg = sum over rows of dn x r
//   SiLU     silu'(z) = s(z) (1 + z (1 - s(z))), s = sigmoid
//   SwiGLU   m = silu(gate) up:  dup = dm silu(gate), dgate = dm up silu'(gate)
//            (tied gate, up = gate = u: du = dup + dgate)
#pragma once

#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace whale {

__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + __expf(-z)); }
__device__ __forceinline__ float silu_grad_f(float z) {
  const float s = sigmoid_f(z);
  return s * (1.0f + z * (1.0f - s));
}

// The element-wise kernels below take 8 consecutive values per thread and step (32-byte fp32 and
// 16-byte bf16 accesses), so that enough bytes are in flight per SM to approach the HBM bandwidth.
__device__ __forceinline__ void ld8f(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void st8f(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
// bf16 hi = bf16(v) and lo = bf16(v - hi) of 8 values, each as one 16-byte word
__device__ __forceinline__ void split8(const float (&v)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    h[j] = *reinterpret_cast<const uint32_t*>(&hh);
    const float2 hf = __bfloat1622float2(hh);
    l[j] = pack_bf16x2(v[2 * j] - hf.x, v[2 * j + 1] - hf.y);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}
// Writes 8 values at element offset idx of any of: fp32, bf16 hi, bf16 lo (each may be null).
__device__ __forceinline__ void put8(long long idx, const float (&v)[8], float* f32, __nv_bfloat16* hi,
                                     __nv_bfloat16* lo) {
  if (f32) st8f(f32 + idx, v);
  if (hi) {
    uint4 h, l;
    split8(v, h, l);
    *reinterpret_cast<uint4*>(hi + idx) = h;
    if (lo) *reinterpret_cast<uint4*>(lo + idx) = l;
  }
}
// i / m for the index range of one launch (32-bit division when the range allows)
__device__ __forceinline__ long long div_idx(long long i, long long m, long long n) {
  return n < (1ll << 31) ? (long long)((unsigned)i / (unsigned)m) : i / m;
}

// x (fp32, row stride ldx) -> bf16 hi = bf16(x) and lo = bf16(x - hi) (lo may be null), row stride ldo.
// cols, ldx and ldo multiples of 8.
__global__ void split_pair_kernel(const float* __restrict__ x, long long ldx, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo, long long ldo, long long rows, int cols) {
  pdl_wait();
  pdl_trigger();
  const int cg = cols >> 3;
  const long long n = rows * cg;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = div_idx(i, cg, n);
    const int c = (int)(i - r * cg) * 8;
    float v[8];
    ld8f(x + r * ldx + c, v);
    put8(r * ldo + c, v, nullptr, hi, lo);
  }
}

// G = SiLU(Z); Z fp32 [n]; outputs (each may be null): fp32, and a bf16 pair (hi, lo).
__global__ void silu_pair_kernel(const float* __restrict__ z, float* __restrict__ g32, __nv_bfloat16* __restrict__ hi,
                                 __nv_bfloat16* __restrict__ lo, long long n) {
  pdl_wait();
  pdl_trigger();
  const long long n8 = n >> 3, t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long long i = t0; i < n8; i += (long long)gridDim.x * blockDim.x) {
    float v[8];
    ld8f(z + 8 * i, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] *= sigmoid_f(v[j]);
    put8(8 * i, v, g32, hi, lo);
  }
  if (t0 < n - 8 * n8) {  // the last n % 8 values
    const long long i = 8 * n8 + t0;
    const float v = z[i] * sigmoid_f(z[i]);
    if (g32) g32[i] = v;
    if (hi) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      hi[i] = h;
      if (lo) lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
  }
}

// dZ = dH * silu'(Z) as fp32 (optional) and a bf16 pair (optional).
__global__ void silu_bwd_kernel(const float* __restrict__ dh, const float* __restrict__ z, float* __restrict__ dz32,
                                __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo, long long n) {
  pdl_wait();
  pdl_trigger();
  const long long n8 = n >> 3, t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long long i = t0; i < n8; i += (long long)gridDim.x * blockDim.x) {
    float g[8], zz[8];
    ld8f(dh + 8 * i, g);
    ld8f(z + 8 * i, zz);
#pragma unroll
    for (int j = 0; j < 8; ++j) g[j] *= silu_grad_f(zz[j]);
    put8(8 * i, g, dz32, hi, lo);
  }
  if (t0 < n - 8 * n8) {
    const long long i = 8 * n8 + t0;
    const float v = dh[i] * silu_grad_f(z[i]);
    if (dz32) dz32[i] = v;
    if (hi) {
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      hi[i] = h;
      if (lo) lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
  }
}

// SwiGLU backward. ug: fp32 [rows, ugw] pre-activations ([up | gate], or u alone with a tied gate);
// dm: fp32 [rows, H] gradient of m = SiLU(gate) * up. Outputs (each may be null): m as bf16 [rows, H],
// and dug = [dup | dgate] (or du) as fp32 and as a bf16 pair, [rows, ugw]; m also as fp32 (m32) and
// as the bf16 residue of m_out (m_lo). H a multiple of 8.
__global__ void swiglu_bwd_kernel(const float* __restrict__ ug, const float* __restrict__ dm, long long rows, int H,
                                  int tied, __nv_bfloat16* __restrict__ m_out, __nv_bfloat16* __restrict__ m_lo,
                                  float* __restrict__ m32,
                                  float* __restrict__ dug32, __nv_bfloat16* __restrict__ dug_hi,
                                  __nv_bfloat16* __restrict__ dug_lo) {
  pdl_wait();
  pdl_trigger();
  const int ugw = tied ? H : 2 * H;
  const int hg = H >> 3;
  const long long n = rows * hg;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = div_idx(i, hg, n);
    const int c = (int)(i - r * hg) * 8;
    float up[8], gate[8], g[8];
    ld8f(ug + r * ugw + c, up);
    if (tied) {
#pragma unroll
      for (int j = 0; j < 8; ++j) gate[j] = up[j];
    } else {
      ld8f(ug + r * ugw + H + c, gate);
    }
    ld8f(dm + r * H + c, g);
    float mv[8], dup[8], dgate[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float sg0 = sigmoid_f(gate[j]);
      const float sg = gate[j] * sg0;  // silu(gate)
      mv[j] = sg * up[j];
      dup[j] = g[j] * sg;
      dgate[j] = g[j] * up[j] * sg0 * (1.0f + gate[j] * (1.0f - sg0));
    }
    put8(r * H + c, mv, m32, m_out, m_lo);
    if (tied) {
#pragma unroll
      for (int j = 0; j < 8; ++j) dup[j] += dgate[j];
      put8(r * ugw + c, dup, dug32, dug_hi, dug_lo);
    } else {
      put8(r * ugw + c, dup, dug32, dug_hi, dug_lo);
      put8(r * ugw + H + c, dgate, dug32, dug_hi, dug_lo);
    }
  }
}

// 8 consecutive values of a row as fp32 (16-byte loads: one of bf16, two of fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  bf16x8_to_f32(*reinterpret_cast<const uint4*>(p), v);
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
// bf16 of 8 values (hi) and, if lo is set, the bf16 of their rounding residues
__device__ __forceinline__ void store8_pair(__nv_bfloat16* hi, __nv_bfloat16* lo, const float (&v)[8]) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    h[j] = *reinterpret_cast<const uint32_t*>(&hh);
    const float2 hf = __bfloat1622float2(hh);
    l[j] = pack_bf16x2(v[2 * j] - hf.x, v[2 * j + 1] - hf.y);
  }
  *reinterpret_cast<uint4*>(hi) = make_uint4(h[0], h[1], h[2], h[3]);
  if (lo) *reinterpret_cast<uint4*>(lo) = make_uint4(l[0], l[1], l[2], l[3]);
}

// RMSNorm backward, one warp per row (d a multiple of 8, at most 1024; lane l takes the 8-column
// chunks l, l + 32, ...: 16-byte loads and stores), for n = r x g:
//   dx = r (dn g) - x (r^3 / d) sum_c (dn g x)_c  [+ resid1 + resid2]
// x: bf16 or fp32 [rows, d] (row stride d); dn fp32 [rows, d]; outputs (each may be null): dx as fp32,
// as bf16 (dx_hi, with its residue dx_lo), n = r x g as a bf16 pair (n_out, n_lo) or fp32 (n32).
// colp [gridDim.x, d]: this block's column sums of dn x r (the gain's gradient, summed over the
// block's rows; a second pass sums the blocks in order).
// PRE: dn is already scaled by the row factor (dn' = r dn, as the history side's backward forms it):
// dx = dn' g - x r^2/d sum(dn' g x) and the gain's column sums are of dn' x.
template <typename TX, int MAXCH, bool PRE = false>
__global__ void __launch_bounds__(256, MAXCH <= 2 ? 2 : 1) rms_bwd_kernel(const TX* __restrict__ x, const float* __restrict__ g,
                                                      const float* __restrict__ dn, long long rows, int d, float eps,
                                                      const float* __restrict__ resid1, long long ld1,
                                                      const float* __restrict__ resid2, long long ld2,
                                                      float* __restrict__ dx32, __nv_bfloat16* __restrict__ dx_hi,
                                                      __nv_bfloat16* __restrict__ dx_lo,
                                                      __nv_bfloat16* __restrict__ n_out,
                                                      __nv_bfloat16* __restrict__ n_lo, float* __restrict__ n32,
                                                      float* __restrict__ colp) {
  // MAXCH: 8-column chunks per lane (d <= 256 MAXCH); fewer registers for narrower rows, more blocks per SM
  __shared__ float red[8][256 * MAXCH];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = d >> 3;
  float cg[MAXCH][8];
#pragma unroll
  for (int i = 0; i < MAXCH; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) cg[i][j] = 0.f;
  // the gains of this lane's columns, once for all rows
  float gr[MAXCH][8];
#pragma unroll
  for (int i = 0; i < MAXCH; ++i) {
    const int c8 = lane + 32 * i;
    if (c8 < nch) load8(g + 8 * c8, gr[i]);
  }
  const long long per = (rows + gridDim.x - 1) / gridDim.x;
  const long long r0 = (long long)blockIdx.x * per, r1 = min(rows, r0 + per);
  for (long long r = r0 + warp; r < r1; r += 8) {
    float xv[MAXCH][8], dv[MAXCH][8], u[MAXCH][8];
    float ss = 0.f, sux = 0.f;
    // the row of x and of dn in one round of loads
#pragma unroll
    for (int i = 0; i < MAXCH; ++i) {
      const int c8 = lane + 32 * i;
      if (c8 < nch) {
        load8(x + r * d + 8 * c8, xv[i]);
        load8(dn + r * d + 8 * c8, dv[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < MAXCH; ++i) {
      const int c8 = lane + 32 * i;
      if (c8 < nch) {
#pragma unroll
        for (int j = 0; j < 8; ++j) ss = fmaf(xv[i][j], xv[i][j], ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rr = rsqrtf(ss / (float)d + eps);
#pragma unroll
    for (int i = 0; i < MAXCH; ++i) {
      const int c8 = lane + 32 * i;
      if (c8 < nch) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          u[i][j] = dv[i][j] * gr[i][j];
          sux = fmaf(u[i][j], xv[i][j], sux);
          cg[i][j] = fmaf(dv[i][j], PRE ? xv[i][j] : xv[i][j] * rr, cg[i][j]);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sux += __shfl_xor_sync(0xffffffffu, sux, o);
    const float k = (PRE ? rr * rr : rr * rr * rr) / (float)d * sux;
    const float ru = PRE ? 1.0f : rr;
#pragma unroll
    for (int i = 0; i < MAXCH; ++i) {
      const int c8 = lane + 32 * i;
      if (c8 < nch) {
        const int c = 8 * c8;
        float v[8], r1v[8], r2v[8];
        if (resid1) load8(resid1 + r * ld1 + c, r1v);
        if (resid2) load8(resid2 + r * ld2 + c, r2v);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v[j] = ru * u[i][j] - xv[i][j] * k;
          if (resid1) v[j] += r1v[j];
          if (resid2) v[j] += r2v[j];
        }
        if (dx32) store8(dx32 + r * d + c, v);
        if (dx_hi) store8_pair(dx_hi + r * d + c, dx_lo ? dx_lo + r * d + c : nullptr, v);
        if (n_out || n32) {
          float nv[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) nv[j] = xv[i][j] * rr * gr[i][j];
          if (n_out) store8_pair(n_out + r * d + c, n_lo ? n_lo + r * d + c : nullptr, nv);
          if (n32) store8(n32 + r * d + c, nv);
        }
      }
    }
  }
  if (colp) {
#pragma unroll
    for (int i = 0; i < MAXCH; ++i) {
      const int c8 = lane + 32 * i;
      if (c8 < nch)
#pragma unroll
        for (int j = 0; j < 8; ++j) red[warp][8 * c8 + j] = cg[i][j];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) sum += red[w][c];
      colp[(long long)blockIdx.x * d + c] = sum;
    }
  }
}

// n = r x g as a bf16 pair (n_out, n_lo) and/or fp32 (n32): the normalised rows the weight gradients
// contract with, one warp per row (8-column chunks per lane, as above).
template <typename TX>
__global__ void __launch_bounds__(256) rms_rows_kernel(const TX* __restrict__ x, const float* __restrict__ g,
                                                       long long rows, int d, float eps,
                                                       __nv_bfloat16* __restrict__ n_out,
                                                       __nv_bfloat16* __restrict__ n_lo, float* __restrict__ n32) {
  constexpr int MAXCH = 4;  // 8-column chunks per lane (d <= 1024)
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int nch = d >> 3;
  const long long warps = (long long)gridDim.x * 8;
  for (long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += warps) {
    float xv[MAXCH][8];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < MAXCH; ++i) {
      const int c8 = lane + 32 * i;
      if (c8 < nch) {
        load8(x + r * d + 8 * c8, xv[i]);
#pragma unroll
        for (int j = 0; j < 8; ++j) ss = fmaf(xv[i][j], xv[i][j], ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rr = rsqrtf(ss / (float)d + eps);
#pragma unroll
    for (int i = 0; i < MAXCH; ++i) {
      const int c8 = lane + 32 * i;
      if (c8 < nch) {
        const int c = 8 * c8;
        float gv[8], nv[8];
        load8(g + c, gv);
#pragma unroll
        for (int j = 0; j < 8; ++j) nv[j] = xv[i][j] * rr * gv[j];
        if (n_out) store8_pair(n_out + r * d + c, n_lo ? n_lo + r * d + c : nullptr, nv);
        if (n32) store8(n32 + r * d + c, nv);
      }
    }
  }
}

// out[c] = sum_b part[b * n + c] over b = 0..nb-1, for n columns: a block per 32 columns, its eight
// warps summing row stripes b = w, w + 8, ... and then combined in warp order (deterministic).
__global__ void __launch_bounds__(256) col_sums_kernel(const float* __restrict__ part, int nb, int n,
                                                       float* __restrict__ out) {
  __shared__ float red[8][32];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (c < n)
    for (int b = warp; b < nb; b += 8) s += part[(long long)b * n + c];
  red[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && c < n) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w][lane];
    out[c] = t;
  }
}

// SwiGLU forward: m = SiLU(gate) * up from the pre-activations ug fp32 [rows, ugw] ([up | gate], or u
// alone with a tied gate), as a bf16 pair [rows, H].
__global__ void swiglu_pair_kernel(const float* __restrict__ ug, long long rows, int H, int tied,
                                   __nv_bfloat16* __restrict__ m_hi, __nv_bfloat16* __restrict__ m_lo) {
  pdl_wait();
  pdl_trigger();
  const int ugw = tied ? H : 2 * H;
  const long long n = rows * H;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / H;
    const int c = (int)(i - r * H);
    const float up = ug[r * ugw + c];
    const float gate = tied ? up : ug[r * ugw + H + c];
    const float v = gate * sigmoid_f(gate) * up;
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    m_hi[i] = h;
    m_lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// out[r, c] (row stride ldo) = sum_b part[b][r][c] over b = 0..nb-1 in order (deterministic);
// part holds nb dense [rows, cols] blocks. sum_partials4_kernel: the same four columns at a time
// (cols and ldo multiples of 4, out 16-byte aligned), the same sums.
__global__ void sum_partials4_kernel(const float* __restrict__ part, int nb, long long rows, int cols,
                                     float* __restrict__ out, long long ldo) {
  pdl_wait();
  pdl_trigger();
  const int c4 = cols >> 2;
  const long long n4 = rows * c4, nn = rows * cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const long long r = div_idx(i, c4, n4);
    const int c = (int)(i - r * c4) * 4;
    const float* src = part + r * cols + c;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int b = 0; b < nb; ++b) {
      const float4 v = *reinterpret_cast<const float4*>(src + (long long)b * nn);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    *reinterpret_cast<float4*>(out + r * ldo + c) = s;
  }
}

__global__ void sum_partials_kernel(const float* __restrict__ part, int nb, long long rows, int cols,
                                    float* __restrict__ out, long long ldo) {
  pdl_wait();
  pdl_trigger();
  const long long n = rows * cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int b = 0; b < nb; ++b) s += part[(long long)b * n + i];
    const long long r = i / cols;
    out[r * ldo + (i - r * cols)] = s;
  }
}

// ---------------------------------------------------------------------------------------------
// fp32 (correctness) mode
// ---------------------------------------------------------------------------------------------
// C[m, n] = sum_k A[m sam + k sak] * B[k sbk + n sbn] (+ C if accumulate), fp32, any strides: 64 x 64
// tiles, 256 threads with 4 x 4 outputs each, K in steps of 16 through shared memory.
__global__ void __launch_bounds__(256) gemm_strided_f32_kernel(const float* __restrict__ A, long long sam,
                                                               long long sak, const float* __restrict__ B,
                                                               long long sbk, long long sbn, float* __restrict__ C,
                                                               long long ldc, long long M, long long N, long long K,
                                                               int accumulate) {
  __shared__ float As[16][64 + 1];
  __shared__ float Bs[16][64 + 1];
  const long long m0 = (long long)blockIdx.y * 64, n0 = (long long)blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (long long k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kk = i / 64, mm = i % 64;
      const long long gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? A[gm * sam + gk * sak] : 0.f;
      const long long gn = n0 + mm;
      Bs[kk][mm] = (gn < N && gk < K) ? B[gk * sbk + gn * sbn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long gn = n0 + tx * 4 + j;
      if (gn >= N) continue;
      float* c = C + gm * ldc + gn;
      *c = accumulate ? *c + acc[i][j] : acc[i][j];
    }
  }
}

// fp32 attention backward, one block per (example, head): all of the example's queries stay in
// shared memory; each thread takes history rows in turn and writes their dK, dV rows itself (one
// block holds every query of the pair, so no reduction over queries is needed), while dQ collects
// in shared memory. Phase 1 recomputes each query's softmax statistics and delta = sum_t p_t dp_t
// (warp per query). kv rows: K in columns [head*DH, ...), V at v_col0 + head*DH; dkv the same
// layout (shared K = V: dK + dV in the K columns). Needs N * (3 DH + 3) floats of shared memory.
template <int DH>
__global__ void __launch_bounds__(256) attn_bwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ kv,
                                                           int kvw, int v_col0, const float* __restrict__ da,
                                                           long long ld_da, const int* __restrict__ offsets,
                                                           long long total_L, int N,
                                                           int d, int n_heads, float scale, float* __restrict__ dq,
                                                           float* __restrict__ dkv, int shared_kv) {
  extern __shared__ float sm[];
  float* qs = sm;                 // [N][DH]
  float* das = qs + N * DH;       // [N][DH]
  float* dqs = das + N * DH;      // [N][DH]
  float* mx = dqs + N * DH;       // [N]
  float* ls = mx + N;             // [N] sum of exp(s - mx)
  float* del = ls + N;            // [N]
  const int b = blockIdx.x, head = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long lo = offsets[b], hi = offsets[b + 1];
  lo = lo < 0 ? 0 : (lo > total_L ? total_L : lo);
  hi = hi < lo ? lo : (hi > total_L ? total_L : hi);
  const int hc = head * DH;
  for (int i = threadIdx.x; i < N * DH; i += blockDim.x) {
    const int n = i / DH, c = i % DH;
    qs[i] = q[((long long)b * N + n) * d + hc + c];
    das[i] = da[((long long)b * N + n) * ld_da + hc + c];
    dqs[i] = 0.f;
  }
  __syncthreads();
  const float* kcol = kv + hc;
  const float* vcol = kv + v_col0 + hc;
  // phase 1: statistics and delta, one warp per query
  for (int n = warp; n < N; n += 8) {
    float m = -INFINITY, l = 0.f;
    for (long long t = lo + lane; t < hi; t += 32) {
      float s = 0.f;
      for (int c = 0; c < DH; ++c) s = fmaf(qs[n * DH + c], kcol[t * kvw + c], s);
      s *= scale;
      const float mn = fmaxf(m, s);
      l = l * __expf(m - mn) + __expf(s - mn);
      m = mn;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
      const float mn = fmaxf(m, m2);
      l = (m == -INFINITY ? 0.f : l * __expf(m - mn)) + (m2 == -INFINITY ? 0.f : l2 * __expf(m2 - mn));
      m = mn;
    }
    float dl = 0.f;
    for (long long t = lo + lane; t < hi; t += 32) {
      float s = 0.f, dp = 0.f;
      for (int c = 0; c < DH; ++c) {
        s = fmaf(qs[n * DH + c], kcol[t * kvw + c], s);
        dp = fmaf(das[n * DH + c], vcol[t * kvw + c], dp);
      }
      dl += __expf(s * scale - m) / l * dp;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
    if (lane == 0) {
      mx[n] = m;
      ls[n] = l;
      del[n] = dl;
    }
  }
  __syncthreads();
  // phase 2: one history row per thread
  for (long long t = lo + threadIdx.x; t < hi; t += blockDim.x) {
    float kr[DH], vr[DH], dk[DH], dv[DH];
#pragma unroll
    for (int c = 0; c < DH; ++c) {
      kr[c] = kcol[t * kvw + c];
      vr[c] = vcol[t * kvw + c];
      dk[c] = 0.f;
      dv[c] = 0.f;
    }
    for (int n = 0; n < N; ++n) {
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < DH; ++c) {
        s = fmaf(qs[n * DH + c], kr[c], s);
        dp = fmaf(das[n * DH + c], vr[c], dp);
      }
      const float p = __expf(s * scale - mx[n]) / ls[n];
      const float ds = p * (dp - del[n]);
#pragma unroll
      for (int c = 0; c < DH; ++c) {
        dv[c] = fmaf(p, das[n * DH + c], dv[c]);
        dk[c] = fmaf(ds * scale, qs[n * DH + c], dk[c]);
        atomicAdd(&dqs[n * DH + c], ds * scale * kr[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < DH; ++c) {
      if (shared_kv) {
        dkv[t * kvw + hc + c] = dk[c] + dv[c];
      } else {
        dkv[t * kvw + hc + c] = dk[c];
        dkv[t * kvw + v_col0 + hc + c] = dv[c];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < N * DH; i += blockDim.x) {
    const int n = i / DH, c = i % DH;
    dq[((long long)b * N + n) * d + hc + c] = dqs[i];
  }
}

// hi/lo pair of W diag(g): w [rows, cols] bf16, g [cols] fp32 (the history-side projection weights
// with the states' RMSNorm gain, for the backward's recompute).
__global__ void scale_cols_pair_kernel(const __nv_bfloat16* __restrict__ w, const float* __restrict__ g,
                                       long long rows, int cols, __nv_bfloat16* __restrict__ hi,
                                       __nv_bfloat16* __restrict__ lo) {
  pdl_wait();
  pdl_trigger();
  const long long n = rows * cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = __bfloat162float(w[i]) * g[i % cols];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// Rows [offsets[B], total_L) of a history slab belong to no example, so their K|V gradient is zero;
// the attention backward writes the examples' rows only. This clears the others in x and, if given,
// x_lo (each [total_L, width] row-major). Nothing is written when the examples cover the slab.
template <typename T>
__global__ void zero_tail_rows_kernel(const int* __restrict__ offsets, int B, long long total_L, int width,
                                      T* __restrict__ x, T* __restrict__ x_lo) {
  pdl_wait();
  pdl_trigger();
  long long r0 = offsets[B];
  r0 = r0 < 0 ? 0 : (r0 > total_L ? total_L : r0);
  const long long n = (total_L - r0) * width;
  T* p = x + r0 * width;
  T* q = x_lo ? x_lo + r0 * width : nullptr;
  const T zero = T(0.0f);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    p[i] = zero;
    if (q) q[i] = zero;
  }
}

// c[r, col] *= g[col] for a row-major fp32 [rows, cols] matrix (row stride ld).
__global__ void scale_cols_kernel(float* __restrict__ c, long long ld, const float* __restrict__ g, long long rows,
                                  int cols) {
  pdl_wait();
  pdl_trigger();
  const long long n = rows * cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / cols;
    const int col = (int)(i - r * cols);
    c[r * ld + col] *= g[col];
  }
}

}  // namespace whale
