// fp32_path.cuh — fp32 SIMT kernels for the fp32 storage mode (correctness mode, 1e-4
// tolerance). tcgen05 has no true-fp32 MMA kind, so this path uses FFMA; it is not the
// roofline path. RMSNorm is applied while loading A tiles (row factor r and gain g), so
// no normalised copy of the input is written.
#pragma once

#include "ptx.cuh"

namespace whale {

// r[row] = 1 / sqrt(mean(x[row]^2) + eps); one warp per row.
__global__ void row_rms_f32(const float* __restrict__ x, long long ldx, long long rows, int d, float eps,
                            float* __restrict__ r) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  float ss = 0.f;
  for (int c = lane; c < d; c += 32) {
    const float v = x[row * ldx + c];
    ss = fmaf(v, v, ss);
  }
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) r[row] = rsqrtf(ss / (float)d + eps);
}

enum F32Epi : int { F32_NONE = 0, F32_SILU = 1, F32_RESID = 2 };

// C[M,N] = epi( [A0 | A1] W^T ), A0 optionally normalised on load: A0'[m,k] = A0[m,k] r[m] g[k].
// 64x64 output tile per 256-thread block, 4x4 per thread, K step 16.
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A0, long long lda0, int K0,
                                                       const float* __restrict__ A1, long long lda1, int K1,
                                                       const float* __restrict__ rnorm, const float* __restrict__ gnorm,
                                                       const float* __restrict__ W, float* __restrict__ C,
                                                       long long ldc, long long M, int N, int epi,
                                                       const float* __restrict__ R, long long ldr) {
  __shared__ float sa[16][64 + 1];
  __shared__ float sw[16][64 + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const long long m0 = (long long)blockIdx.y * 64;
  const int n0 = blockIdx.x * 64;
  const int K = K0 + K1;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kk = i % 16, mm = i / 16;
      const long long m = m0 + mm;
      const int k = k0 + kk;
      float v = 0.f;
      if (m < M && k < K) {
        if (k < K0) {
          v = A0[m * lda0 + k];
          if (rnorm) v *= rnorm[m] * gnorm[k];
        } else {
          v = A1[m * lda1 + (k - K0)];
        }
      }
      sa[kk][mm] = v;
      const int n = n0 + mm;
      sw[kk][mm] = (n < N && k < K) ? W[(long long)n * K + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float av[4], wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = sa[kk][ty * 4 + i];
        wv[i] = sw[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (epi == F32_SILU) v = v / (1.0f + expf(-v));
      if (epi == F32_RESID) v += R[m * ldr + n];
      C[m * ldc + n] = v;
    }
  }
}

// h[m, i] = SiLU(gate) * up with up = ug[m, i], gate = ug[m, H + i] (tied: gate = up).
__global__ void swiglu_f32_kernel(const float* __restrict__ ug, long long ldug, float* __restrict__ h, long long M,
                                  int H, int tied) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= M * H) return;
  const long long m = idx / H;
  const int i = (int)(idx % H);
  const float up = ug[m * ldug + i];
  const float gate = tied ? up : ug[m * ldug + H + i];
  h[idx] = gate / (1.0f + expf(-gate)) * up;
}

// Eq. (4) in fp32: one warp per (example, query, head); lanes split the history, each lane
// keeps its own online-softmax state, then the warp merges the 32 states.
template <int DH>
__global__ void attn_f32_kernel(const float* __restrict__ Q, const float* __restrict__ KV, int ldkv, int v_col0,
                                const int* __restrict__ offsets, float* __restrict__ A, int B, int N, int d,
                                int n_heads, long long total_L, float scale) {
  const long long wid = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (wid >= (long long)B * N * n_heads) return;
  const int lane = threadIdx.x & 31;
  const int head = (int)(wid % n_heads);
  const long long bn = wid / n_heads;
  const int b = (int)(bn / N);
  long long lo = offsets[b], hi = offsets[b + 1];
  lo = lo < 0 ? 0 : (lo > total_L ? total_L : lo);
  hi = hi < lo ? lo : (hi > total_L ? total_L : hi);
  float q[DH];
#pragma unroll
  for (int c = 0; c < DH; ++c) q[c] = Q[bn * d + head * DH + c];
  float m = -INFINITY, l = 0.f, o[DH];
#pragma unroll
  for (int c = 0; c < DH; ++c) o[c] = 0.f;
  for (long long t = lo + lane; t < hi; t += 32) {
    const float* kr = KV + t * ldkv + head * DH;
    const float* vr = KV + t * ldkv + v_col0 + head * DH;
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < DH; ++c) s = fmaf(q[c], kr[c], s);
    s *= scale;
    const float mn = fmaxf(m, s);
    const float corr = expf(m - mn), p = expf(s - mn);
    l = l * corr + p;
#pragma unroll
    for (int c = 0; c < DH; ++c) o[c] = o[c] * corr + p * vr[c];
    m = mn;
  }
  float mw = m;
  for (int off = 16; off; off >>= 1) mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, off));
  const float w = (m == -INFINITY) ? 0.f : expf(m - mw);
  l *= w;
  for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  float* arow = A + bn * d + head * DH;
#pragma unroll
  for (int c = 0; c < DH; ++c) {
    float v = o[c] * w;
    for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == (c & 31)) arow[c] = (hi > lo) ? v / l : 0.f;
  }
}

}  // namespace whale
