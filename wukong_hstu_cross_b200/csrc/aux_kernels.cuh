// aux_kernels.cuh — weight preparation for the bf16 path, the debug offset check and the self-test
// of the bounded device waits.
#pragma once

#include "ptx.cuh"

namespace whale {

// Prepared weight matrix: out[r, c] = bf16(W[src(r), c] * g[c]) (g may be null = ones).
// mode 0: src(r) = r.
// mode 1 (SwiGLU packing for the fused up|gate epilogue): rows in blocks of 32, block p holds
//         W_up rows 16p..16p+15 then W_gate rows 16p..16p+15, where W = [W_up ; W_gate] and
//         W_gate starts at row H.
// mode 2 (absorbed keys): W = W_K [d, d], out has rows = h*d (row j*d + n) and cols = d_head (H
//         holds d_head, `src_cols` holds d): out[j*d + n, k] = bf16(W[j*d_head + k, n] * g[n] * scale).
struct FoldJob {
  const __nv_bfloat16* w;
  const float* g;
  __nv_bfloat16* out;
  int rows, cols, mode, H, src_cols;
  float scale;
};
struct FoldJobs {
  FoldJob job[4];
  int n;
};

// One thread per 8 consecutive columns (16-byte loads and stores; cols % 8 == 0).
__global__ void fold_weights_kernel(const FoldJobs jobs) {
  pdl_wait();
  pdl_trigger();
  if ((int)blockIdx.y >= jobs.n) return;
  const FoldJob j = jobs.job[blockIdx.y];
  const int cols8 = j.cols >> 3;
  const int total8 = j.rows * cols8;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total8; idx += gridDim.x * blockDim.x) {
    const int r = idx / cols8, c8 = idx - r * cols8;
    if (j.mode == 2) {
      const int dsrc = j.src_cols, head = r / dsrc, n = r - head * dsrc;
      const float gn = (j.g ? j.g[n] : 1.f) * j.scale;
      uint4 ov;
      uint32_t* op = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const size_t k0 = (size_t)head * j.H + c8 * 8 + 2 * i;
        op[i] = pack_bf16x2(__bfloat162float(j.w[k0 * dsrc + n]) * gn, __bfloat162float(j.w[(k0 + 1) * dsrc + n]) * gn);
      }
      *reinterpret_cast<uint4*>(j.out + (size_t)idx * 8) = ov;
      continue;
    }
    int src = r;
    if (j.mode == 1) {
      const int p = r >> 5, w = r & 31;
      src = (w < 16) ? (16 * p + w) : (j.H + 16 * p + (w - 16));
    }
    const uint4 wv = *reinterpret_cast<const uint4*>(j.w + (size_t)src * j.cols + c8 * 8);
    const __nv_bfloat162* wh = reinterpret_cast<const __nv_bfloat162*>(&wv);
    float g[8];
    if (j.g) {
      const float4 g0 = *reinterpret_cast<const float4*>(j.g + c8 * 8);
      const float4 g1 = *reinterpret_cast<const float4*>(j.g + c8 * 8 + 4);
      g[0] = g0.x; g[1] = g0.y; g[2] = g0.z; g[3] = g0.w; g[4] = g1.x; g[5] = g1.y; g[6] = g1.z; g[7] = g1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) g[i] = 1.f;
    }
    uint4 ov;
    uint32_t* op = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(wh[i]);
      op[i] = pack_bf16x2(f.x * g[2 * i], f.y * g[2 * i + 1]);
    }
    *reinterpret_cast<uint4*>(j.out + (size_t)idx * 8) = ov;
  }
}

// Debug-mode validation of the jagged offsets against the host-side shape hint.
__global__ void check_offsets_kernel(const int* __restrict__ off, int B, int max_L, long long total_L) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b <= B; b += gridDim.x * blockDim.x) {
    bool bad = false;
    if (b == 0) bad = off[0] != 0;
    else {
      const long long L = (long long)off[b] - off[b - 1];
      bad = L < 0 || L > max_L;
    }
    if (b == B) bad = bad || (long long)off[B] > total_L;
    if (bad) atomicOr(&g_device_error, kErrOffsets);
  }
}

// Self-test of the bounded waits every pipeline here relies on (mbar_wait, wait_nonzero_gpu):
// thread 0 waits on an mbarrier that no thread arrives on, thread 32 on a word in global memory that
// no thread sets, each for at most limit_ns. Both waits give up, record kErrTimeout in
// g_device_error and return; the kernel then exits normally (nothing else is in flight).
__device__ int g_wait_test_flag;  // never written by any kernel: stays 0
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, limit_ns);
  if (threadIdx.x == 32) (void)wait_nonzero_gpu(&g_wait_test_flag, limit_ns);
  __syncthreads();
}

}  // namespace whale
