// aux_kernels.cuh — weight preparation for the bf16 path and the debug offset check.
#pragma once

#include "ptx.cuh"

namespace whale {

// Prepared weight matrix: out[r, c] = bf16(W[src(r), c] * g[c]) (g may be null = ones).
// mode 0: src(r) = r.
// mode 1 (SwiGLU packing for the fused up|gate epilogue): rows in blocks of 32, block p holds
//         W_up rows 16p..16p+15 then W_gate rows 16p..16p+15, where W = [W_up ; W_gate] and
//         W_gate starts at row H.
struct FoldJob {
  const __nv_bfloat16* w;
  const float* g;
  __nv_bfloat16* out;
  int rows, cols, mode, H;
};
struct FoldJobs {
  FoldJob job[3];
  int n;
};

__global__ void fold_weights_kernel(const FoldJobs jobs) {
  if ((int)blockIdx.y >= jobs.n) return;
  const FoldJob j = jobs.job[blockIdx.y];
  const long long total = (long long)j.rows * j.cols;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(idx / j.cols), c = (int)(idx % j.cols);
    int src = r;
    if (j.mode == 1) {
      const int p = r >> 5, w = r & 31;
      src = (w < 16) ? (16 * p + w) : (j.H + 16 * p + (w - 16));
    }
    float v = __bfloat162float(j.w[(long long)src * j.cols + c]);
    if (j.g) v *= j.g[c];
    j.out[idx] = __float2bfloat16_rn(v);
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

}  // namespace whale
