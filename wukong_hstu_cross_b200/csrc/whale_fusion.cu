// whale_fusion.cu — C ABI of the WHALE attention-fusion forward (see include/whale_fusion.h).
//
// Host side: argument checks, workspace layout, TMA descriptor encoding and the launch
// sequence of one layer (all on the caller's stream, no device->host sync):
//   bf16:  fold gains into W_Q, [W_K;W_V], [W_up;W_gate] (+ SwiGLU packing)
//          S1 Q   = r(H_w) * H_w W_Q'^T                      tcgen05 GEMM, row-norm epilogue
//          S2 K|V = r(H_s) * H_s [W_K;W_V]'^T                tcgen05 GEMM, row-norm epilogue
//          S3 A   = attention (split-L) + log-sum-exp combine
//          S4 G   = SiLU([A | H_w] W_F1^T),  F = H_w + G W_F2^T   (two-source GEMM, SiLU / residual)
//          S5 U   = SiLU(gate) * up of r(F) * F W_ug'^T,  H_f = F + U W_down^T
//   Precision policy (bf16 mode): weights, states, Q, K, V and P are bf16 tensor-core operands;
//   the residual stream (H_w between layers, F, H_f) is kept in fp32, and every token-side
//   activation that feeds a GEMM (H_w, A, G, F, U) is carried as a bf16 hi/lo pair whose two
//   MMAs per k-step give ~16-bit operand precision. Only the final H_f is rounded to bf16.
//   fp32:  the same steps with SIMT kernels (correctness mode).
#include "whale_fusion.h"

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <functional>
#include <utility>
#include <mutex>
#include <vector>

#include "absorbed.cuh"
#include "aux_kernels.cuh"
#include "attention.cuh"
#include "attention_qtile.cuh"
#include "attention_bwd.cuh"
#include "attention_bwd_tc.cuh"
#include "backward.cuh"
#include "fp32_path.cuh"
#include "gemm_2sm.cuh"
#include "gemm_tc.cuh"
#include "ptx.cuh"

using namespace whale;

namespace {

#define WCHECK(x)                          \
  do {                                     \
    whale_status _s = (x);                 \
    if (_s != WHALE_OK) return _s;         \
  } while (0)
#define CUCHECK(x)                         \
  do {                                     \
    cudaError_t _e = (x);                  \
    if (_e != cudaSuccess) {               \
      (void)cudaGetLastError();            \
      return WHALE_ERR_CUDA;               \
    }                                      \
  } while (0)

// An NVTX range over one entry point or one layer, for timeline tools (Nsight Systems); with no
// tool attached the push and pop return at once.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kNumSM = 148;
constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
template <class T>
inline T cdiv(T a, T b) { return (a + b - 1) / b; }

// ------------------------------------------------------------------------------------------
// Launch with programmatic dependent launch (PDL): the kernel may start while the previous kernel
// of the stream drains; it waits (griddepcontrol.wait) before touching global memory.
// ------------------------------------------------------------------------------------------

// Per-kernel timing (whale_profile_begin / whale_profile_end): while on, every kernel launched by
// launch_pdl is followed by an event on its stream (the first one also by a start event). The
// events serialise the launches (no overlap of a kernel's prologue with its predecessor's tail).
struct ProfRec {
  const void* fn;
  cudaEvent_t ev;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
int g_prof_cap = 0;
cudaEvent_t g_prof_start = nullptr;
std::vector<ProfRec> g_prof;

inline void prof_record(const void* fn, cudaStream_t st, bool before) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) return;
  if (before) {
    if (!g_prof_start && cudaEventCreate(&g_prof_start) == cudaSuccess) cudaEventRecord(g_prof_start, st);
    return;
  }
  if ((int)g_prof.size() >= g_prof_cap) return;
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return;
  cudaEventRecord(e, st);
  g_prof.push_back({fn, e});
}

// The same with a cluster shape given at launch (kernels without __cluster_dims__).
template <typename... KArgs, typename... Args>
whale_status launch_cluster_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                unsigned cluster_x, Args&&... args) {
  if (g_prof_on) prof_record(reinterpret_cast<const void*>(kern), st, true);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (g_prof_on) prof_record(reinterpret_cast<const void*>(kern), st, false);
  CUCHECK(e);
  return WHALE_OK;
}

template <typename... KArgs, typename... Args>
whale_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                        Args&&... args) {
  if (g_prof_on) prof_record(reinterpret_cast<const void*>(kern), st, true);
  struct After {
    const void* fn;
    cudaStream_t st;
    ~After() {
      if (g_prof_on) prof_record(fn, st, false);
    }
  } after{reinterpret_cast<const void*>(kern), st};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  CUCHECK(cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...));
  return WHALE_OK;
}

// ------------------------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point (no link-time dependency on libcuda)
// ------------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

whale_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? WHALE_OK : WHALE_ERR_CUDA;
}

// 2-D bf16 row-major tensor [rows, cols] with row stride ld, box [box_rows, box_cols]; the swizzle
// spans one box row (box_cols 64: 128-byte swizzle, 32: 64-byte, 16: 32-byte).
whale_status tmap_bf16_box(CUtensorMap* tm, const void* base, long long rows, long long cols, long long ld,
                           int box_cols, int box_rows) {
  WCHECK(get_encoder());
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * 2) % 16 || rows <= 0 || cols <= 0) return WHALE_ERR_INVALID_ARG;
  if (box_cols != 64 && box_cols != 32 && box_cols != 16) return WHALE_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                       : (box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B),
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WHALE_OK : WHALE_ERR_CUDA;
}

// Box [box_rows, 64 columns], 128-byte swizzle.
whale_status tmap_bf16(CUtensorMap* tm, const void* base, long long rows, long long cols, long long ld, int box_rows) {
  return tmap_bf16_box(tm, base, rows, cols, ld, 64, box_rows);
}

// A K-major bf16 operand [rows, K] (row stride ld, K a multiple of 64) seen as {64 columns, rows,
// K / 64 blocks}: one box {64, box_rows, kps} brings kps consecutive 64-column blocks, each a
// 128-byte-swizzled [box_rows][64] tile.
whale_status tmap_bf16_kblocks(CUtensorMap* tm, const void* base, long long rows, long long K, long long ld,
                               int box_rows, int kps) {
  WCHECK(get_encoder());
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * 2) % 16 || rows <= 0 || K <= 0 || K % 64 || K > ld)
    return WHALE_ERR_INVALID_ARG;
  cuuint64_t dims[3] = {64u, (cuuint64_t)rows, (cuuint64_t)(K / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), 128u};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, (cuuint32_t)kps};
  cuuint32_t es[3] = {1u, 1u, 1u};
  CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WHALE_OK : WHALE_ERR_CUDA;
}

// fp32 splits x [rows, cols] row-major (row stride ld, split stride rows * ld) as {cols, rows, splits}
// with a box of 32 x 32 x 1 (128-byte rows, 128-byte swizzle): the GEMM epilogue's tensor stores,
// which clip rows past `rows` within each split.
whale_status tmap_f32_32(CUtensorMap* tm, const void* base, long long rows, long long cols, long long ld,
                         long long splits) {
  WCHECK(get_encoder());
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * 4) % 16 || rows <= 0 || cols <= 0 || splits <= 0)
    return WHALE_ERR_INVALID_ARG;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)splits};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * 4), (cuuint64_t)(rows * ld * 4)};
  cuuint32_t box[3] = {32u, 32u, 1u};
  cuuint32_t es[3] = {1u, 1u, 1u};
  CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WHALE_OK : WHALE_ERR_CUDA;
}

// The epilogue's store maps o[0..2] (fp32, bf16 hi, bf16 lo) over the GEMM's outputs: cols output
// columns (N, or N / 2 for the SwiGLU epilogue), out_rows rows (M but for the per-head row scatter);
// the fp32 output holds `splits` split-K partials of M rows each. A missing output gets a copy of
// `any` (never stored through).
whale_status epi_maps(CUtensorMap* o, const GemmArgs& g, long long cols, long long splits, const CUtensorMap& any,
                      long long out_rows = 0) {
  if (out_rows <= 0) out_rows = g.M;
  o[0] = o[1] = o[2] = any;
  if (g.out32) WCHECK(tmap_f32_32(&o[0], g.out32, g.M, cols, g.ldo, splits));
  if (g.out_hi) WCHECK(tmap_bf16_box(&o[1], g.out_hi, out_rows, cols, g.ldo, 32, 32));
  if (g.out_lo) WCHECK(tmap_bf16_box(&o[2], g.out_lo, out_rows, cols, g.ldo, 32, 32));
  return WHALE_OK;
}

// Both halves of a K-major bf16 pair [rows, K] (row stride ld) as two planes one byte stride apart:
// base = the lower of the two addresses, pstride = their distance (a multiple of 16, below 2^40).
// kps 1: {K, rows, 2} with box {64, box_rows, 2}; kps 2: {64, rows, K / 64, 2} with box {64,
// box_rows, 2, 2}. One copy then brings [plane][block][row][64], the layout of a stage's A halves.
whale_status tmap_bf16_pair(CUtensorMap* tm, const void* base, long long pstride, long long rows, long long K,
                            long long ld, int box_rows, int kps) {
  WCHECK(get_encoder());
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * 2) % 16 || rows <= 0 || K <= 0 || K % 64 || K > ld ||
      pstride <= 0 || pstride % 16 || pstride >= (1ll << 40))
    return WHALE_ERR_INVALID_ARG;
  CUresult r;
  cuuint32_t es[4] = {1u, 1u, 1u, 1u};
  if (kps == 1) {
    cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, 2u};
    cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)pstride};
    cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 2u};
    r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    cuuint64_t dims[4] = {64u, (cuuint64_t)rows, (cuuint64_t)(K / 64), 2u};
    cuuint64_t strides[3] = {(cuuint64_t)(ld * 2), 128u, (cuuint64_t)pstride};
    cuuint32_t box[4] = {64u, (cuuint32_t)box_rows, (cuuint32_t)kps, 2u};
    r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS ? WHALE_OK : WHALE_ERR_CUDA;
}

// The pair map of an operand when its halves allow one (see tmap_bf16_pair); false otherwise.
bool pair_map(CUtensorMap* tm, const void* hi, const void* lo, long long rows, long long K, long long ld, int box_rows,
              int kps) {
  if (!hi || !lo) return false;
  const uintptr_t h = reinterpret_cast<uintptr_t>(hi), l = reinterpret_cast<uintptr_t>(lo);
  const long long d = h < l ? (long long)(l - h) : (long long)(h - l);
  return tmap_bf16_pair(tm, h < l ? hi : lo, d, rows, K, ld, box_rows, kps) == WHALE_OK;
}

// A K-major operand's map for stages of kps K blocks (kps 1: the 2-D map).
whale_status tmap_operand(CUtensorMap* tm, const void* base, long long rows, long long K, long long ld, int box_rows,
                          int kps) {
  return kps == 1 ? tmap_bf16(tm, base, rows, K, ld, box_rows) : tmap_bf16_kblocks(tm, base, rows, K, ld, box_rows, kps);
}

// ------------------------------------------------------------------------------------------
// Validated shape
// ------------------------------------------------------------------------------------------
struct Shape {
  bool bf16;
  int layers, d, h, dh, N, H, Fh;
  bool shared_kv, tied, debug, prepared;
  bool absorbed;  // bf16 attention with K and V folded into the queries (absorbed.cuh)
  float eps;
  int kvw;  // kv row width: 2d, or d with shared K = V
  int ugw;  // rows of the up|gate matrix: 2H, or H with a tied gate
  size_t es;  // element size
};

// Shapes the absorbed attention handles: 256 absorbed queries per example (two CTAs of 128), one
// 64-column K block per head for the query-side GEMM, d a multiple of the 256-column MMA.
bool absorbed_shape(const Shape& s) {
  return s.bf16 && (long long)s.N * s.h == kAbsQ && s.dh == 64 && (s.d == 256 || s.d == 512);
}

whale_status validate(const whale_config* c, Shape* s) {
  if (!c || !s) return WHALE_ERR_INVALID_ARG;
  if (c->n_layers < 1 || c->d < 1 || c->n_heads < 1 || c->n_tokens < 1 || c->ffn_hidden < 1 ||
      c->fusion_hidden < 0 || !(c->eps >= 0.f) || (c->dtype != WHALE_FP32 && c->dtype != WHALE_BF16) ||
      (c->flags & ~(WHALE_SHARED_KV | WHALE_TIED_GATE | WHALE_DEBUG | WHALE_PREPARED_WEIGHTS | WHALE_MATERIALIZED_KV)) ||
      c->d % c->n_heads)
    return WHALE_ERR_INVALID_ARG;
  s->bf16 = c->dtype == WHALE_BF16;
  s->layers = c->n_layers;
  s->d = c->d;
  s->h = c->n_heads;
  s->dh = c->d / c->n_heads;
  s->N = c->n_tokens;
  s->H = c->ffn_hidden;
  s->Fh = c->fusion_hidden;
  s->shared_kv = c->flags & WHALE_SHARED_KV;
  s->tied = c->flags & WHALE_TIED_GATE;
  s->debug = c->flags & WHALE_DEBUG;
  s->prepared = (c->flags & WHALE_PREPARED_WEIGHTS) && c->dtype == WHALE_BF16;
  s->eps = c->eps;
  s->kvw = s->shared_kv ? s->d : 2 * s->d;
  s->ugw = s->tied ? s->H : 2 * s->H;
  s->es = s->bf16 ? 2 : 4;
  s->absorbed = absorbed_shape(*s) && !(c->flags & WHALE_MATERIALIZED_KV);
  if (s->bf16) {
    const int hg = s->h < 8 ? s->h : 8;
    if (s->d % 64 || (s->dh != 32 && s->dh != 64) || s->h % hg || (hg * s->dh) % 64 || (hg != 2 && hg != 4 && hg != 8) ||
        s->H % 64 || s->Fh % 64)
      return WHALE_ERR_UNSUPPORTED;
  } else {
    if (s->dh != 8 && s->dh != 16 && s->dh != 32 && s->dh != 64 && s->dh != 128) return WHALE_ERR_UNSUPPORTED;
  }
  return WHALE_OK;
}

whale_status check_hint(const whale_shape_hint* h) {
  if (!h || h->B < 0 || h->max_L < 0 || h->total_L < 0 || h->total_L >= (1ll << 31)) return WHALE_ERR_INVALID_ARG;
  return WHALE_OK;
}

// ------------------------------------------------------------------------------------------
// Attention plan (bf16 split-L kernel)
// ------------------------------------------------------------------------------------------
struct AttnPlan {
  int QT, QB, nqb, T, HG, G;
  size_t po_elems, pml_elems, cnt_elems;
  // scratch layout: partial o | partial (m, l) | per-item counters
  size_t po_off() const { return 0; }
  size_t pml_off() const { return align_up(po_elems * 4); }
  size_t cnt_off() const { return pml_off() + align_up(pml_elems * 4); }
  size_t bytes() const { return cnt_off() + cnt_elems * 4; }
};

AttnPlan plan_attention(const Shape& s, int B, long long total_L) {
  AttnPlan p{};
  p.QT = s.N <= 16 ? 1 : (s.N <= 32 ? 2 : 4);
  p.QB = 16 * p.QT;
  p.nqb = cdiv(s.N, p.QB);
  p.T = (s.dh == 64 || p.QT == 4) ? 32 : 64;
  p.HG = s.h < 8 ? s.h : 8;
  // one CTA per SM (the stage ring takes most of shared memory); each CTA streams an equal
  // slice of the flattened work rows, at least a few tiles of them
  const long long work_rows = total_L * p.nqb;
  long long G = cdiv<long long>(work_rows, 4ll * p.T);
  if (G > kNumSM) G = kNumSM;
  if (G < 1) G = 1;
  p.G = (int)G;
  const size_t slots = (size_t)B * p.nqb + p.G;
  p.pml_elems = slots * s.h * p.QB * 2;
  p.po_elems = slots * s.h * p.QB * s.dh;
  p.cnt_elems = (size_t)B * p.nqb;
  return p;
}

// ------------------------------------------------------------------------------------------
// Workspace layout of the forward (the step entry points use prefixes of their own)
// ------------------------------------------------------------------------------------------
struct Layout {
  size_t wq, wkv, wug;   // prepared weights (bf16)
  size_t po, pml;        // attention partials (bf16)
  size_t r;              // row factors (fp32 path)
  size_t q, kv, a, g, f, u, ug, x0, x1;   // fp32 path, and q / kv of the bf16 path
  // bf16 path: lo halves of the token-side operand pairs and the fp32 residual stream
  size_t a_lo, g_lo, f_lo, u_lo, f32, x32[2], xhi[2], xlo[2];
  // absorbed attention: folded key weights, absorbed queries, weights pw, unit references,
  // segment statistics, partial z, unit starts, z as a bf16 pair
  size_t wkabs, qa, pw, mref, stw, stp, pz, ust, zh, pst, pq;
  long long units_max;
  size_t total;
};

constexpr int kMaxPairs = kAbsMaxPairs;
static_assert(kAbsMaxPairs == kNumSM / 2, "one CTA pair per two SMs");

// Units of 256 history rows: sum_b ceil(L_b / 256) <= ceil(total_L / 256) + B.
long long abs_units_max(const whale_shape_hint& h) { return cdiv<long long>(h.total_L, kAbsRows) + h.B; }

Layout make_layout(const Shape& s, const whale_shape_hint& hint) {
  Layout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  const size_t rows = (size_t)hint.B * s.N;
  const size_t tl = (size_t)hint.total_L;
  if (s.bf16) {
    L.wq = take((size_t)s.d * s.d * 2);
    L.wkv = take((size_t)s.kvw * s.d * 2);
    L.wug = take((size_t)s.ugw * s.d * 2);
    AttnPlan p = plan_attention(s, hint.B, hint.total_L);  // also the step entry points' scratch
    L.po = take(p.bytes());
    L.pml = 0;
  } else {
    L.r = take((rows > tl ? rows : tl) * 4);
  }
  L.q = take(rows * s.d * s.es);
  L.kv = s.absorbed ? 0 : take(tl * s.kvw * s.es);
  if (s.absorbed) {
    L.units_max = abs_units_max(hint);
    L.wkabs = take((size_t)s.h * s.d * s.dh * 2);
    L.qa = take((size_t)hint.B * kAbsQ * s.d * 2);
    L.pw = take((size_t)L.units_max * kAbsRows * kAbsQ * 2);
    L.mref = take((size_t)L.units_max * kAbsQ * 4);
    L.stw = take((size_t)hint.B * kAbsQ * 8);
    L.stp = take((size_t)2 * kMaxPairs * kAbsQ * 8);
    L.pz = take((size_t)2 * kMaxPairs * kAbsQ * s.d * 2);
    L.ust = take(((size_t)hint.B + 1) * 4);
    L.pst = take((size_t)kMaxPairs * 8 * 4);
    L.pq = take((size_t)(2 + kMaxPairs) * 4);
    L.zh = take((size_t)hint.B * kAbsQ * s.d * 2);
  }
  L.a = take(rows * s.d * s.es);
  L.g = take(rows * (size_t)s.Fh * s.es);
  L.f = take(rows * s.d * s.es);
  L.u = take(rows * (size_t)s.H * s.es);
  if (s.bf16) {
    L.a_lo = take(rows * s.d * 2);
    L.g_lo = take(rows * (size_t)s.Fh * 2);
    L.f_lo = take(rows * s.d * 2);
    L.u_lo = take(rows * (size_t)s.H * 2);
    L.f32 = take(rows * s.d * 4);
    for (int i = 0; i < 2; ++i) {
      L.x32[i] = take(rows * s.d * 4);
      L.xhi[i] = take(rows * s.d * 2);
      L.xlo[i] = take(rows * s.d * 2);
    }
  } else {
    L.ug = take(rows * (size_t)s.ugw * 4);
    L.x0 = take(rows * s.d * s.es);
    L.x1 = take(rows * s.d * s.es);
  }
  L.total = o;
  return L;
}

inline char* at(void* ws, size_t off) { return static_cast<char*>(ws) + off; }

// ------------------------------------------------------------------------------------------
// bf16 tcgen05 GEMM dispatch
// ------------------------------------------------------------------------------------------
// A GEMM operand: bf16 rows [M, K] with row stride ld; `lo` (optional) is the second half of
// a hi/lo pair (SPLIT mode).
struct Opnd {
  const void* hi;
  const void* lo;
  long long ld;
  int K;
};
// Where the epilogue writes (any may be null): bf16 hi, bf16 residue lo, fp32.
struct Outs {
  void* hi;
  void* lo;
  float* f32;
  long long ld;
};

// tm: the operand maps [A0, A0 lo, A1, A1 lo, W] and, for TST, the store maps [fp32, hi, lo] (eight).
template <int BN, int EPI, bool RN, bool SPLIT, bool A_MN = false, bool B_MN = false, bool SPLIT_B = false,
          int KPS = 1, bool TST = true>
whale_status launch_gemm_t(const CUtensorMap* tm, const GemmArgs& g, long long tiles, cudaStream_t st) {
  if constexpr (GemmSmem<BN, SPLIT, SPLIT_B, KPS, TST>::STAGES < 2) {
    return WHALE_ERR_UNSUPPORTED;  // two stages of this tile do not fit in shared memory
  } else {
    const size_t smem = GemmSmem<BN, SPLIT, SPLIT_B, KPS, TST>::BYTES;
    auto kern = gemm_tc_kernel<BN, EPI, RN, SPLIT, A_MN, B_MN, SPLIT_B, KPS, TST>;
    CUCHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    const unsigned grid = (unsigned)(tiles < kNumSM ? tiles : kNumSM);
    return launch_pdl(kern, dim3(grid), dim3(gemm_threads<RN>()), smem, st, tm[0], tm[1], tm[2], tm[3], tm[4], tm[5],
                      tm[6], tm[7], g);
  }
}

template <int BN, int KPS>
whale_status launch_gemm_bn(int epi, bool rn, bool split, const CUtensorMap* tm, const GemmArgs& g, long long tiles,
                            cudaStream_t st) {
  if (rn && epi == EPI_STORE && !split)
    return launch_gemm_t<BN, EPI_STORE, true, false, false, false, false, KPS>(tm, g, tiles, st);
  if (rn && epi == EPI_STORE && split)
    return launch_gemm_t<BN, EPI_STORE, true, true, false, false, false, KPS>(tm, g, tiles, st);
  if (!split) return WHALE_ERR_UNSUPPORTED;
  if (!rn && epi == EPI_STORE) return launch_gemm_t<BN, EPI_STORE, false, true, false, false, false, KPS>(tm, g, tiles, st);
  if (rn && epi == EPI_SWIGLU) return launch_gemm_t<BN, EPI_SWIGLU, true, true, false, false, false, KPS>(tm, g, tiles, st);
  if (rn && epi == EPI_SWIGLU_TIED)
    return launch_gemm_t<BN, EPI_SWIGLU_TIED, true, true, false, false, false, KPS>(tm, g, tiles, st);
  if (!rn && epi == EPI_SILU) return launch_gemm_t<BN, EPI_SILU, false, true, false, false, false, KPS>(tm, g, tiles, st);
  if (!rn && epi == EPI_RESID) return launch_gemm_t<BN, EPI_RESID, false, true, false, false, false, KPS>(tm, g, tiles, st);
  return WHALE_ERR_UNSUPPORTED;
}

// Pipeline cost of one stage in SM cycles, as measured for TMA tensor copies of L2-resident tiles on
// B200 (one CTA per SM, rings of 2 to 8 stages of 1 to 8 copies): each stage (one mbarrier) costs a
// fixed ~470 cycles, each copy ~160 more and its bytes one cycle per ~240, almost independent of how
// many stages are in flight. Two-K-block stages took the K loop of the Fusion MLP's GEMMs from 0.51
// to 0.40 us per K block when run alone.
inline double gemm_stage_cycles(int bn, bool split, int kps) {
  const double copies = split ? 3.0 : 2.0;
  const double bytes = kps * ((split ? 32768.0 : 16384.0) + bn * 128.0);
  const double load = 470.0 + 160.0 * copies + bytes / 240.0;
  const double mma = kps * (split ? 4.0 : 2.0) * bn;
  return std::max(load, mma);
}

// Shared memory of a tile configuration holds at least two stages.
template <int BN>
bool gemm_kps2_fits(bool split) {
  return split ? GemmSmem<BN, true, false, 2, true>::STAGES >= 2 : GemmSmem<BN, false, false, 2, true>::STAGES >= 2;
}

// Co-resident 2-CTA clusters of the 2-SM GEMM on the current device (cached per device).
whale_status g2_max_pairs(int* pairs) {
  static std::mutex mu;
  static int cache[64];
  int dev = 0;
  CUCHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return WHALE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    auto kern = gemm_rownorm_2sm_kernel;
    CUCHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G2Smem::BYTES));
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(2 * kNumSM / 2, 1, 1);
    lc.blockDim = dim3(kG2Threads, 1, 1);
    lc.dynamicSmemBytes = G2Smem::BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int n = 0;
    CUCHECK(cudaOccupancyMaxActiveClusters(&n, kern, &lc));
    cache[dev] = n > 0 ? n : -1;
  }
  *pairs = cache[dev];
  return WHALE_OK;
}

// out = r(A) * (A W^T) in bf16 on 256 x 256 tiles, one persistent CTA pair per two SMs.
whale_status gemm_rownorm_2sm(const Opnd& a0, const void* W, int N, const Outs& out, long long M, float eps,
                              int pairs, cudaStream_t st) {
  CUtensorMap ta, tb, to;
  WCHECK(tmap_bf16(&ta, a0.hi, M, a0.K, a0.ld, 128));
  WCHECK(tmap_bf16(&tb, W, N, a0.K, a0.K, 128));
  WCHECK(tmap_bf16(&to, out.hi, M, N, out.ld, 32));
  G2Args g{};
  g.M = (int)M;
  g.N = N;
  g.kb = a0.K / 64;
  g.tiles_n = N / 256;
  g.num_tiles = (int)(cdiv<long long>(M, 256) * g.tiles_n);
  g.inv_k = 1.0f / (float)a0.K;
  g.eps = eps;
  if (pairs > g.num_tiles) pairs = g.num_tiles;
  auto kern = gemm_rownorm_2sm_kernel;
  CUCHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G2Smem::BYTES));
  return launch_pdl(kern, dim3(2 * pairs), dim3(kG2Threads), G2Smem::BYTES, st, ta, tb, to, g);
}

// out = epi([A0 | A1] W^T), W [N, K0+K1] bf16; SPLIT when the operands carry lo halves.
whale_status gemm_bf16(const Opnd& a0, const Opnd& a1, const void* W, int N, const Outs& out, const float* resid32,
                       long long ldr, long long M, int epi, bool rn, float eps, cudaStream_t st) {
  if (M <= 0) return WHALE_OK;
  if (M >= (1ll << 31)) return WHALE_ERR_UNSUPPORTED;
  const bool split = a0.lo != nullptr;
  if (a0.K % 64 || a1.K % 64 || N % 64 || (a1.K > 0 && (a1.lo != nullptr) != split)) return WHALE_ERR_UNSUPPORTED;
  const long long tm = cdiv<long long>(M, 128);
  // Large single-source row-norm projections (the history-side K|V GEMM): the 2-SM persistent kernel
  // (256 x 256 tiles on CTA pairs) where N allows; otherwise the one-CTA kernel below.
  if (!split && rn && epi == EPI_STORE && a1.K == 0 && out.hi && !out.lo && !out.f32 && N % 128 == 0 &&
      tm * (N / 128) >= 2 * kNumSM) {
    int pairs = 0;
    if (N % 256 == 0) WCHECK(g2_max_pairs(&pairs));
    if (pairs > 0) return gemm_rownorm_2sm(a0, W, N, out, M, eps, pairs, st);
  }
  // Tile width and K blocks per stage by a small cost model (cycles): per-CTA fixed cost + tiles per
  // persistent CTA x stages per tile x the larger of a stage's MMA time and its TMA cost.
  const int KB = (a0.K + a1.K) / 64;
  const bool kps2_ok = KB % 2 == 0 && (a0.K / 64) % 2 == 0;
  auto cost = [&](int bn, int kps) -> double {
    if (N % bn) return 1e300;
    if (kps == 2) {
      const bool fits = bn == 64 ? gemm_kps2_fits<64>(split) : bn == 128 ? gemm_kps2_fits<128>(split)
                                                                         : gemm_kps2_fits<256>(split);
      if (!kps2_ok || !fits) return 1e300;
    }
    const double per_cta = (double)cdiv<long long>(tm * (N / bn), kNumSM);  // tiles per persistent CTA
    return 5600.0 + per_cta * (KB / kps) * gemm_stage_cycles(bn, split, kps);
  };
  int bn = 64, kps = 1;
  for (int cand : {64, 128, 256})
    for (int kc : {1, 2})
      if (cost(cand, kc) < cost(bn, kps)) {
        bn = cand;
        kps = kc;
      }
  CUtensorMap maps[8];
  // hi/lo pairs: one two-plane map per source where both sources allow it (one copy per stage each)
  bool planes = split && pair_map(&maps[0], a0.hi, a0.lo, M, a0.K, a0.ld, 128, kps) &&
                (a1.K == 0 || pair_map(&maps[2], a1.hi, a1.lo, M, a1.K, a1.ld, 128, kps));
  if (planes) {
    maps[1] = maps[0];
    if (a1.K == 0) maps[2] = maps[0];
    maps[3] = maps[2];
  } else {
    WCHECK(tmap_operand(&maps[0], a0.hi, M, a0.K, a0.ld, 128, kps));
    if (split) WCHECK(tmap_operand(&maps[1], a0.lo, M, a0.K, a0.ld, 128, kps));
    else maps[1] = maps[0];
    if (a1.K > 0) {
      WCHECK(tmap_operand(&maps[2], a1.hi, M, a1.K, a1.ld, 128, kps));
      if (split) WCHECK(tmap_operand(&maps[3], a1.lo, M, a1.K, a1.ld, 128, kps));
      else maps[3] = maps[2];
    } else {
      maps[2] = maps[0];
      maps[3] = maps[1];
    }
  }
  WCHECK(tmap_operand(&maps[4], W, N, a0.K + a1.K, a0.K + a1.K, bn, kps));
  GemmArgs g{};
  g.M = (int)M;
  g.N = N;
  g.kb0 = a0.K / 64;
  g.kb1 = a1.K / 64;
  g.tiles_n = N / bn;
  g.num_tiles = (int)(tm * g.tiles_n);
  g.inv_k = 1.0f / (float)a0.K;
  g.eps = eps;
  g.out_hi = static_cast<__nv_bfloat16*>(out.hi);
  g.out_lo = static_cast<__nv_bfloat16*>(out.lo);
  g.out32 = out.f32;
  g.ldo = out.ld;
  g.resid32 = resid32;
  g.ldr = ldr;
  g.a_planes = planes ? 1 : 0;
  WCHECK(epi_maps(maps + 5, g, epi == EPI_SWIGLU ? N / 2 : N, 1, maps[0]));
  const long long tiles = tm * g.tiles_n;
  if (kps == 2) {
    if (bn == 256) return launch_gemm_bn<256, 2>(epi, rn, split, maps, g, tiles, st);
    if (bn == 128) return launch_gemm_bn<128, 2>(epi, rn, split, maps, g, tiles, st);
    return launch_gemm_bn<64, 2>(epi, rn, split, maps, g, tiles, st);
  }
  if (bn == 256) return launch_gemm_bn<256, 1>(epi, rn, split, maps, g, tiles, st);
  if (bn == 128) return launch_gemm_bn<128, 1>(epi, rn, split, maps, g, tiles, st);
  return launch_gemm_bn<64, 1>(epi, rn, split, maps, g, tiles, st);
}

// ------------------------------------------------------------------------------------------
// General bf16 contraction into fp32 for the backward pass: C[M, N] = sum_k A(m, k) B(k, n).
//   A: K-major [M, K] (a.hi, optional bf16 residue a.lo: two MMAs per k-step; row stride a.ld), or
//      with a_mn MN-major [K, M] (a.hi only, row stride a.ld);
//   B: K-major [N, K] (row stride ldb) or, with b_mn, MN-major [K, N] (row stride ldb).
// K need not be a multiple of 64 (the TMA boxes read zeros past K). Output tiles that would leave SMs
// idle with a long K take split-K: fp32 partials of ksplit K ranges in `part` (part_cap floats), then
// summed in split order (deterministic).
// ------------------------------------------------------------------------------------------
template <int BN>
whale_status launch_acc32_bn(bool split, bool split_b, bool a_mn, bool b_mn, const CUtensorMap* tm, const GemmArgs& g,
                             long long tiles, cudaStream_t st) {
  if (!b_mn) return WHALE_ERR_UNSUPPORTED;
  if (!a_mn && split && !split_b) return launch_gemm_t<BN, EPI_STORE, false, true, false, true>(tm, g, tiles, st);
  if (!a_mn && !split && !split_b) return launch_gemm_t<BN, EPI_STORE, false, false, false, true>(tm, g, tiles, st);
  if (a_mn && !split && !split_b) return launch_gemm_t<BN, EPI_STORE, false, false, true, true>(tm, g, tiles, st);
  if (a_mn && split && !split_b) return launch_gemm_t<BN, EPI_STORE, false, true, true, true>(tm, g, tiles, st);
  if (a_mn && split && split_b) return launch_gemm_t<BN, EPI_STORE, false, true, true, true, true>(tm, g, tiles, st);
  return WHALE_ERR_UNSUPPORTED;
}

whale_status gemm_acc32(const void* a_hi, const void* a_lo, long long lda, bool a_mn, const void* b, long long ldb,
                        bool b_mn, long long M, int N, long long K, float* c, long long ldc, float* part,
                        size_t part_cap, cudaStream_t st, const void* b_lo = nullptr) {
  if (M <= 0 || N <= 0) return WHALE_OK;
  if (K <= 0) {
    for (long long r = 0; r < M; ++r) CUCHECK(cudaMemsetAsync(c + r * ldc, 0, (size_t)N * 4, st));
    return WHALE_OK;
  }
  if (M >= (1ll << 31) || K >= (1ll << 31) || N % 64) return WHALE_ERR_UNSUPPORTED;
  const bool split = a_lo != nullptr, split_b = b_lo != nullptr;
  if (split_b && !split) return WHALE_ERR_UNSUPPORTED;
  const long long tm = cdiv<long long>(M, 128);
  const long long KB = cdiv<long long>(K, 64);
  // Tile width and split-K together, by a cost model (cycles): waves of CTAs x K blocks per CTA x
  // max(MMA time, operand bytes at ~80 B/clk per SM). When the output has fewer tiles than SMs and K
  // is long, ks K ranges per tile (fp32 partials within part_cap, at least 8 K blocks each) fill the
  // SMs in one wave; wider tiles then re-read the operands fewer times.
  const double mma_per_col = split ? (split_b ? 6.0 : 4.0) : 2.0;
  auto plan = [&](int bn, int* ks_out) -> double {
    if (N % bn) return 1e300;
    const long long tiles = tm * (N / bn);
    int k = 1;
    if (tiles < kNumSM && KB >= 16 && part) {
      long long want = std::min<long long>(std::max<long long>(1, kNumSM / tiles), KB / 8);
      while (want > 1 && (size_t)want * M * N > part_cap) --want;
      k = (int)std::max<long long>(1, std::min<long long>(want, 64));
    }
    *ks_out = k;
    const double waves = (double)cdiv<long long>(tiles * k, kNumSM);
    const double bytes = (split ? 32768.0 : 16384.0) + bn * 128.0 * (split_b ? 2 : 1);
    return 5600.0 + waves * (double)cdiv<long long>(KB, k) * std::max(mma_per_col * bn, bytes / 80.0);
  };
  int bn = 64, ks = 1, ks_c = 1;
  double best = plan(64, &ks);
  for (int cand : {128, 256}) {
    const double cost = plan(cand, &ks_c);
    if (cost < best) {
      best = cost;
      bn = cand;
      ks = ks_c;
    }
  }
  const long long tiles_mn = tm * (N / bn);
  int kb_split = (int)cdiv<long long>(KB, ks);
  ks = (int)cdiv<long long>(KB, kb_split);  // no empty split
  CUtensorMap maps[8];
  if (a_mn) {
    WCHECK(tmap_bf16_box(&maps[0], a_hi, K, M, lda, 64, 64));
    if (split) WCHECK(tmap_bf16_box(&maps[1], a_lo, K, M, lda, 64, 64));
    else maps[1] = maps[0];
  } else {
    WCHECK(tmap_bf16(&maps[0], a_hi, M, K, lda, 128));
    if (split) WCHECK(tmap_bf16(&maps[1], a_lo, M, K, lda, 128));
    else maps[1] = maps[0];
  }
  maps[2] = maps[0];
  maps[3] = maps[1];
  if (b_mn) {
    WCHECK(tmap_bf16_box(&maps[4], b, K, N, ldb, 64, 64));
    if (split_b) WCHECK(tmap_bf16_box(&maps[2], b_lo, K, N, ldb, 64, 64));  // B's lo half rides in the A1 slot
  } else {
    WCHECK(tmap_bf16(&maps[4], b, N, K, ldb, bn));
    if (split_b) WCHECK(tmap_bf16(&maps[2], b_lo, N, K, ldb, bn));
  }
  GemmArgs g{};
  g.M = (int)M;
  g.N = N;
  g.kb0 = (int)KB;
  g.kb1 = 0;
  g.tiles_n = N / bn;
  g.num_tiles = (int)(tiles_mn * ks);
  g.ksplit = ks;
  g.kb_split = kb_split;
  if (ks > 1) {
    g.out32 = part;
    g.ldo = N;
    g.split_stride = M * N;
  } else {
    g.out32 = c;
    g.ldo = ldc;
  }
  WCHECK(epi_maps(maps + 5, g, N, ks, maps[0]));
  const long long tiles = tiles_mn * ks;
  whale_status r;
  if (bn == 256) r = launch_acc32_bn<256>(split, split_b, a_mn, b_mn, maps, g, tiles, st);
  else if (bn == 128) r = launch_acc32_bn<128>(split, split_b, a_mn, b_mn, maps, g, tiles, st);
  else r = launch_acc32_bn<64>(split, split_b, a_mn, b_mn, maps, g, tiles, st);
  WCHECK(r);
  if (ks > 1) {
    if (N % 4 == 0 && ldc % 4 == 0 && !(reinterpret_cast<uintptr_t>(c) & 15)) {
      const unsigned grid = (unsigned)std::min<long long>(cdiv<long long>(M * N / 4, 256), 8 * kNumSM);
      WCHECK(launch_pdl(sum_partials4_kernel, dim3(grid), dim3(256), 0, st, (const float*)part, ks, M, N, c, ldc));
    } else {
      const unsigned grid = (unsigned)std::min<long long>(cdiv<long long>(M * N, 256), 8 * kNumSM);
      WCHECK(launch_pdl(sum_partials_kernel, dim3(grid), dim3(256), 0, st, (const float*)part, ks, M, N, c, ldc));
    }
  }
  return WHALE_OK;
}

// fp32 (SIMT) contraction with arbitrary strides: C[m, n] = sum_k A[m sam + k sak] B[k sbk + n sbn].
whale_status gemm_strided_f32(const float* A, long long sam, long long sak, const float* B, long long sbk,
                              long long sbn, float* C, long long ldc, long long M, long long N, long long K,
                              cudaStream_t st) {
  if (M <= 0 || N <= 0) return WHALE_OK;
  const long long gy = cdiv<long long>(M, 64);
  if (gy > 65535) return WHALE_ERR_UNSUPPORTED;
  gemm_strided_f32_kernel<<<dim3((unsigned)cdiv<long long>(N, 64), (unsigned)gy), 256, 0, st>>>(
      A, sam, sak, B, sbk, sbn, C, ldc, M, N, K, 0);
  CUCHECK(cudaGetLastError());
  return WHALE_OK;
}

inline Opnd opnd(const void* hi, const void* lo, long long ld, int K) { return Opnd{hi, lo, ld, K}; }
inline Opnd no_opnd() { return Opnd{nullptr, nullptr, 0, 0}; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

whale_status pair_from_bf16(const void* x, float* x32, void* lo, long long n, cudaStream_t st) {
  if (n <= 0) return WHALE_OK;
  if (aligned16(x) && aligned16(x32) && aligned16(lo)) {
    const unsigned grid = (unsigned)std::min<long long>(cdiv<long long>(cdiv<long long>(n, 8), 256), 8 * kNumSM);
    return launch_pdl(pair_from_bf16_8_kernel, dim3(grid), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x),
                      x32, static_cast<__nv_bfloat16*>(lo), n);
  }
  const unsigned grid = (unsigned)std::min<long long>(cdiv<long long>(n, 256), 8 * kNumSM);
  return launch_pdl(pair_from_bf16_kernel, dim3(grid), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x), x32,
                    static_cast<__nv_bfloat16*>(lo), n);
}

// ------------------------------------------------------------------------------------------
// bf16 steps
// ------------------------------------------------------------------------------------------
// Log2(e) / sqrt(d_head): the attention scale in base-2 units.
inline float scale_log2_of(const Shape& s) { return (float)(1.4426950408889634 / std::sqrt((double)s.dh)); }

// Fold the gains into the weights (one launch for all jobs). `okabs` (optional) receives the
// absorbed key weights from W_K = the first d rows of `wkv_kabs` with gain `gkv_kabs`.
whale_status fold_weights(const Shape& s, const __nv_bfloat16* wq, const float* gq, const __nv_bfloat16* wkv,
                          const float* gkv, const __nv_bfloat16* wug, const float* gffn, __nv_bfloat16* oq,
                          __nv_bfloat16* okv, __nv_bfloat16* oug, cudaStream_t st,
                          const __nv_bfloat16* wkv_kabs = nullptr, const float* gkv_kabs = nullptr,
                          __nv_bfloat16* okabs = nullptr) {
  FoldJobs jobs{};
  long long maxe = 0;
  auto add = [&](const __nv_bfloat16* w, const float* g, __nv_bfloat16* out, int rows, int cols, int mode) {
    if (!w || !out) return;
    FoldJob& j = jobs.job[jobs.n++];
    j.w = w;
    j.g = g;
    j.out = out;
    j.rows = rows;
    j.cols = cols;
    j.mode = mode;
    j.H = mode == 2 ? s.dh : s.H;
    j.src_cols = s.d;
    j.scale = mode == 2 ? scale_log2_of(s) : 1.f;
    maxe = std::max(maxe, (long long)rows * cols);
  };
  add(wq, gq, oq, s.d, s.d, 0);
  add(wkv, gkv, okv, s.kvw, s.d, 0);
  add(wug, gffn, oug, s.ugw, s.d, s.tied ? 0 : 1);
  add(wkv_kabs, gkv_kabs, okabs, s.h * s.d, s.dh, 2);
  if (jobs.n == 0) return WHALE_OK;
  const unsigned gx = (unsigned)std::min<long long>(cdiv<long long>(maxe / 8, 256), 8 * kNumSM);
  return launch_pdl(fold_weights_kernel, dim3(gx, jobs.n), dim3(256), 0, st, jobs);
}

template <int DH, int QT, int HG>
whale_status launch_attn_t(const CUtensorMap& tm, const AttnArgs& a, dim3 grid, cudaStream_t st) {
  constexpr int T = (DH == 64 || QT == 4) ? 32 : 64;
  using C = AttnCfg<DH, QT, T, HG>;
  constexpr int stage = 2 * C::KV_BYTES;
  constexpr int ST = (196608 / stage) > 4 ? 4 : ((196608 / stage) < 2 ? 2 : (196608 / stage));
  const size_t smem = 1024 + (size_t)ST * stage + 256;
  auto kern = attn_splitl_kernel<DH, QT, T, HG, ST>;
  CUCHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  return launch_pdl(kern, grid, dim3(C::THREADS), smem, st, tm, a);
}

template <int DH, int QT>
whale_status launch_attn_hg(int hg, const CUtensorMap& tm, const AttnArgs& a, dim3 grid, cudaStream_t st) {
  if (hg == 8) return launch_attn_t<DH, QT, 8>(tm, a, grid, st);
  if (hg == 4) return launch_attn_t<DH, QT, 4>(tm, a, grid, st);
  if (hg == 2) return launch_attn_t<DH, QT, 2>(tm, a, grid, st);
  return WHALE_ERR_UNSUPPORTED;
}

// Query-tiled attention (attention_qtile.cuh): one CTA per (example, 128 queries, head box).
whale_status attention_qtile(const Shape& s, const void* q, const void* kv, const int* offsets, void* out,
                             void* out_lo, int B, long long total_L, cudaStream_t st) {
  QtArgs a{};
  a.offsets = offsets;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.out_lo = static_cast<__nv_bfloat16*>(out_lo);
  a.B = B;
  a.N = s.N;
  a.d = s.d;
  a.n_qt = (int)cdiv<long long>(s.N, 128);
  a.n_hb = s.h / (64 / s.dh);
  a.v_col0 = s.shared_kv ? 0 : s.d;
  a.total_L = total_L;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)s.dh));
  const long long grid = (long long)B * a.n_qt * a.n_hb;
  if (grid <= 0) return WHALE_OK;
  if (grid > 0x7fffffffll) return WHALE_ERR_UNSUPPORTED;
  CUtensorMap tq, tkv;
  WCHECK(tmap_bf16(&tq, q, (long long)B * s.N, s.d, s.d, 128));
  WCHECK(tmap_bf16(&tkv, kv, total_L, s.kvw, s.kvw, 128));
  if (s.dh == 32) {
    CUCHECK(cudaFuncSetAttribute(attn_qtile_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)QtSmem<32>::BYTES));
    return launch_pdl(attn_qtile_kernel<32>, dim3((unsigned)grid), dim3(kQtThreads), QtSmem<32>::BYTES, st, tq, tkv, a);
  }
  CUCHECK(cudaFuncSetAttribute(attn_qtile_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)QtSmem<64>::BYTES));
  return launch_pdl(attn_qtile_kernel<64>, dim3((unsigned)grid), dim3(kQtThreads), QtSmem<64>::BYTES, st, tq, tkv, a);
}

// Histories attended by many queries (N >= 128 per example) take the query-tiled tcgen05 kernel, which
// needs no scratch; the split-L kernel (partials in the scratch of plan_attention) takes the rest.
bool attention_is_query_tiled(const Shape& s) { return s.N >= 128 && (s.dh == 32 || s.dh == 64); }

// lse (optional, split-L kernel only): [B*N, h] log2 softmax denominators for the backward pass.
whale_status attention_bf16(const Shape& s, const void* q, const void* kv, const int* offsets, void* out,
                            void* out_lo, int B, long long total_L, void* scratch, cudaStream_t st,
                            float* lse = nullptr) {
  if (B == 0) return WHALE_OK;
  const AttnPlan p = plan_attention(s, B, total_L);
  const size_t rows = (size_t)B * s.N;
  if (total_L <= 0) {  // every history is empty: A = 0
    CUCHECK(cudaMemsetAsync(out, 0, rows * s.d * 2, st));
    if (out_lo) CUCHECK(cudaMemsetAsync(out_lo, 0, rows * s.d * 2, st));
    return WHALE_OK;
  }
  if (attention_is_query_tiled(s)) {
    if (lse) return WHALE_ERR_UNSUPPORTED;
    return attention_qtile(s, q, kv, offsets, out, out_lo, B, total_L, st);
  }
  AttnArgs a{};
  a.lse = lse;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.offsets = offsets;
  a.part_o = reinterpret_cast<float*>(at(scratch, p.po_off()));
  a.part_ml = reinterpret_cast<float*>(at(scratch, p.pml_off()));
  a.counters = reinterpret_cast<int*>(at(scratch, p.cnt_off()));
  a.out = static_cast<__nv_bfloat16*>(out);
  a.out_lo = static_cast<__nv_bfloat16*>(out_lo);
  a.B = B;
  a.N = s.N;
  a.QB = p.QB;
  a.n_qblocks = p.nqb;
  a.d = s.d;
  a.n_heads = s.h;
  a.v_col0 = s.shared_kv ? 0 : s.d;
  a.shared_kv = s.shared_kv ? 1 : 0;
  a.G = p.G;
  a.total_L = total_L;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)s.dh));
  if ((long long)B * p.nqb > (1ll << 30)) return WHALE_ERR_UNSUPPORTED;
  CUCHECK(cudaMemsetAsync(a.counters, 0, p.cnt_elems * 4, st));
  CUtensorMap tm;
  WCHECK(tmap_bf16(&tm, kv, total_L, s.kvw, s.kvw, p.T));
  const dim3 grid(p.G, s.h / p.HG);
  whale_status r = WHALE_ERR_UNSUPPORTED;
  if (s.dh == 32) {
    if (p.QT == 1) r = launch_attn_hg<32, 1>(p.HG, tm, a, grid, st);
    else if (p.QT == 2) r = launch_attn_hg<32, 2>(p.HG, tm, a, grid, st);
    else r = launch_attn_hg<32, 4>(p.HG, tm, a, grid, st);
  } else {
    if (p.QT == 1) r = launch_attn_hg<64, 1>(p.HG, tm, a, grid, st);
    else if (p.QT == 2) r = launch_attn_hg<64, 2>(p.HG, tm, a, grid, st);
    else r = launch_attn_hg<64, 4>(p.HG, tm, a, grid, st);
  }
  return r;
}

// ------------------------------------------------------------------------------------------
// absorbed attention (bf16; absorbed.cuh)
// ------------------------------------------------------------------------------------------
// Co-resident clusters of both passes (cached per device): their shared memory allows one CTA per SM.
whale_status abs_max_pairs(int E, int* pairs) {
  static std::mutex mu;
  static int cache[64][2];
  int dev = 0;
  CUCHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return WHALE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  int& c = cache[dev][E - 1];
  if (c == 0) {
    auto query = [&](const void* kern, size_t smem, int threads, int* n) -> whale_status {
      CUCHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      cudaLaunchConfig_t lc = {};
      lc.gridDim = dim3(kNumSM, 1, 1);
      lc.blockDim = dim3(threads, 1, 1);
      lc.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      lc.attrs = attr;
      lc.numAttrs = 1;
      CUCHECK(cudaOccupancyMaxActiveClusters(n, kern, &lc));
      return WHALE_OK;
    };
    int na = 0, nb = 0;
    if (E == 1) {
      WCHECK(query(reinterpret_cast<const void*>(abs_scores_kernel<1>), AbsASmem<1>::BYTES, kAbsAThreads, &na));
      WCHECK(query(reinterpret_cast<const void*>(abs_values_kernel<1>), AbsBSmem<1>::BYTES, kAbsBThreads, &nb));
    } else {
      WCHECK(query(reinterpret_cast<const void*>(abs_scores_kernel<2>), AbsASmem<2>::BYTES, kAbsAThreads, &na));
      WCHECK(query(reinterpret_cast<const void*>(abs_values_kernel<2>), AbsBSmem<2>::BYTES, kAbsBThreads, &nb));
    }
    const int n = std::min(std::min(na, nb), kMaxPairs);
    c = n > 0 ? n : -1;
  }
  *pairs = c;
  return c > 0 ? WHALE_OK : WHALE_ERR_UNSUPPORTED;
}

// qa[b*256 + j*N + n, :] = q[b*N + n, j*64 : j*64 + 64] W~_j^T with W~ [h*d, 64] (one K block per
// head: a block-diagonal GEMM over the h*d output columns, rows scattered per head).
whale_status gemm_qabs(const Shape& s, const void* q, const void* wkabs, void* qa, long long rows, cudaStream_t st) {
  constexpr int BN = 256;
  if (s.d % BN || s.dh != 64) return WHALE_ERR_UNSUPPORTED;
  CUtensorMap maps[8];
  WCHECK(tmap_bf16(&maps[0], q, rows, s.d, s.d, 128));
  maps[1] = maps[2] = maps[3] = maps[5] = maps[6] = maps[7] = maps[0];
  WCHECK(tmap_bf16(&maps[4], wkabs, (long long)s.h * s.d, s.dh, s.dh, BN));
  GemmArgs g{};
  g.M = (int)rows;
  g.N = s.h * s.d;
  g.kb0 = s.dh / 64;
  g.kb1 = 0;
  g.tiles_n = g.N / BN;
  const long long tiles = cdiv<long long>(rows, 128) * g.tiles_n;
  g.num_tiles = (int)tiles;
  g.out_hi = static_cast<__nv_bfloat16*>(qa);
  g.ldo = s.d;
  g.head_tiles = s.d / BN;
  g.a_kb_step = s.dh / 64;
  g.a_row_step = 0;
  g.qabs_N = s.N;
  g.qabs_d = s.d;
  g.qabs_rows = kAbsQ;
  if (s.N % 32 == 0) {  // a warp's 32 rows are one example's: tensor stores
    WCHECK(epi_maps(maps + 5, g, s.d, 1, maps[0], rows / s.N * kAbsQ));
    return launch_gemm_t<BN, EPI_QABS, false, false>(maps, g, tiles, st);
  }
  return launch_gemm_t<BN, EPI_QABS, false, false, false, false, false, 1, false>(maps, g, tiles, st);
}

// A[:, j*64 : j*64 + 64] = z_j W'_V,j^T for every head j in one launch: z is the stack [h, rows, d]
// (bf16), W'_V the gain-folded [d, d] value weights (row j*64 + c); A as a bf16 pair.
whale_status gemm_vabs(const Shape& s, const void* zh, const void* wv, void* a, void* a_lo, long long rows,
                       cudaStream_t st) {
  if (s.dh != 64) return WHALE_ERR_UNSUPPORTED;
  const int kps = (s.d / 64) % 2 == 0 ? 2 : 1;
  CUtensorMap maps[8];
  WCHECK(tmap_operand(&maps[0], zh, (long long)s.h * rows, s.d, s.d, 128, kps));
  maps[1] = maps[2] = maps[3] = maps[0];
  WCHECK(tmap_operand(&maps[4], wv, s.d, s.d, s.d, 64, kps));
  GemmArgs g{};
  g.M = (int)rows;
  g.N = s.d;
  g.kb0 = s.d / 64;
  g.kb1 = 0;
  g.tiles_n = s.d / 64;
  const long long tiles = cdiv<long long>(rows, 128) * g.tiles_n;
  g.num_tiles = (int)tiles;
  g.out_hi = static_cast<__nv_bfloat16*>(a);
  g.out_lo = static_cast<__nv_bfloat16*>(a_lo);
  g.ldo = s.d;
  g.head_tiles = 1;
  g.a_kb_step = 0;
  g.a_row_step = rows;
  WCHECK(epi_maps(maps + 5, g, s.d, 1, maps[0]));
  if (kps == 2) return launch_gemm_t<64, EPI_STORE, false, false, false, false, false, 2>(maps, g, tiles, st);
  return launch_gemm_t<64, EPI_STORE, false, false>(maps, g, tiles, st);
}

// CTA pairs of the two-pass kernels.
whale_status abs_two_pass_pairs(const Shape& s, const Layout& L, int* P) {
  *P = 0;
  int pairs = 0;
  WCHECK(abs_max_pairs(s.d / 256, &pairs));
  *P = (int)std::max<long long>(1, std::min<long long>(pairs, L.units_max));
  return WHALE_OK;
}

// Unit starts of the batch and the pairs' starting states (once per forward: the offsets are shared
// by every layer).
whale_status abs_units(const Shape& s, const int* offsets, const whale_shape_hint& hint, void* ws, const Layout& L,
                       cudaStream_t st) {
  if (!s.absorbed || hint.B == 0) return WHALE_OK;
  if (L.units_max >= (1ll << 31) / kAbsRows) return WHALE_ERR_UNSUPPORTED;
  int P = 0;
  WCHECK(abs_two_pass_pairs(s, L, &P));
  return launch_pdl(abs_units_kernel, dim3(1), dim3(1024), 0, st, offsets, hint.B, (long long)hint.total_L,
                    (int)L.units_max, reinterpret_cast<int*>(at(ws, L.ust)), P, reinterpret_cast<int*>(at(ws, L.pst)),
                    reinterpret_cast<int*>(at(ws, L.pq)));
}

// S3 through the absorbed path: q (bf16 [B*N, d]) -> A (bf16 pair [B*N, d]).
whale_status attention_absorbed(const Shape& s, const void* q, const void* slab, const int* offsets,
                                const void* wkabs, const void* wv, void* out, void* out_lo, const whale_shape_hint& hint,
                                void* ws, const Layout& L, cudaStream_t st) {
  if (hint.B == 0) return WHALE_OK;
  const long long rows = (long long)hint.B * s.N;
  const int E = s.d / 256;
  WCHECK(gemm_qabs(s, q, wkabs, at(ws, L.qa), rows, st));
  AbsArgs a{};
  a.offsets = offsets;
  a.ustart = reinterpret_cast<const int*>(at(ws, L.ust));
  a.B = hint.B;
  a.N = s.N;
  a.d = s.d;
  a.total_L = hint.total_L;
  a.inv_d = 1.0f / (float)s.d;
  a.eps = s.eps;
  a.mref = reinterpret_cast<float*>(at(ws, L.mref));
  a.stats_whole = reinterpret_cast<float*>(at(ws, L.stw));
  a.stats_part = reinterpret_cast<float*>(at(ws, L.stp));
  a.part_z = reinterpret_cast<__nv_bfloat16*>(at(ws, L.pz));
  a.z_hi = reinterpret_cast<__nv_bfloat16*>(at(ws, L.zh));
  int P = 0;
  WCHECK(abs_two_pass_pairs(s, L, &P));
  a.n_pairs = P;  // the pair count abs_units tabulated the starts for
  a.pstart = reinterpret_cast<const int*>(at(ws, L.pst));
  a.pq = reinterpret_cast<int*>(at(ws, L.pq));  // pass B takes each pair of pass A as it finishes
  if (hint.total_L > 0) {
    CUtensorMap tq, th, tps;
    WCHECK(tmap_bf16(&tq, at(ws, L.qa), (long long)hint.B * kAbsQ, s.d, s.d, 128));
    WCHECK(tmap_bf16(&th, slab, hint.total_L, s.d, s.d, 128));
    const long long pw_rows = L.units_max * (kAbsRows / 64) * kAbsQ;  // tiled: [4 units_max * 256, 64]
    WCHECK(tmap_bf16_box(&tps, at(ws, L.pw), pw_rows, 64, 64, kAbsEpiCols, 32));
    if (E == 1) {
      CUCHECK(cudaFuncSetAttribute(abs_scores_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)AbsASmem<1>::BYTES));
      WCHECK(launch_pdl(abs_scores_kernel<1>, dim3(2 * a.n_pairs), dim3(kAbsAThreads), AbsASmem<1>::BYTES, st, tq, th,
                        tps, a));
    } else {
      CUCHECK(cudaFuncSetAttribute(abs_scores_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)AbsASmem<2>::BYTES));
      WCHECK(launch_pdl(abs_scores_kernel<2>, dim3(2 * a.n_pairs), dim3(kAbsAThreads), AbsASmem<2>::BYTES, st, tq, th,
                        tps, a));
    }
    CUtensorMap tpl, th64;
    WCHECK(tmap_bf16(&tpl, at(ws, L.pw), pw_rows, 64, 64, 128));
    WCHECK(tmap_bf16(&th64, slab, hint.total_L, s.d, s.d, 64));
    if (E == 1) {
      CUCHECK(cudaFuncSetAttribute(abs_values_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)AbsBSmem<1>::BYTES));
      WCHECK(launch_pdl(abs_values_kernel<1>, dim3(2 * a.n_pairs), dim3(kAbsBThreads), AbsBSmem<1>::BYTES, st, tpl,
                        th64, a));
    } else {
      CUCHECK(cudaFuncSetAttribute(abs_values_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)AbsBSmem<2>::BYTES));
      WCHECK(launch_pdl(abs_values_kernel<2>, dim3(2 * a.n_pairs), dim3(kAbsBThreads), AbsBSmem<2>::BYTES, st, tpl,
                        th64, a));
    }
  }
  WCHECK(launch_pdl(abs_merge_kernel, dim3(hint.B, kAbsQ / 8), dim3(256), 0, st, a));
  return gemm_vabs(s, at(ws, L.zh), wv, out, out_lo, rows, st);
}

// ------------------------------------------------------------------------------------------
// fp32 steps
// ------------------------------------------------------------------------------------------
whale_status row_rms(const float* x, long long rows, int d, float eps, float* r, cudaStream_t st) {
  if (rows <= 0) return WHALE_OK;
  row_rms_f32<<<(unsigned)cdiv<long long>(rows, 8), 256, 0, st>>>(x, d, rows, d, eps, r);
  CUCHECK(cudaGetLastError());
  return WHALE_OK;
}

whale_status gemm_f32(const float* A0, int K0, const float* A1, int K1, const float* rn, const float* gn,
                      const float* W, int N, float* C, long long M, int epi, const float* R, cudaStream_t st) {
  if (M <= 0) return WHALE_OK;
  const long long gy = cdiv<long long>(M, 64);
  if (gy > 65535) return WHALE_ERR_UNSUPPORTED;
  gemm_f32_kernel<<<dim3(cdiv(N, 64), (unsigned)gy), 256, 0, st>>>(A0, K0, K0, A1, K1, K1, rn, gn, W, C, N, M, N, epi,
                                                                    R, N);
  CUCHECK(cudaGetLastError());
  return WHALE_OK;
}

whale_status attention_f32(const Shape& s, const float* q, const float* kv, const int* offsets, float* a, int B,
                           long long total_L, cudaStream_t st) {
  const long long warps = (long long)B * s.N * s.h;
  if (warps == 0) return WHALE_OK;
  const unsigned grid = (unsigned)cdiv<long long>(warps, 4);
  const float scale = (float)(1.0 / std::sqrt((double)s.dh));
  const int v0 = s.shared_kv ? 0 : s.d;
#define ATT32(DH) attn_f32_kernel<DH><<<grid, 128, 0, st>>>(q, kv, s.kvw, v0, offsets, a, B, s.N, s.d, s.h, total_L, scale)
  switch (s.dh) {
    case 8: ATT32(8); break;
    case 16: ATT32(16); break;
    case 32: ATT32(32); break;
    case 64: ATT32(64); break;
    case 128: ATT32(128); break;
    default: return WHALE_ERR_UNSUPPORTED;
  }
#undef ATT32
  CUCHECK(cudaGetLastError());
  return WHALE_OK;
}

whale_status swiglu_f32(const Shape& s, const float* f, const float* gffn, const float* wug, const float* wdown,
                        float* y, long long rows, float* r, float* ug, float* u, cudaStream_t st) {
  WCHECK(row_rms(f, rows, s.d, s.eps, r, st));
  WCHECK(gemm_f32(f, s.d, nullptr, 0, r, gffn, wug, s.ugw, ug, rows, F32_NONE, nullptr, st));
  if (rows > 0) {
    swiglu_f32_kernel<<<(unsigned)cdiv<long long>(rows * s.H, 256), 256, 0, st>>>(ug, s.ugw, u, rows, s.H, s.tied);
    CUCHECK(cudaGetLastError());
  }
  return gemm_f32(u, s.H, nullptr, 0, nullptr, nullptr, wdown, s.d, y, rows, F32_RESID, f, st);
}

// fp32 Fusion MLP (correctness path).
whale_status fusion_mlp_f32(const Shape& s, long long rows, const float* a, const float* x, const float* wf1,
                            const float* wf2, float* f, float* gbuf, cudaStream_t st) {
  if (s.Fh > 0) {
    WCHECK(gemm_f32(a, s.d, x, s.d, nullptr, nullptr, wf1, s.Fh, gbuf, rows, F32_SILU, nullptr, st));
    return gemm_f32(gbuf, s.Fh, nullptr, 0, nullptr, nullptr, wf2, s.d, f, rows, F32_RESID, x, st);
  }
  return gemm_f32(a, s.d, x, s.d, nullptr, nullptr, wf2, s.d, f, rows, F32_RESID, x, st);
}

bool weights_ok(const Shape& s, const whale_layer_weights* w) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  const bool gains = s.prepared || (w && w->g_q && w->g_kv && w->g_ffn);
  return w && gains && w->w_q && w->w_kv && w->w_f2 && w->w_upgate && w->w_down &&
         (s.Fh == 0 || w->w_f1) && al(w->g_q) && al(w->g_kv) && al(w->g_ffn) && al(w->w_q) && al(w->w_kv) &&
         al(w->w_f1) && al(w->w_f2) && al(w->w_upgate) && al(w->w_down) && al(w->w_kabs);
}

// A token-side tensor of the bf16 path: fp32 value plus its bf16 hi/lo pair (any may be null
// for an output that is not needed).
struct Stream3 {
  float* f32;
  void* hi;
  void* lo;
};

// S4 + S5 of the bf16 path, shared by the layer and by the step entry points:
//   F = X + W_F2 SiLU(W_F1 [A ; X])  (or X + W_F [A ; X]);  Y = F + W_down (SiLU(gate) * up)
whale_status fusion_bf16(const Shape& s, long long rows, const Opnd& A, const Opnd& X, const float* x32,
                         const void* wf1, const void* wf2, void* g, void* g_lo, const Stream3& F, cudaStream_t st) {
  const Outs fo{F.hi, F.lo, F.f32, s.d};
  if (s.Fh > 0) {
    WCHECK(gemm_bf16(A, X, wf1, s.Fh, Outs{g, g_lo, nullptr, s.Fh}, nullptr, 0, rows, EPI_SILU, false, 0.f, st));
    return gemm_bf16(opnd(g, g_lo, s.Fh, s.Fh), no_opnd(), wf2, s.d, fo, x32, s.d, rows, EPI_RESID, false, 0.f, st);
  }
  return gemm_bf16(A, X, wf2, s.d, fo, x32, s.d, rows, EPI_RESID, false, 0.f, st);
}

whale_status ffn_bf16(const Shape& s, long long rows, const Opnd& F, const float* f32, const void* wug_folded,
                      const void* wdown, void* u, void* u_lo, const Stream3& Y, cudaStream_t st) {
  WCHECK(gemm_bf16(F, no_opnd(), wug_folded, s.ugw, Outs{u, u_lo, nullptr, s.H}, nullptr, 0, rows,
                   s.tied ? EPI_SWIGLU_TIED : EPI_SWIGLU, true, s.eps, st));
  return gemm_bf16(opnd(u, u_lo, s.H, s.H), no_opnd(), wdown, s.d, Outs{Y.hi, Y.lo, Y.f32, s.d}, f32, s.d, rows,
                   EPI_RESID, false, 0.f, st);
}

// One bf16 layer. `in` is the residual-stream tensor (f32, hi, lo all set), `out` receives
// H_f in the forms requested.
whale_status layer_bf16(const Shape& s, const Stream3& in, const void* slab, const int* offsets,
                        const whale_layer_weights& w, const Stream3& out, const whale_shape_hint& hint, void* ws,
                        const Layout& L, cudaStream_t st) {
  const long long rows = (long long)hint.B * s.N;
  const void* wq = w.w_q;
  const void* wkv = w.w_kv;
  const void* wug = w.w_upgate;
  const void* wkabs = s.absorbed ? w.w_kabs : nullptr;
  auto* wkabs_ws = reinterpret_cast<__nv_bfloat16*>(s.absorbed ? at(ws, L.wkabs) : nullptr);
  if (!s.prepared) {
    wq = at(ws, L.wq);
    wkv = at(ws, L.wkv);
    wug = at(ws, L.wug);
    wkabs = wkabs_ws;
    WCHECK(fold_weights(s, static_cast<const __nv_bfloat16*>(w.w_q), w.g_q, static_cast<const __nv_bfloat16*>(w.w_kv),
                        w.g_kv, static_cast<const __nv_bfloat16*>(w.w_upgate), w.g_ffn,
                        reinterpret_cast<__nv_bfloat16*>(at(ws, L.wq)), reinterpret_cast<__nv_bfloat16*>(at(ws, L.wkv)),
                        reinterpret_cast<__nv_bfloat16*>(at(ws, L.wug)), st,
                        s.absorbed ? static_cast<const __nv_bfloat16*>(w.w_kv) : nullptr, w.g_kv, wkabs_ws));
  } else if (s.absorbed && !wkabs) {  // prepared weights without the absorbed keys: form them from W_K'
    wkabs = wkabs_ws;
    WCHECK(fold_weights(s, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, st,
                        static_cast<const __nv_bfloat16*>(w.w_kv), nullptr, wkabs_ws));
  }
  const Opnd X = opnd(in.hi, in.lo, s.d, s.d);
  // S1 queries
  WCHECK(gemm_bf16(X, no_opnd(), wq, s.d, Outs{at(ws, L.q), nullptr, nullptr, s.d}, nullptr, 0, rows, EPI_STORE, true,
                   s.eps, st));
  if (s.absorbed) {
    // S2 + S3 with K and V folded into the queries -> A as a hi/lo pair
    const void* wv = s.shared_kv ? wkv : static_cast<const char*>(wkv) + (size_t)s.d * s.d * 2;
    WCHECK(attention_absorbed(s, at(ws, L.q), slab, offsets, wkabs, wv, at(ws, L.a), at(ws, L.a_lo), hint, ws, L,
                              st));
  } else {
    // S2 keys|values, S3 attention -> A as a hi/lo pair
    WCHECK(gemm_bf16(opnd(slab, nullptr, s.d, s.d), no_opnd(), wkv, s.kvw,
                     Outs{at(ws, L.kv), nullptr, nullptr, s.kvw}, nullptr, 0, hint.total_L, EPI_STORE, true, s.eps, st));
    WCHECK(attention_bf16(s, at(ws, L.q), at(ws, L.kv), offsets, at(ws, L.a), at(ws, L.a_lo), hint.B, hint.total_L,
                          at(ws, L.po), st));
  }
  // S4 Fusion MLP -> F (fp32 + pair)
  auto* f32 = reinterpret_cast<float*>(at(ws, L.f32));
  WCHECK(fusion_bf16(s, rows, opnd(at(ws, L.a), at(ws, L.a_lo), s.d, s.d), X, in.f32, w.w_f1, w.w_f2, at(ws, L.g),
                     at(ws, L.g_lo), Stream3{f32, at(ws, L.f), at(ws, L.f_lo)}, st));
  // S5 SwiGLU FFN -> H_f
  return ffn_bf16(s, rows, opnd(at(ws, L.f), at(ws, L.f_lo), s.d, s.d), f32, wug, w.w_down, at(ws, L.u),
                  at(ws, L.u_lo), out, st);
}

// One fp32 layer (SIMT correctness path).
whale_status layer_f32(const Shape& s, const void* x_in, const void* slab, const int* offsets,
                       const whale_layer_weights& w, void* x_out, const whale_shape_hint& hint, void* ws,
                       const Layout& L, cudaStream_t st) {
  const long long rows = (long long)hint.B * s.N;
  auto F = [&](size_t off) { return reinterpret_cast<float*>(at(ws, off)); };
  const float* xf = static_cast<const float*>(x_in);
  const float* sf = static_cast<const float*>(slab);
  WCHECK(row_rms(xf, rows, s.d, s.eps, F(L.r), st));
  WCHECK(gemm_f32(xf, s.d, nullptr, 0, F(L.r), w.g_q, static_cast<const float*>(w.w_q), s.d, F(L.q), rows, F32_NONE,
                  nullptr, st));
  WCHECK(row_rms(sf, hint.total_L, s.d, s.eps, F(L.r), st));
  WCHECK(gemm_f32(sf, s.d, nullptr, 0, F(L.r), w.g_kv, static_cast<const float*>(w.w_kv), s.kvw, F(L.kv),
                  hint.total_L, F32_NONE, nullptr, st));
  WCHECK(attention_f32(s, F(L.q), F(L.kv), offsets, F(L.a), hint.B, hint.total_L, st));
  WCHECK(fusion_mlp_f32(s, rows, F(L.a), xf, static_cast<const float*>(w.w_f1), static_cast<const float*>(w.w_f2),
                        F(L.f), F(L.g), st));
  return swiglu_f32(s, F(L.f), w.g_ffn, static_cast<const float*>(w.w_upgate), static_cast<const float*>(w.w_down),
                    static_cast<float*>(x_out), rows, F(L.r), F(L.ug), F(L.u), st);
}

// The stack over device buffers: tokens (layer-0 H_w) -> out (last H_f).
// `hook(l, before)` (optional) runs on the host before and after layer l is enqueued.
using LayerHook = std::function<whale_status(int, bool)>;
whale_status stack_impl(const Shape& s, const void* tokens, const void* seq_states, const int* offsets,
                        const whale_layer_weights* weights, int first_layer, int n_layers, void* out,
                        const whale_shape_hint& hint, void* ws, const Layout& L, cudaStream_t st,
                        const void* const* slabs /* per layer, or null: seq_states + l * slab */,
                        const LayerHook& hook = nullptr) {
  const size_t slab_bytes = (size_t)hint.total_L * s.d * s.es;
  auto slab_of = [&](int l) -> const void* {
    if (slabs) return slabs[l];
    return seq_states ? static_cast<const char*>(seq_states) + (size_t)(first_layer + l) * slab_bytes : nullptr;
  };
  const long long rows = (long long)hint.B * s.N;
  if (!s.bf16) {
    const void* x = tokens;
    for (int l = 0; l < n_layers; ++l) {
      char name[32];
      snprintf(name, sizeof name, "whale layer %d", first_layer + l);
      NvtxRange range(name);
      void* y = (l == n_layers - 1) ? out : at(ws, (l & 1) ? L.x1 : L.x0);
      if (hook) WCHECK(hook(l, true));
      WCHECK(layer_f32(s, x, slab_of(l), offsets, weights[first_layer + l], y, hint, ws, L, st));
      if (hook) WCHECK(hook(l, false));
      x = y;
    }
    return WHALE_OK;
  }
  auto buf = [&](int i) {
    return Stream3{reinterpret_cast<float*>(at(ws, L.x32[i])), at(ws, L.xhi[i]), at(ws, L.xlo[i])};
  };
  Stream3 in = buf(0);
  in.hi = const_cast<void*>(tokens);  // bf16 tokens are their own hi half; lo = 0
  WCHECK(pair_from_bf16(tokens, in.f32, in.lo, rows * s.d, st));
  WCHECK(abs_units(s, offsets, hint, ws, L, st));
  for (int l = 0; l < n_layers; ++l) {
    char name[32];
    snprintf(name, sizeof name, "whale layer %d", first_layer + l);
    NvtxRange range(name);
    const Stream3 y = (l == n_layers - 1) ? Stream3{nullptr, out, nullptr} : buf((l + 1) & 1);
    if (hook) WCHECK(hook(l, true));
    WCHECK(layer_bf16(s, in, slab_of(l), offsets, weights[first_layer + l], y, hint, ws, L, st));
    if (hook) WCHECK(hook(l, false));
    in = y;
  }
  return WHALE_OK;
}

whale_status common_checks(const whale_config* cfg, const whale_shape_hint* hint, Shape* s, void* ws, size_t ws_bytes,
                           Layout* L) {
  WCHECK(validate(cfg, s));
  WCHECK(check_hint(hint));
  *L = make_layout(*s, *hint);
  if (!ws || ws_bytes < L->total || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return WHALE_ERR_WORKSPACE;
  return WHALE_OK;
}


whale_status debug_check(const Shape& s, const int* offsets, const whale_shape_hint& hint, cudaStream_t st) {
  if (!s.debug) return WHALE_OK;
  check_offsets_kernel<<<cdiv(hint.B + 1, 256), 256, 0, st>>>(offsets, hint.B, hint.max_L, hint.total_L);
  CUCHECK(cudaGetLastError());
  return WHALE_OK;
}

// Per-device copy stream and events of the host-buffer forward (created once, kept). A call holds
// `mu` while it enqueues: each of its waits must see its own event records, not another call's
// recorded in between on another stream (a copy into a staging buffer would then not wait for the
// layer of its own call that still reads that buffer).
struct HostPipe {
  cudaStream_t copy = nullptr;
  cudaEvent_t copied[2] = {nullptr, nullptr}, consumed[2] = {nullptr, nullptr};
  std::mutex mu;
};
std::mutex g_pipe_mu;
HostPipe g_pipes[64];

whale_status host_pipe(HostPipe** out) {
  int dev = 0;
  CUCHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return WHALE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_pipe_mu);
  HostPipe& p = g_pipes[dev];
  if (!p.copy) {
    CUCHECK(cudaStreamCreateWithFlags(&p.copy, cudaStreamNonBlocking));
    for (int i = 0; i < 2; ++i) {
      CUCHECK(cudaEventCreateWithFlags(&p.copied[i], cudaEventDisableTiming));
      CUCHECK(cudaEventCreateWithFlags(&p.consumed[i], cudaEventDisableTiming));
    }
  }
  *out = &p;
  return WHALE_OK;
}

size_t host_staging_bytes(const Shape& s, const whale_shape_hint& h, size_t* o_tok, size_t* o_slab0, size_t* o_slab1,
                          size_t* o_off, size_t* o_out) {
  const size_t rows = (size_t)h.B * s.N;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t a = o;
    o = align_up(o + bytes);
    return a;
  };
  *o_tok = take(rows * s.d * s.es);
  *o_slab0 = take((size_t)h.total_L * s.d * s.es);
  *o_slab1 = take((size_t)h.total_L * s.d * s.es);
  *o_off = take(((size_t)h.B + 1) * 4);
  *o_out = take(rows * s.d * s.es);
  return o;
}

// ============================================================================================
// Backward pass of one fusion layer (the vector-Jacobian product for dY = dLoss/dH_f): the forward
// is recomputed (materialised K|V path, with the softmax log-sum-exp kept), then its steps are
// reversed. bf16 mode: tcgen05 GEMMs (MN-major operands for the untransposed weights and for the
// weight gradients, which contract over token or history rows; split-K where the output is small),
// the KV-parallel tensor-core attention backward, fused element-wise and RMSNorm-backward row
// kernels. fp32 mode: the same steps with SIMT kernels.
// ============================================================================================
constexpr int kColpBlocks = 8 * kNumSM;  // row-kernel blocks (column partials of the gain gradients)

inline int rows_blocks(long long rows) {
  return (int)std::max<long long>(1, std::min<long long>(cdiv<long long>(rows, 32), kColpBlocks));
}

// out = r(x) (x W^T) as a bf16 pair, W given as a pair (w_hi + w_lo, [N, K] K-major), x bf16 [M, K]
// (row stride K); r = 1/sqrt(mean(x^2) + eps) per row, also written to rows_r. Two MMAs per k-step.
whale_status gemm_rownorm_wpair(const void* x, long long M, int K, const void* w_hi, const void* w_lo, int N,
                                void* out_hi, void* out_lo, float* rows_r, float eps, cudaStream_t st) {
  if (M <= 0) return WHALE_OK;
  if (M >= (1ll << 31) || K % 64 || N % 64) return WHALE_ERR_UNSUPPORTED;
  const int bn = N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : 64);
  CUtensorMap maps[8];
  WCHECK(tmap_bf16(&maps[0], x, M, K, K, 128));
  maps[1] = maps[0];
  WCHECK(tmap_bf16(&maps[2], w_lo, N, K, K, bn));  // B's lo half rides in the A1 slot
  maps[3] = maps[2];
  WCHECK(tmap_bf16(&maps[4], w_hi, N, K, K, bn));
  GemmArgs g{};
  g.M = (int)M;
  g.N = N;
  g.kb0 = K / 64;
  g.kb1 = 0;
  g.tiles_n = N / bn;
  const long long tiles = cdiv<long long>(M, 128) * g.tiles_n;
  g.num_tiles = (int)tiles;
  g.inv_k = 1.0f / (float)K;
  g.eps = eps;
  g.out_hi = static_cast<__nv_bfloat16*>(out_hi);
  g.out_lo = static_cast<__nv_bfloat16*>(out_lo);
  g.ldo = N;
  g.rows_r = rows_r;
  WCHECK(epi_maps(maps + 5, g, N, 1, maps[0]));
  if (bn == 256) return launch_gemm_t<256, EPI_STORE, true, false, false, false, true>(maps, g, tiles, st);
  if (bn == 128) return launch_gemm_t<128, EPI_STORE, true, false, false, false, true>(maps, g, tiles, st);
  return launch_gemm_t<64, EPI_STORE, true, false, false, false, true>(maps, g, tiles, st);
}

struct BwdBufs {
  // forward recompute
  void *x32, *xlo, *r, *q, *q_lo, *sn, *wg, *wg_lo, *rkv, *kv, *kv_lo, *attn, *a, *a_lo, *lse, *z1, *g, *g_lo, *f32,
      *f, *f_lo, *ug;
  // backward
  void *dy, *dy_lo, *dm, *msw, *msw_lo, *dug, *dug_lo, *dn, *nrm, *nrm_lo, *nq, *nq_lo, *df32, *df, *df_lo, *dhid,
      *dz, *dz_lo, *dc, *da16, *da_lo, *delta, *dq, *dq_hi, *dq_lo, *cst, *dkv, *dkv_lo, *dsn, *colp, *part;
  size_t part_floats;
};

// The forward activations one layer's backward reads (bf16 mode): q and its normalised rows, K|V and
// the history rows' factors, A and its log-sum-exp, z1 and G, F, UG and the FFN's normalised rows.
// The stack backward keeps one set per layer so that each layer's forward runs once.
template <typename Take>
void act_buffers(const Shape& s, const whale_shape_hint& h, Take take, BwdBufs* b) {
  const size_t rows = (size_t)h.B * s.N, T = (size_t)h.total_L, d = s.d, Fh = s.Fh;
  b->lse = take(rows * s.h * 4);
  b->nq = take(rows * d * 2);
  b->nq_lo = take(rows * d * 2);
  b->q = take(rows * d * 2);
  b->q_lo = take(rows * d * 2);
  b->kv = take(T * s.kvw * 2);
  b->kv_lo = take(T * s.kvw * 2);
  b->rkv = take(T * 4);
  b->a = take(rows * d * 2);
  b->a_lo = take(rows * d * 2);
  if (Fh) {
    b->z1 = take(rows * Fh * 4);
    b->g = take(rows * Fh * 2);
    b->g_lo = take(rows * Fh * 2);
  }
  b->f32 = take(rows * d * 4);
  b->f = take(rows * d * 2);
  b->f_lo = take(rows * d * 2);
  b->ug = take(rows * s.ugw * 4);
  b->nrm = take(rows * d * 2);
  b->nrm_lo = take(rows * d * 2);
}

// Buffers of the backward workspace (null pointers when base is null); returns its size in bytes.
size_t bwd_buffers(const Shape& s, const whale_shape_hint& h, char* base, BwdBufs* b) {
  size_t o = 0;
  auto take = [&](size_t bytes) -> void* {
    void* p = base ? base + o : nullptr;
    o = align_up(o + bytes);
    return p;
  };
  const size_t rows = (size_t)h.B * s.N, T = (size_t)h.total_L, d = s.d, H = s.H, Fh = s.Fh;
  const size_t ugw = s.ugw, kvw = s.kvw, nh = s.h;
  const size_t e = s.bf16 ? 2 : 4;  // element size of the operand copies
  *b = BwdBufs{};
  if (s.bf16) {
    act_buffers(s, h, take, b);
    b->x32 = take(rows * d * 4);
    b->xlo = take(rows * d * 2);
    b->attn = take(plan_attention(s, h.B, h.total_L).bytes());
    b->wg = take(kvw * d * 2);  // W_kv diag(g_kv) as a pair
    b->wg_lo = take(kvw * d * 2);
  } else {
    b->r = take(std::max(rows, T) * 4);
    b->q = take(rows * d * 4);
    b->kv = take(T * kvw * 4);
    b->sn = take(T * d * 4);
    b->a = take(rows * d * 4);
    if (Fh) {
      b->z1 = take(rows * Fh * 4);
      b->g = take(rows * Fh * 4);
    }
    b->f32 = take(rows * d * 4);
    b->ug = take(rows * ugw * 4);
    b->nrm = take(rows * d * 4);
  }
  if (s.bf16) {
    b->dy = take(rows * d * 2);
    b->dy_lo = take(rows * d * 2);
  }
  b->dm = take(rows * H * 4);
  b->msw = take(rows * H * e);
  if (s.bf16) b->msw_lo = take(rows * H * 2);
  b->dug = take(rows * ugw * e);
  if (s.bf16) b->dug_lo = take(rows * ugw * 2);
  b->dn = take(rows * d * 4);
  b->df32 = take(rows * d * 4);
  if (s.bf16) {
    b->df = take(rows * d * 2);
    b->df_lo = take(rows * d * 2);
  }
  if (Fh) {
    b->dhid = take(rows * Fh * 4);
    b->dz = take(rows * Fh * e);
    if (s.bf16) b->dz_lo = take(rows * Fh * 2);
  }
  b->dc = take(rows * 2 * d * 4);
  if (s.bf16) {
    b->da16 = take(rows * d * 2);
    b->da_lo = take(rows * d * 2);
    b->delta = take(rows * nh * 4);
    b->dq_hi = take(rows * d * 2);
    b->dq_lo = take(rows * d * 2);
    b->cst = take(((size_t)h.B + 1) * 4);
  }
  b->dq = take(rows * d * 4);
  b->dkv = take(T * kvw * e);
  if (s.bf16) b->dkv_lo = take(T * kvw * 2);
  b->dsn = take(T * d * 4);
  b->colp = take((size_t)kColpBlocks * d * 4);
  const size_t mn = std::max({d * H, ugw * d, d * std::max(Fh, d), kvw * d});
  b->part_floats = s.bf16 ? 16 * mn : 0;
  b->part = s.bf16 ? take(b->part_floats * 4) : nullptr;
  return o;
}

// Gain gradient: the row kernel's column partials summed in block order.
whale_status gain_grad(const float* colp, int blocks, int d, float* dg, cudaStream_t st) {
  if (!dg) return WHALE_OK;
  return launch_pdl(col_sums_kernel, dim3((unsigned)cdiv(d, 32)), dim3(256), 0, st, colp, blocks, d, dg);
}

template <typename TX>
whale_status rms_bwd(const TX* x, const float* g, const float* dn, long long rows, int d, float eps,
                     const float* r1, long long ld1, const float* r2, long long ld2, float* dx32, void* dx_hi,
                     void* dx_lo, void* n_out, void* n_lo, float* n32, float* colp, float* dg, cudaStream_t st,
                     bool pre = false) {
  if (rows <= 0) {
    if (dg) CUCHECK(cudaMemsetAsync(dg, 0, (size_t)d * 4, st));
    return WHALE_OK;
  }
  const int blocks = rows_blocks(rows);
  auto go = [&](auto kern) {
    return launch_pdl(kern, dim3(blocks), dim3(256), 0, st, x, g, dn, rows, d, eps, r1, ld1, r2, ld2, dx32,
                      static_cast<__nv_bfloat16*>(dx_hi), static_cast<__nv_bfloat16*>(dx_lo),
                      static_cast<__nv_bfloat16*>(n_out), static_cast<__nv_bfloat16*>(n_lo), n32, colp);
  };
  if (pre) {
    if (d <= 256) WCHECK(go(rms_bwd_kernel<TX, 1, true>));
    else if (d <= 512) WCHECK(go(rms_bwd_kernel<TX, 2, true>));
    else WCHECK(go(rms_bwd_kernel<TX, 4, true>));
  } else {
    if (d <= 256) WCHECK(go(rms_bwd_kernel<TX, 1>));
    else if (d <= 512) WCHECK(go(rms_bwd_kernel<TX, 2>));
    else WCHECK(go(rms_bwd_kernel<TX, 4>));
  }
  return gain_grad(colp, blocks, d, dg, st);
}

template <typename F, typename... A>
whale_status ew_launch(F kern, long long n, cudaStream_t st, A... args) {
  if (n <= 0) return WHALE_OK;
  const unsigned grid = (unsigned)std::min<long long>(cdiv<long long>(n, 256), 8 * kNumSM);
  return launch_pdl(kern, dim3(grid), dim3(256), 0, st, args...);
}
// The same for the kernels that take 8 elements per thread and step (n elements in all).
template <typename F, typename... A>
whale_status ew8_launch(F kern, long long n, cudaStream_t st, A... args) {
  return ew_launch(kern, cdiv<long long>(n, 8), st, args...);
}

template <int DH, int NQ>
whale_status launch_attn_bwd(const AttnBwdArgs& a, unsigned chunks, cudaStream_t st) {
  using C = AttnBwdCfg<DH, NQ>;
  if (a.n_heads % C::HG) return WHALE_ERR_UNSUPPORTED;
  CUCHECK(cudaFuncSetAttribute(attn_bwd_kernel<DH, NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES));
  return launch_pdl(attn_bwd_kernel<DH, NQ>, dim3(chunks, a.n_heads / C::HG), dim3(C::THREADS), C::BYTES, st, a);
}

// The tensor-core attention backward (d_h = 64, N <= 32): one CTA per (chunk, head); K|V, q, dA
// (all bf16 pairs) read through tensor maps.
whale_status launch_attn_bwd_tc(const AttnBwdArgs& a, unsigned chunks, cudaStream_t st) {
  if (a.d % 64 || a.N > 32 || a.N < 1 || a.kvw % 64 || a.total_L <= 0) return WHALE_ERR_UNSUPPORTED;
  const long long rows = (long long)a.B * a.N;
  CUtensorMap m[8];
  WCHECK(tmap_bf16(&m[0], a.kv, a.total_L, a.kvw, a.kvw, 128));
  WCHECK(tmap_bf16(&m[1], a.kv_lo, a.total_L, a.kvw, a.kvw, 128));
  WCHECK(tmap_bf16(&m[2], a.q, rows, a.d, a.d, 32));
  WCHECK(tmap_bf16(&m[3], a.q_lo, rows, a.d, a.d, 32));
  WCHECK(tmap_bf16(&m[4], a.da, rows, a.d, a.d, 32));
  WCHECK(tmap_bf16(&m[5], a.da_lo, rows, a.d, a.d, 32));
  WCHECK(tmap_bf16(&m[6], a.dkv, a.total_L, a.kvw, a.kvw, 32));
  WCHECK(tmap_bf16(&m[7], a.dkv_lo, a.total_L, a.kvw, a.kvw, 32));
  CUCHECK(cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)AttnBwdTcSmem::BYTES));
  return launch_pdl(attn_bwd_tc_kernel, dim3(chunks, a.n_heads), dim3(kAttnBwdTcThreads), AttnBwdTcSmem::BYTES, st,
                    m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], a);
}

// Shapes the backward pass supports: bf16 with at most 32 queries per example (the KV-parallel
// attention backward keeps all of an example's queries resident), d a multiple of 128 (its head
// groups span 128 columns) and d <= 1024 (row kernels); fp32 with d_head <= 64. The SwiGLU backward
// takes 8 hidden columns per thread: ffn_hidden a multiple of 8.
bool backward_shape_ok(const Shape& s) {
  if (s.d > 1024 || s.d % 32 || s.H % 8) return false;
  if (s.bf16) return s.N <= 32 && (s.dh == 32 || s.dh == 64) && s.d % 128 == 0;
  return s.dh == 8 || s.dh == 16 || s.dh == 32 || s.dh == 64;
}

// The forward of one layer in bf16 mode as the backward pass recomputes it, into the backward buffers
// (q, K|V, A and its log-sum-exp, z1, G, F, UG). The layer input is a residual-stream tensor `in`:
// fp32 plus its bf16 hi/lo pair (a layer of the stack gets its exact input, the layer entry point its
// bf16 tokens with lo = 0).
whale_status recompute_bf16(const Shape& s, const Stream3& in, const void* slab, const int* offsets,
                            const whale_layer_weights& w, const whale_shape_hint& h, const BwdBufs& b,
                            cudaStream_t st) {
  using bf = __nv_bfloat16;
  const long long rows = (long long)h.B * s.N, T = h.total_L;
  const int d = s.d, Fh = s.Fh, ugw = s.ugw, kvw = s.kvw;
  auto F = [](void* p) { return static_cast<float*>(p); };
  const float* x32 = in.f32;
  const Opnd X = opnd(in.hi, in.lo, d, d);
  // Token side: the normalised rows n = r x g as a hi/lo pair times the raw (exact) weights; folding g
  // into a bf16 weight would round every product's weight by up to 2^-9, an error the weight
  // gradients (sums over rows) would carry.
  WCHECK(launch_pdl(rms_rows_kernel<float>, dim3(rows_blocks(rows)), dim3(256), 0, st, x32, w.g_q, rows, d, s.eps,
                    static_cast<bf*>(b.nq), static_cast<bf*>(b.nq_lo), (float*)nullptr));
  WCHECK(gemm_bf16(opnd(b.nq, b.nq_lo, d, d), no_opnd(), w.w_q, d, Outs{b.q, b.q_lo, nullptr, d}, nullptr, 0, rows,
                   EPI_STORE, false, 0.f, st));
  // History side: K|V = r (s (W_kv diag(g))^T) with the raw states s (exact bf16) times W_kv diag(g) as
  // a pair, the row factor r in the epilogue (and kept for the backward), written as a pair (the
  // attention backward reads both halves; the forward attention below reads hi).
  if (T > 0) {
    WCHECK(ew_launch(scale_cols_pair_kernel, (long long)kvw * d, st, static_cast<const bf*>(w.w_kv), w.g_kv,
                     (long long)kvw, d, static_cast<bf*>(b.wg), static_cast<bf*>(b.wg_lo)));
    WCHECK(gemm_rownorm_wpair(slab, T, d, b.wg, b.wg_lo, kvw, b.kv, b.kv_lo, F(b.rkv), s.eps, st));
  }
  WCHECK(attention_bf16(s, b.q, b.kv, offsets, b.a, b.a_lo, h.B, T, b.attn, st, F(b.lse)));
  const Opnd A = opnd(b.a, b.a_lo, d, d);
  if (Fh > 0) {
    WCHECK(gemm_bf16(A, X, w.w_f1, Fh, Outs{nullptr, nullptr, F(b.z1), Fh}, nullptr, 0, rows, EPI_STORE, false, 0.f,
                     st));
    WCHECK(ew8_launch(silu_pair_kernel, rows * Fh, st, (const float*)F(b.z1), (float*)nullptr, static_cast<bf*>(b.g),
                     static_cast<bf*>(b.g_lo), rows * Fh));
    WCHECK(gemm_bf16(opnd(b.g, b.g_lo, Fh, Fh), no_opnd(), w.w_f2, d, Outs{b.f, b.f_lo, F(b.f32), d}, x32, d,
                     rows, EPI_RESID, false, 0.f, st));
  } else {
    WCHECK(gemm_bf16(A, X, w.w_f2, d, Outs{b.f, b.f_lo, F(b.f32), d}, x32, d, rows, EPI_RESID, false, 0.f, st));
  }
  WCHECK(launch_pdl(rms_rows_kernel<float>, dim3(rows_blocks(rows)), dim3(256), 0, st, (const float*)F(b.f32),
                    w.g_ffn, rows, d, s.eps, static_cast<bf*>(b.nrm), static_cast<bf*>(b.nrm_lo), (float*)nullptr));
  return gemm_bf16(opnd(b.nrm, b.nrm_lo, d, d), no_opnd(), w.w_upgate, ugw, Outs{nullptr, nullptr, F(b.ug), ugw},
                   nullptr, 0, rows, EPI_STORE, false, 0.f, st);
}

// The layer's output from the recomputed intermediates: H_f = F + W_down (SiLU(gate) * up), as a
// residual-stream tensor (fp32 and its pair): the next layer's input in the stack backward.
whale_status layer_output_bf16(const Shape& s, const whale_layer_weights& w, const whale_shape_hint& h,
                               const BwdBufs& b, const Stream3& out, cudaStream_t st) {
  using bf = __nv_bfloat16;
  const long long rows = (long long)h.B * s.N;
  WCHECK(ew_launch(swiglu_pair_kernel, rows * s.H, st, (const float*)static_cast<float*>(b.ug), rows, s.H,
                   s.tied ? 1 : 0, static_cast<bf*>(b.msw), static_cast<bf*>(b.msw_lo)));
  return gemm_bf16(opnd(b.msw, b.msw_lo, s.H, s.H), no_opnd(), w.w_down, s.d, Outs{out.hi, out.lo, out.f32, s.d},
                   static_cast<const float*>(b.f32), s.d, rows, EPI_RESID, false, 0.f, st);
}

// One layer's backward in bf16 mode (input as for recompute_bf16). With recompute false the forward
// activations in b are those of this layer's input already (the stack backward's forward loop).
whale_status layer_backward_bf16(const Shape& s, const Stream3& in, const void* slab, const int* offsets,
                                 const whale_layer_weights& w, const float* dy, float* dx, void* ds,
                                 const whale_layer_grads& gr, const whale_shape_hint& h, const BwdBufs& b,
                                 cudaStream_t st, bool recompute = true) {
  using bf = __nv_bfloat16;
  const long long rows = (long long)h.B * s.N, T = h.total_L;
  const int d = s.d, H = s.H, Fh = s.Fh, ugw = s.ugw, kvw = s.kvw;
  auto F = [](void* p) { return static_cast<float*>(p); };
  const void* x = in.hi;
  const float* x32 = in.f32;
  if (recompute) WCHECK(recompute_bf16(s, in, slab, offsets, w, h, b, st));
  // ---- S5 backward: SwiGLU FFN ----
  float* part = F(b.part);
  const size_t pc = b.part_floats;
  WCHECK(ew8_launch(split_pair_kernel, rows * d, st, dy, (long long)d, static_cast<bf*>(b.dy), static_cast<bf*>(b.dy_lo),
                   (long long)d, rows, d));
  WCHECK(gemm_acc32(b.dy, b.dy_lo, d, false, w.w_down, H, true, rows, H, d, F(b.dm), H, part, pc, st));
  WCHECK(ew8_launch(swiglu_bwd_kernel, rows * H, st, (const float*)F(b.ug), (const float*)F(b.dm), rows, H,
                   s.tied ? 1 : 0, static_cast<bf*>(b.msw), static_cast<bf*>(b.msw_lo), (float*)nullptr,
                   (float*)nullptr, static_cast<bf*>(b.dug), static_cast<bf*>(b.dug_lo)));
  // token-side weight gradients: both operands as hi/lo pairs (their sums over rows cancel)
  WCHECK(gemm_acc32(b.dy, b.dy_lo, d, true, b.msw, H, true, d, H, rows, gr.w_down, H, part, pc, st, b.msw_lo));
  WCHECK(gemm_acc32(b.dug, b.dug_lo, ugw, false, w.w_upgate, d, true, rows, d, ugw, F(b.dn), d, part, pc, st));
  WCHECK(rms_bwd<float>(F(b.f32), w.g_ffn, F(b.dn), rows, d, s.eps, dy, d, nullptr, 0, F(b.df32), b.df, b.df_lo,
                        nullptr, nullptr, nullptr, F(b.colp), gr.g_ffn, st));
  WCHECK(gemm_acc32(b.dug, b.dug_lo, ugw, true, b.nrm, d, true, ugw, d, rows, gr.w_upgate, d, part, pc, st, b.nrm_lo));
  // ---- S4 backward: Fusion MLP (dc = d[A | H_w]) ----
  if (Fh > 0) {
    WCHECK(gemm_acc32(b.df, b.df_lo, d, false, w.w_f2, Fh, true, rows, Fh, d, F(b.dhid), Fh, part, pc, st));
    WCHECK(ew8_launch(silu_bwd_kernel, rows * Fh, st, (const float*)F(b.dhid), (const float*)F(b.z1), (float*)nullptr,
                     static_cast<bf*>(b.dz), static_cast<bf*>(b.dz_lo), rows * Fh));
    WCHECK(gemm_acc32(b.df, b.df_lo, d, true, b.g, Fh, true, d, Fh, rows, gr.w_f2, Fh, part, pc, st, b.g_lo));
    WCHECK(gemm_acc32(b.dz, b.dz_lo, Fh, false, w.w_f1, 2 * d, true, rows, 2 * d, Fh, F(b.dc), 2 * d, part, pc, st));
    WCHECK(gemm_acc32(b.dz, b.dz_lo, Fh, true, b.a, d, true, Fh, d, rows, gr.w_f1, 2 * d, part, pc, st, b.a_lo));
    WCHECK(gemm_acc32(b.dz, b.dz_lo, Fh, true, x, d, true, Fh, d, rows, gr.w_f1 + d, 2 * d, part, pc, st, in.lo));
  } else {
    WCHECK(gemm_acc32(b.df, b.df_lo, d, false, w.w_f2, 2 * d, true, rows, 2 * d, d, F(b.dc), 2 * d, part, pc, st));
    WCHECK(gemm_acc32(b.df, b.df_lo, d, true, b.a, d, true, d, d, rows, gr.w_f2, 2 * d, part, pc, st, b.a_lo));
    WCHECK(gemm_acc32(b.df, b.df_lo, d, true, x, d, true, d, d, rows, gr.w_f2 + d, 2 * d, part, pc, st, in.lo));
  }
  // ---- S3 backward: attention (KV-parallel) ----
  WCHECK(ew8_launch(attn_bwd_prep_kernel, rows * d, st, (const float*)F(b.dc), (long long)(2 * d),
                   (const bf*)b.a, (const bf*)b.a_lo, rows, d, s.h, F(b.delta), static_cast<bf*>(b.da16),
                   static_cast<bf*>(b.da_lo)));
  CUCHECK(cudaMemsetAsync(b.dq, 0, (size_t)rows * d * 4, st));
  if (T > 0) {
    const int chunk = s.dh == 64 ? kBwdChunkTc : kBwdChunk;
    const long long cmax = cdiv<long long>(T, chunk) + h.B;
    if (cmax >= (1ll << 31)) return WHALE_ERR_UNSUPPORTED;
    WCHECK(ew_launch(zero_tail_rows_kernel<bf>, T * kvw, st, offsets, h.B, T, kvw, static_cast<bf*>(b.dkv),
                     static_cast<bf*>(b.dkv_lo)));
    WCHECK(launch_pdl(chunk_starts_kernel, dim3(1), dim3(1024), 0, st, offsets, h.B, T, chunk, (int)cmax,
                      static_cast<int*>(b.cst)));
    AttnBwdArgs aa{};
    aa.q = static_cast<const bf*>(b.q);
    aa.q_lo = static_cast<const bf*>(b.q_lo);
    aa.kv = static_cast<const bf*>(b.kv);
    aa.kv_lo = static_cast<const bf*>(b.kv_lo);
    aa.da = static_cast<const bf*>(b.da16);
    aa.da_lo = static_cast<const bf*>(b.da_lo);
    aa.dkv_lo = static_cast<bf*>(b.dkv_lo);
    aa.lse = F(b.lse);
    aa.delta = F(b.delta);
    aa.offsets = offsets;
    aa.cstart = static_cast<const int*>(b.cst);
    aa.chunk = chunk;
    aa.dq = F(b.dq);
    aa.dkv = static_cast<bf*>(b.dkv);
    aa.row_scale = F(b.rkv);  // dK|V' = r dK|V: what both history-side products below contract with
    aa.B = h.B;
    aa.N = s.N;
    aa.d = d;
    aa.n_heads = s.h;
    aa.kvw = kvw;
    aa.v_col0 = s.shared_kv ? 0 : d;
    aa.shared_kv = s.shared_kv ? 1 : 0;
    aa.total_L = T;
    aa.scale = (float)(1.0 / std::sqrt((double)s.dh));
    aa.scale_log2 = scale_log2_of(s);
    whale_status r;
    if (s.dh == 64) r = launch_attn_bwd_tc(aa, (unsigned)cmax, st);
    else r = s.N <= 16 ? launch_attn_bwd<32, 16>(aa, (unsigned)cmax, st) : launch_attn_bwd<32, 32>(aa, (unsigned)cmax, st);
    WCHECK(r);
  }
  // ---- S1 backward: query projection and its RMSNorm; d_tokens ----
  WCHECK(ew8_launch(split_pair_kernel, rows * d, st, (const float*)F(b.dq), (long long)d, static_cast<bf*>(b.dq_hi),
                   static_cast<bf*>(b.dq_lo), (long long)d, rows, d));
  WCHECK(gemm_acc32(b.dq_hi, b.dq_lo, d, false, w.w_q, d, true, rows, d, d, F(b.dn), d, part, pc, st));
  WCHECK(gemm_acc32(b.dq_hi, b.dq_lo, d, true, b.nq, d, true, d, d, rows, gr.w_q, d, part, pc, st, b.nq_lo));
  WCHECK(rms_bwd<float>(x32, w.g_q, F(b.dn), rows, d, s.eps, F(b.df32), d, F(b.dc) + d, 2 * d, dx, nullptr, nullptr,
                        nullptr, nullptr, nullptr, F(b.colp), gr.g_q, st));
  // ---- S2 backward: K|V projection and the states' RMSNorm ----
  // With dK|V' = r dK|V (rows scaled by the attention backward): dsn' = dK|V' W_kv = r dsn feeds the
  // RMSNorm backward in its prescaled form, and dW_kv = dK|V^T (r s g) = (dK|V'^T s) diag(g) contracts
  // with the raw states (exact bf16: two MMAs per k-step instead of three with a normalised pair).
  if (T > 0) {
    WCHECK(gemm_acc32(b.dkv, b.dkv_lo, kvw, false, w.w_kv, d, true, T, d, kvw, F(b.dsn), d, part, pc, st));
    WCHECK(rms_bwd<bf>(static_cast<const bf*>(slab), w.g_kv, F(b.dsn), T, d, s.eps, nullptr, 0, nullptr, 0, nullptr, ds,
                       nullptr, nullptr, nullptr, nullptr, F(b.colp), gr.g_kv, st, true));
    WCHECK(gemm_acc32(b.dkv, b.dkv_lo, kvw, true, slab, d, true, kvw, d, T, gr.w_kv, d, part, pc, st));
    WCHECK(ew_launch(scale_cols_kernel, (long long)kvw * d, st, gr.w_kv, (long long)d, w.g_kv, (long long)kvw, d));
  } else {
    CUCHECK(cudaMemsetAsync(gr.g_kv, 0, (size_t)d * 4, st));
    CUCHECK(cudaMemsetAsync(gr.w_kv, 0, (size_t)kvw * d * 4, st));
  }
  return WHALE_OK;
}

whale_status layer_backward_f32(const Shape& s, const float* x, const float* slab, const int* offsets,
                                const whale_layer_weights& w, const float* dy, float* dx, float* ds,
                                const whale_layer_grads& gr, const whale_shape_hint& h, const BwdBufs& b,
                                cudaStream_t st) {
  const long long rows = (long long)h.B * s.N, T = h.total_L;
  const int d = s.d, H = s.H, Fh = s.Fh, ugw = s.ugw, kvw = s.kvw;
  auto F = [](void* p) { return static_cast<float*>(p); };
  auto W32 = [](const void* p) { return static_cast<const float*>(p); };
  // C = A B with A [M, K] and B [K, N] row-major (dX = dY W)
  auto mm = [&](const float* A, long long lda, const float* B, long long ldb, float* C, long long ldc, long long M,
                long long N, long long K) { return gemm_strided_f32(A, lda, 1, B, ldb, 1, C, ldc, M, N, K, st); };
  // C = A^T B with A [K, M] and B [K, N] row-major (dW = dY^T X)
  auto mtm = [&](const float* A, long long lda, const float* B, long long ldb, float* C, long long ldc, long long M,
                 long long N, long long K) { return gemm_strided_f32(A, 1, lda, B, ldb, 1, C, ldc, M, N, K, st); };
  // ---- forward recompute ----
  WCHECK(row_rms(x, rows, d, s.eps, F(b.r), st));
  WCHECK(gemm_f32(x, d, nullptr, 0, F(b.r), w.g_q, W32(w.w_q), d, F(b.q), rows, F32_NONE, nullptr, st));
  WCHECK(row_rms(slab, T, d, s.eps, F(b.r), st));
  WCHECK(gemm_f32(slab, d, nullptr, 0, F(b.r), w.g_kv, W32(w.w_kv), kvw, F(b.kv), T, F32_NONE, nullptr, st));
  WCHECK(attention_f32(s, F(b.q), F(b.kv), offsets, F(b.a), h.B, T, st));
  if (Fh > 0) {
    WCHECK(gemm_f32(F(b.a), d, x, d, nullptr, nullptr, W32(w.w_f1), Fh, F(b.z1), rows, F32_NONE, nullptr, st));
    WCHECK(ew8_launch(silu_pair_kernel, rows * Fh, st, (const float*)F(b.z1), F(b.g), (__nv_bfloat16*)nullptr,
                     (__nv_bfloat16*)nullptr, rows * Fh));
    WCHECK(gemm_f32(F(b.g), Fh, nullptr, 0, nullptr, nullptr, W32(w.w_f2), d, F(b.f32), rows, F32_RESID, x, st));
  } else {
    WCHECK(gemm_f32(F(b.a), d, x, d, nullptr, nullptr, W32(w.w_f2), d, F(b.f32), rows, F32_RESID, x, st));
  }
  WCHECK(row_rms(F(b.f32), rows, d, s.eps, F(b.r), st));
  WCHECK(gemm_f32(F(b.f32), d, nullptr, 0, F(b.r), w.g_ffn, W32(w.w_upgate), ugw, F(b.ug), rows, F32_NONE, nullptr,
                  st));
  // ---- S5 backward ----
  WCHECK(mm(dy, d, W32(w.w_down), H, F(b.dm), H, rows, H, d));
  WCHECK(ew8_launch(swiglu_bwd_kernel, rows * H, st, (const float*)F(b.ug), (const float*)F(b.dm), rows, H,
                   s.tied ? 1 : 0, (__nv_bfloat16*)nullptr, (__nv_bfloat16*)nullptr, F(b.msw), F(b.dug),
                   (__nv_bfloat16*)nullptr, (__nv_bfloat16*)nullptr));
  WCHECK(mtm(dy, d, F(b.msw), H, gr.w_down, H, d, H, rows));
  WCHECK(mm(F(b.dug), ugw, W32(w.w_upgate), d, F(b.dn), d, rows, d, ugw));
  WCHECK(rms_bwd<float>(F(b.f32), w.g_ffn, F(b.dn), rows, d, s.eps, dy, d, nullptr, 0, F(b.df32), nullptr, nullptr,
                        nullptr, nullptr, F(b.nrm), F(b.colp), gr.g_ffn, st));
  WCHECK(mtm(F(b.dug), ugw, F(b.nrm), d, gr.w_upgate, d, ugw, d, rows));
  // ---- S4 backward ----
  if (Fh > 0) {
    WCHECK(mm(F(b.df32), d, W32(w.w_f2), Fh, F(b.dhid), Fh, rows, Fh, d));
    WCHECK(ew8_launch(silu_bwd_kernel, rows * Fh, st, (const float*)F(b.dhid), (const float*)F(b.z1), F(b.dz),
                     (__nv_bfloat16*)nullptr, (__nv_bfloat16*)nullptr, rows * Fh));
    WCHECK(mtm(F(b.df32), d, F(b.g), Fh, gr.w_f2, Fh, d, Fh, rows));
    WCHECK(mm(F(b.dz), Fh, W32(w.w_f1), 2 * d, F(b.dc), 2 * d, rows, 2 * d, Fh));
    WCHECK(mtm(F(b.dz), Fh, F(b.a), d, gr.w_f1, 2 * d, Fh, d, rows));
    WCHECK(mtm(F(b.dz), Fh, x, d, gr.w_f1 + d, 2 * d, Fh, d, rows));
  } else {
    WCHECK(mm(F(b.df32), d, W32(w.w_f2), 2 * d, F(b.dc), 2 * d, rows, 2 * d, d));
    WCHECK(mtm(F(b.df32), d, F(b.a), d, gr.w_f2, 2 * d, d, d, rows));
    WCHECK(mtm(F(b.df32), d, x, d, gr.w_f2 + d, 2 * d, d, d, rows));
  }
  // ---- S3 backward ----
  if (h.B > 0) {
    const size_t smem = (size_t)s.N * (3 * s.dh + 3) * 4;
    if (smem > 227 * 1024) return WHALE_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)h.B, (unsigned)s.h);
    const float scale = (float)(1.0 / std::sqrt((double)s.dh));
    const int v0 = s.shared_kv ? 0 : d;
    if (T > 0)
      WCHECK(ew_launch(zero_tail_rows_kernel<float>, T * kvw, st, offsets, h.B, T, kvw, F(b.dkv), (float*)nullptr));
#define ATTB32(DH)                                                                                                    \
  do {                                                                                                                \
    CUCHECK(cudaFuncSetAttribute(attn_bwd_f32_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));   \
    attn_bwd_f32_kernel<DH><<<grid, 256, smem, st>>>(F(b.q), F(b.kv), kvw, v0, F(b.dc), 2ll * d, offsets, T, s.N, d,   \
                                                     s.h, scale, F(b.dq), F(b.dkv), s.shared_kv ? 1 : 0);             \
  } while (0)
    switch (s.dh) {
      case 8: ATTB32(8); break;
      case 16: ATTB32(16); break;
      case 32: ATTB32(32); break;
      case 64: ATTB32(64); break;
      default: return WHALE_ERR_UNSUPPORTED;
    }
#undef ATTB32
    CUCHECK(cudaGetLastError());
  }
  // ---- S1 backward ----
  WCHECK(mm(F(b.dq), d, W32(w.w_q), d, F(b.dn), d, rows, d, d));
  WCHECK(launch_pdl(rms_rows_kernel<float>, dim3(rows_blocks(rows)), dim3(256), 0, st, x, w.g_q, rows, d, s.eps,
                    (__nv_bfloat16*)nullptr, (__nv_bfloat16*)nullptr, F(b.nrm)));
  WCHECK(mtm(F(b.dq), d, F(b.nrm), d, gr.w_q, d, d, d, rows));
  WCHECK(rms_bwd<float>(x, w.g_q, F(b.dn), rows, d, s.eps, F(b.df32), d, F(b.dc) + d, 2 * d, dx, nullptr, nullptr,
                        nullptr, nullptr, nullptr, F(b.colp), gr.g_q, st));
  // ---- S2 backward ----
  if (T > 0) {
    WCHECK(mm(F(b.dkv), kvw, W32(w.w_kv), d, F(b.dsn), d, T, d, kvw));
    WCHECK(rms_bwd<float>(slab, w.g_kv, F(b.dsn), T, d, s.eps, nullptr, 0, nullptr, 0, ds, nullptr, nullptr, nullptr,
                          nullptr, F(b.sn), F(b.colp), gr.g_kv, st));
    WCHECK(mtm(F(b.dkv), kvw, F(b.sn), d, gr.w_kv, d, kvw, d, T));
  } else {
    CUCHECK(cudaMemsetAsync(gr.g_kv, 0, (size_t)d * 4, st));
    CUCHECK(cudaMemsetAsync(gr.w_kv, 0, (size_t)kvw * d * 4, st));
  }
  return WHALE_OK;
}

// Workspace of the stack backward (also enough for one layer): the backward buffers, the forward's
// workspace for the fp32 mode's layer inputs, every layer's input as a residual-stream tensor (fp32,
// plus its bf16 pair in bf16 mode), a ping-pong pair of fp32 token gradients and, in bf16 mode, the
// forward activations of every layer but the first (lb[l]: the backward buffers with layer l's
// activations; lb[0] is b itself).
struct StackBwd {
  BwdBufs b;
  BwdBufs lb[64];
  char* fwd;
  Layout fl;
  Stream3 in[64];
  float* g[2];
};
size_t stack_bwd_bytes(const Shape& s, const whale_shape_hint& h, char* base, StackBwd* sb = nullptr) {
  StackBwd local;
  StackBwd& k = sb ? *sb : local;
  size_t o = align_up(bwd_buffers(s, h, base, &k.b));
  k.fwd = nullptr;
  if (!s.bf16) {  // the fp32 stack's forward runs the forward's own layer (its workspace); bf16 recomputes
    k.fl = make_layout(s, h);
    k.fwd = base ? base + o : nullptr;
    o = align_up(o + k.fl.total);
  }
  const size_t rows = (size_t)h.B * s.N;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + o : nullptr;
    o = align_up(o + bytes);
    return p;
  };
  const int nl = std::min(s.layers, 64);
  for (int l = 0; l < nl; ++l) {
    k.in[l].f32 = reinterpret_cast<float*>(take(rows * s.d * 4));
    k.in[l].hi = s.bf16 ? take(rows * s.d * 2) : nullptr;
    k.in[l].lo = s.bf16 ? take(rows * s.d * 2) : nullptr;
  }
  for (int i = 0; i < 2; ++i) k.g[i] = reinterpret_cast<float*>(take(rows * s.d * 4));
  if (s.bf16)
    for (int l = 0; l < nl; ++l) {
      k.lb[l] = k.b;
      if (l > 0) act_buffers(s, h, [&](size_t bytes) -> void* { return take(bytes); }, &k.lb[l]);
    }
  return o;
}

bool grads_ok(const Shape& s, const whale_layer_grads* g) {
  return g && g->g_q && g->g_kv && g->g_ffn && g->w_q && g->w_kv && g->w_f2 && g->w_upgate && g->w_down &&
         (s.Fh == 0 || g->w_f1);
}

}  // namespace

// ============================================================================================
// C ABI
// ============================================================================================
extern "C" {

whale_status whale_profile_begin(int max_kernels) {
  if (max_kernels <= 0) return WHALE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) cudaEventDestroy(r.ev);
  g_prof.clear();
  if (g_prof_start) cudaEventDestroy(g_prof_start);
  g_prof_start = nullptr;
  g_prof_cap = max_kernels;
  g_prof_on = true;
  return WHALE_OK;
}

whale_status whale_profile_end(whale_kernel_time* out, int capacity, int* count) {
  if (!count || (capacity > 0 && !out)) return WHALE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  whale_status st = WHALE_OK;
  int n = 0;
  if (!g_prof.empty() && g_prof_start) {
    if (cudaEventSynchronize(g_prof.back().ev) != cudaSuccess) st = WHALE_ERR_CUDA;
    cudaEvent_t prev = g_prof_start;
    for (const auto& r : g_prof) {
      float ms = 0.f;
      if (st == WHALE_OK && cudaEventElapsedTime(&ms, prev, r.ev) != cudaSuccess) st = WHALE_ERR_CUDA;
      if (n < capacity) {
        const char* name = nullptr;
        if (cudaFuncGetName(&name, r.fn) != cudaSuccess) name = "?";
        out[n] = whale_kernel_time{name, ms};
      }
      ++n;
      prev = r.ev;
    }
  }
  for (auto& r : g_prof) cudaEventDestroy(r.ev);
  g_prof.clear();
  if (g_prof_start) cudaEventDestroy(g_prof_start);
  g_prof_start = nullptr;
  (void)cudaGetLastError();
  *count = n;
  return st;
}

const char* whale_status_string(whale_status s) {
  switch (s) {
    case WHALE_OK: return "ok";
    case WHALE_ERR_INVALID_ARG: return "invalid argument";
    case WHALE_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case WHALE_ERR_CUDA: return "CUDA error";
    case WHALE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case WHALE_ERR_DEVICE_CHECK: return "device-side check recorded an error";
  }
  return "unknown status";
}

size_t whale_prepared_weights_size(const whale_config* cfg) {
  Shape s;
  if (validate(cfg, &s) != WHALE_OK || !s.bf16) return 0;
  const size_t kabs = absorbed_shape(s) ? align_up((size_t)s.h * s.d * s.dh * 2) : 0;
  return (size_t)s.layers * (align_up((size_t)s.d * s.d * 2) + align_up((size_t)s.kvw * s.d * 2) +
                             align_up((size_t)s.ugw * s.d * 2) + kabs);
}

whale_status whale_prepare_weights(const whale_config* cfg, const whale_layer_weights* weights, void* prepared,
                                   size_t prepared_bytes, whale_layer_weights* out_weights, whale_stream_t stream) {
  NvtxRange range("whale_prepare_weights");
  Shape s;
  WCHECK(validate(cfg, &s));
  if (!s.bf16) return WHALE_ERR_UNSUPPORTED;
  if (!weights || !out_weights) return WHALE_ERR_INVALID_ARG;
  s.prepared = false;  // the inputs carry their gains
  for (int l = 0; l < s.layers; ++l)
    if (!weights_ok(s, &weights[l])) return WHALE_ERR_INVALID_ARG;
  if (!prepared || prepared_bytes < whale_prepared_weights_size(cfg) ||
      (reinterpret_cast<uintptr_t>(prepared) & (kAlign - 1)))
    return WHALE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  size_t o = 0;
  for (int l = 0; l < s.layers; ++l) {
    const whale_layer_weights& w = weights[l];
    auto* oq = reinterpret_cast<__nv_bfloat16*>(at(prepared, o));
    o += align_up((size_t)s.d * s.d * 2);
    auto* okv = reinterpret_cast<__nv_bfloat16*>(at(prepared, o));
    o += align_up((size_t)s.kvw * s.d * 2);
    auto* oug = reinterpret_cast<__nv_bfloat16*>(at(prepared, o));
    o += align_up((size_t)s.ugw * s.d * 2);
    __nv_bfloat16* okabs = nullptr;
    if (absorbed_shape(s)) {
      okabs = reinterpret_cast<__nv_bfloat16*>(at(prepared, o));
      o += align_up((size_t)s.h * s.d * s.dh * 2);
    }
    WCHECK(fold_weights(s, static_cast<const __nv_bfloat16*>(w.w_q), w.g_q, static_cast<const __nv_bfloat16*>(w.w_kv),
                        w.g_kv, static_cast<const __nv_bfloat16*>(w.w_upgate), w.g_ffn, oq, okv, oug, st,
                        okabs ? static_cast<const __nv_bfloat16*>(w.w_kv) : nullptr, w.g_kv, okabs));
    out_weights[l] = w;
    out_weights[l].w_q = oq;
    out_weights[l].w_kv = okv;
    out_weights[l].w_upgate = oug;
    out_weights[l].w_kabs = okabs;
  }
  return WHALE_OK;
}

size_t whale_workspace_size(const whale_config* cfg, const whale_shape_hint* hint) {
  Shape s;
  if (validate(cfg, &s) != WHALE_OK || check_hint(hint) != WHALE_OK) return 0;
  return make_layout(s, *hint).total;
}

whale_status whale_fusion_layer_forward(const whale_config* cfg, const void* tokens_in, const void* layer_states,
                                        const int* seq_offsets, const whale_layer_weights* w, void* tokens_out,
                                        const whale_shape_hint* hint, void* ws, size_t ws_bytes,
                                        whale_stream_t stream) {
  NvtxRange range("whale_fusion_layer_forward");
  Shape s;
  Layout L;
  WCHECK(common_checks(cfg, hint, &s, ws, ws_bytes, &L));
  if (hint->B == 0) return WHALE_OK;
  if (!tokens_in || !tokens_out || !seq_offsets || !weights_ok(s, w) || (hint->total_L > 0 && !layer_states))
    return WHALE_ERR_INVALID_ARG;
  if (!aligned16(tokens_in) || !aligned16(tokens_out) || (layer_states && !aligned16(layer_states)))
    return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WCHECK(debug_check(s, seq_offsets, *hint, st));
  const void* slabs[1] = {layer_states};
  return stack_impl(s, tokens_in, nullptr, seq_offsets, w, 0, 1, tokens_out, *hint, ws, L, st, slabs);
}

whale_status whale_fusion_forward(const whale_config* cfg, const void* tokens, const void* seq_states,
                                  const int* seq_offsets, const whale_layer_weights* weights, void* out,
                                  const whale_shape_hint* hint, void* ws, size_t ws_bytes, whale_stream_t stream) {
  NvtxRange range("whale_fusion_forward");
  Shape s;
  Layout L;
  WCHECK(common_checks(cfg, hint, &s, ws, ws_bytes, &L));
  if (hint->B == 0) return WHALE_OK;
  if (!tokens || !out || !seq_offsets || !weights || (hint->total_L > 0 && !seq_states)) return WHALE_ERR_INVALID_ARG;
  for (int l = 0; l < s.layers; ++l)
    if (!weights_ok(s, &weights[l])) return WHALE_ERR_INVALID_ARG;
  if (!aligned16(tokens) || !aligned16(out) || (seq_states && !aligned16(seq_states))) return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WCHECK(debug_check(s, seq_offsets, *hint, st));
  return stack_impl(s, tokens, seq_states, seq_offsets, weights, 0, s.layers, out, *hint, ws, L, st, nullptr);
}

size_t whale_host_workspace_size(const whale_config* cfg, const whale_shape_hint* hint) {
  Shape s;
  if (validate(cfg, &s) != WHALE_OK || check_hint(hint) != WHALE_OK) return 0;
  size_t a, b, c, d, e;
  return align_up(host_staging_bytes(s, *hint, &a, &b, &c, &d, &e)) + make_layout(s, *hint).total;
}

whale_status whale_fusion_forward_host(const whale_config* cfg, const void* host_tokens, const void* host_states,
                                       const int* host_offsets, const whale_layer_weights* weights, void* host_out,
                                       const whale_shape_hint* hint, void* ws, size_t ws_bytes,
                                       whale_stream_t stream) {
  NvtxRange range("whale_fusion_forward_host");
  Shape s;
  WCHECK(validate(cfg, &s));
  WCHECK(check_hint(hint));
  if (s.layers > 64) return WHALE_ERR_UNSUPPORTED;  // the per-layer slab table below
  size_t o_tok, o_s0, o_s1, o_off, o_out;
  const size_t staging = align_up(host_staging_bytes(s, *hint, &o_tok, &o_s0, &o_s1, &o_off, &o_out));
  const Layout L = make_layout(s, *hint);
  if (!ws || ws_bytes < staging + L.total || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)))
    return WHALE_ERR_WORKSPACE;
  if (hint->B == 0) return WHALE_OK;
  if (!host_tokens || !host_out || !host_offsets || !weights || (hint->total_L > 0 && !host_states))
    return WHALE_ERR_INVALID_ARG;
  for (int l = 0; l < s.layers; ++l)
    if (!weights_ok(s, &weights[l])) return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  HostPipe* pipe = nullptr;
  WCHECK(host_pipe(&pipe));
  std::lock_guard<std::mutex> enqueue(pipe->mu);
  void* fws = at(ws, staging);
  const size_t rows = (size_t)hint->B * s.N;
  const size_t tok_bytes = rows * s.d * s.es;
  const size_t slab_bytes = (size_t)hint->total_L * s.d * s.es;
  void* d_tok = at(ws, o_tok);
  void* d_slab[2] = {at(ws, o_s0), at(ws, o_s1)};
  int* d_off = reinterpret_cast<int*>(at(ws, o_off));
  void* d_out = at(ws, o_out);
  CUCHECK(cudaMemcpyAsync(d_off, host_offsets, ((size_t)hint->B + 1) * 4, cudaMemcpyHostToDevice, st));
  CUCHECK(cudaMemcpyAsync(d_tok, host_tokens, tok_bytes, cudaMemcpyHostToDevice, st));
  WCHECK(debug_check(s, d_off, *hint, st));
  // The copy stream starts after everything already queued on `stream` (earlier users of the
  // staging buffers); slab l+1 is copied while layer l computes, into the other buffer.
  CUCHECK(cudaEventRecord(pipe->consumed[0], st));
  CUCHECK(cudaEventRecord(pipe->consumed[1], st));
  auto copy_slab = [&](int l) -> whale_status {
    CUCHECK(cudaStreamWaitEvent(pipe->copy, pipe->consumed[l & 1], 0));
    if (slab_bytes)
      CUCHECK(cudaMemcpyAsync(d_slab[l & 1], static_cast<const char*>(host_states) + (size_t)l * slab_bytes,
                              slab_bytes, cudaMemcpyHostToDevice, pipe->copy));
    CUCHECK(cudaEventRecord(pipe->copied[l & 1], pipe->copy));
    return WHALE_OK;
  };
  WCHECK(copy_slab(0));
  const void* slabs[64];
  for (int l = 0; l < s.layers; ++l) slabs[l] = slab_bytes ? d_slab[l & 1] : nullptr;
  auto hook = [&](int l, bool before) -> whale_status {
    if (before) {
      if (l + 1 < s.layers) WCHECK(copy_slab(l + 1));
      CUCHECK(cudaStreamWaitEvent(st, pipe->copied[l & 1], 0));
    } else {
      CUCHECK(cudaEventRecord(pipe->consumed[l & 1], st));
    }
    return WHALE_OK;
  };
  WCHECK(stack_impl(s, d_tok, nullptr, d_off, weights, 0, s.layers, d_out, *hint, fws, L, st, slabs, hook));
  CUCHECK(cudaMemcpyAsync(host_out, d_out, tok_bytes, cudaMemcpyDeviceToHost, st));
  return WHALE_OK;
}

whale_status whale_project_queries(const whale_config* cfg, long long rows, const void* x, const float* g_q,
                                   const void* w_q, void* q, void* ws, size_t ws_bytes, whale_stream_t stream) {
  NvtxRange range("whale_project_queries");
  Shape s;
  WCHECK(validate(cfg, &s));
  if (rows < 0 || !x || !g_q || !w_q || !q) return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (s.bf16) {
    if (!ws || ws_bytes < (size_t)s.d * s.d * 2) return WHALE_ERR_WORKSPACE;
    auto* wq = static_cast<__nv_bfloat16*>(ws);
    WCHECK(fold_weights(s, static_cast<const __nv_bfloat16*>(w_q), g_q, nullptr, nullptr, nullptr, nullptr, wq, nullptr,
                        nullptr, st));
    return gemm_bf16(opnd(x, nullptr, s.d, s.d), no_opnd(), wq, s.d, Outs{q, nullptr, nullptr, s.d}, nullptr, 0, rows,
                     EPI_STORE, true, s.eps, st);
  }
  if (!ws || ws_bytes < (size_t)rows * 4) return WHALE_ERR_WORKSPACE;
  float* r = static_cast<float*>(ws);
  WCHECK(row_rms(static_cast<const float*>(x), rows, s.d, s.eps, r, st));
  return gemm_f32(static_cast<const float*>(x), s.d, nullptr, 0, r, g_q, static_cast<const float*>(w_q), s.d,
                  static_cast<float*>(q), rows, F32_NONE, nullptr, st);
}

whale_status whale_project_kv(const whale_config* cfg, long long rows, const void* sx, const float* g_kv,
                              const void* w_kv, void* kv, void* ws, size_t ws_bytes, whale_stream_t stream) {
  NvtxRange range("whale_project_kv");
  Shape s;
  WCHECK(validate(cfg, &s));
  if (rows < 0 || !sx || !g_kv || !w_kv || !kv) return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (s.bf16) {
    if (!ws || ws_bytes < (size_t)s.kvw * s.d * 2) return WHALE_ERR_WORKSPACE;
    auto* wkv = static_cast<__nv_bfloat16*>(ws);
    WCHECK(fold_weights(s, nullptr, nullptr, static_cast<const __nv_bfloat16*>(w_kv), g_kv, nullptr, nullptr, nullptr,
                        wkv, nullptr, st));
    return gemm_bf16(opnd(sx, nullptr, s.d, s.d), no_opnd(), wkv, s.kvw, Outs{kv, nullptr, nullptr, s.kvw}, nullptr,
                     0, rows, EPI_STORE, true, s.eps, st);
  }
  if (!ws || ws_bytes < (size_t)rows * 4) return WHALE_ERR_WORKSPACE;
  float* r = static_cast<float*>(ws);
  WCHECK(row_rms(static_cast<const float*>(sx), rows, s.d, s.eps, r, st));
  return gemm_f32(static_cast<const float*>(sx), s.d, nullptr, 0, r, g_kv, static_cast<const float*>(w_kv), s.kvw,
                  static_cast<float*>(kv), rows, F32_NONE, nullptr, st);
}

whale_status whale_attend_states(const whale_config* cfg, const void* q, const void* layer_states,
                                 const int* seq_offsets, const whale_layer_weights* w, void* a,
                                 const whale_shape_hint* hint, void* ws, size_t ws_bytes, whale_stream_t stream) {
  NvtxRange range("whale_attend_states");
  Shape s;
  Layout L;
  WCHECK(common_checks(cfg, hint, &s, ws, ws_bytes, &L));
  if (!s.absorbed) return WHALE_ERR_UNSUPPORTED;
  if (hint->B == 0) return WHALE_OK;
  if (!q || !a || !seq_offsets || !w || !w->w_kv || (!s.prepared && !w->g_kv) || (hint->total_L > 0 && !layer_states))
    return WHALE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(a) || !aligned16(w->w_kv) || !aligned16(w->w_kabs) ||
      (layer_states && !aligned16(layer_states)))
    return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WCHECK(debug_check(s, seq_offsets, *hint, st));
  const void* wkv = w->w_kv;
  const void* wkabs = s.prepared ? w->w_kabs : nullptr;
  auto* wkabs_ws = reinterpret_cast<__nv_bfloat16*>(at(ws, L.wkabs));
  if (!s.prepared) {
    wkv = at(ws, L.wkv);
    wkabs = wkabs_ws;
    WCHECK(fold_weights(s, nullptr, nullptr, static_cast<const __nv_bfloat16*>(w->w_kv), w->g_kv, nullptr, nullptr,
                        nullptr, reinterpret_cast<__nv_bfloat16*>(at(ws, L.wkv)), nullptr, st,
                        static_cast<const __nv_bfloat16*>(w->w_kv), w->g_kv, wkabs_ws));
  } else if (!wkabs) {
    wkabs = wkabs_ws;
    WCHECK(fold_weights(s, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, st,
                        static_cast<const __nv_bfloat16*>(w->w_kv), nullptr, wkabs_ws));
  }
  const void* wv = s.shared_kv ? wkv : static_cast<const char*>(wkv) + (size_t)s.d * s.d * 2;
  WCHECK(abs_units(s, seq_offsets, *hint, ws, L, st));
  return attention_absorbed(s, q, layer_states, seq_offsets, wkabs, wv, a, nullptr, *hint, ws, L, st);
}

whale_status whale_cross_attention(const whale_config* cfg, const void* q, const void* kv, const int* seq_offsets,
                                   void* a, const whale_shape_hint* hint, void* ws, size_t ws_bytes,
                                   whale_stream_t stream) {
  NvtxRange range("whale_cross_attention");
  Shape s;
  WCHECK(validate(cfg, &s));
  WCHECK(check_hint(hint));
  if (hint->B == 0) return WHALE_OK;
  if (!q || !a || !seq_offsets || (hint->total_L > 0 && !kv)) return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (s.bf16) {
    const AttnPlan p = plan_attention(s, hint->B, hint->total_L);
    if (!ws || ws_bytes < p.bytes() || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return WHALE_ERR_WORKSPACE;
    WCHECK(debug_check(s, seq_offsets, *hint, st));
    return attention_bf16(s, q, kv, seq_offsets, a, nullptr, hint->B, hint->total_L, ws, st);
  }
  WCHECK(debug_check(s, seq_offsets, *hint, st));
  return attention_f32(s, static_cast<const float*>(q), static_cast<const float*>(kv), seq_offsets,
                       static_cast<float*>(a), hint->B, hint->total_L, st);
}

whale_status whale_fusion_mlp(const whale_config* cfg, long long rows, const void* a, const void* x, const void* w_f1,
                              const void* w_f2, void* f, void* ws, size_t ws_bytes, whale_stream_t stream) {
  NvtxRange range("whale_fusion_mlp");
  Shape s;
  WCHECK(validate(cfg, &s));
  if (rows < 0 || !a || !x || !w_f2 || !f || (s.Fh > 0 && !w_f1)) return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!s.bf16) {
    if (s.Fh > 0 && (!ws || ws_bytes < (size_t)rows * s.Fh * 4)) return WHALE_ERR_WORKSPACE;
    return fusion_mlp_f32(s, rows, static_cast<const float*>(a), static_cast<const float*>(x),
                          static_cast<const float*>(w_f1), static_cast<const float*>(w_f2), static_cast<float*>(f),
                          static_cast<float*>(ws), st);
  }
  // workspace: x (fp32) | zero lo half | G pair
  const size_t o_z = align_up((size_t)rows * s.d * 4), o_g = o_z + align_up((size_t)rows * s.d * 2);
  const size_t o_gl = o_g + align_up((size_t)rows * s.Fh * 2), need = o_gl + (size_t)rows * s.Fh * 2;
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return WHALE_ERR_WORKSPACE;
  auto* x32 = static_cast<float*>(ws);
  void* zlo = at(ws, o_z);
  WCHECK(pair_from_bf16(x, x32, zlo, rows * s.d, st));
  return fusion_bf16(s, rows, opnd(a, zlo, s.d, s.d), opnd(x, zlo, s.d, s.d), x32, w_f1, w_f2, at(ws, o_g),
                     at(ws, o_gl), Stream3{nullptr, f, nullptr}, st);
}

whale_status whale_swiglu_ffn(const whale_config* cfg, long long rows, const void* f, const float* g_ffn,
                              const void* w_upgate, const void* w_down, void* y, void* ws, size_t ws_bytes,
                              whale_stream_t stream) {
  NvtxRange range("whale_swiglu_ffn");
  Shape s;
  WCHECK(validate(cfg, &s));
  if (rows < 0 || !f || !g_ffn || !w_upgate || !w_down || !y) return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (s.bf16) {
    // workspace: folded up|gate | f (fp32) | zero lo half | U pair
    const size_t o_f = align_up((size_t)s.ugw * s.d * 2), o_z = o_f + align_up((size_t)rows * s.d * 4);
    const size_t o_u = o_z + align_up((size_t)rows * s.d * 2), o_ul = o_u + align_up((size_t)rows * s.H * 2);
    const size_t need = o_ul + (size_t)rows * s.H * 2;
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return WHALE_ERR_WORKSPACE;
    auto* wug = static_cast<__nv_bfloat16*>(ws);
    WCHECK(fold_weights(s, nullptr, nullptr, nullptr, nullptr, static_cast<const __nv_bfloat16*>(w_upgate), g_ffn,
                        nullptr, nullptr, wug, st));
    auto* f32 = reinterpret_cast<float*>(at(ws, o_f));
    void* zlo = at(ws, o_z);
    WCHECK(pair_from_bf16(f, f32, zlo, rows * s.d, st));
    return ffn_bf16(s, rows, opnd(f, zlo, s.d, s.d), f32, wug, w_down, at(ws, o_u), at(ws, o_ul),
                    Stream3{nullptr, y, nullptr}, st);
  }
  const size_t rb = align_up((size_t)rows * 4), ugb = align_up((size_t)rows * s.ugw * 4);
  if (!ws || ws_bytes < rb + ugb + (size_t)rows * s.H * 4) return WHALE_ERR_WORKSPACE;
  float* r = static_cast<float*>(ws);
  float* ug = reinterpret_cast<float*>(at(ws, rb));
  float* u = reinterpret_cast<float*>(at(ws, rb + ugb));
  return swiglu_f32(s, static_cast<const float*>(f), g_ffn, static_cast<const float*>(w_upgate),
                    static_cast<const float*>(w_down), static_cast<float*>(y), rows, r, ug, u, st);
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// Allocation-free attention entry point: partials in a fixed file-scope device array.
// ------------------------------------------------------------------------------------------
namespace {
__device__ __align__(256) unsigned char g_noalloc_scratch[WHALE_NOALLOC_SCRATCH_BYTES];

// The calling thread's current CUDA context, from the driver entry point (no link-time libcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
whale_status current_context(CUcontext* ctx) {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  if (!fn) return WHALE_ERR_CUDA;
  *ctx = nullptr;
  if (fn(ctx) != CUDA_SUCCESS) return WHALE_ERR_CUDA;
  return WHALE_OK;  // *ctx is null if this thread has no current context yet
}

// Device address of g_noalloc_scratch in the current context (the name is only a host-side stand-in
// for the array; kernels must get the real address). Looked up once per context, with the device
// current, and cached under the context: a context created after cudaDeviceReset (a new primary
// context) gets its own lookup, never the address from the old one.
whale_status noalloc_scratch(void** out) {
  static std::mutex mu;
  static std::vector<std::pair<CUcontext, void*>> cache;
  CUcontext ctx = nullptr;
  WCHECK(current_context(&ctx));
  std::lock_guard<std::mutex> lk(mu);
  if (ctx)
    for (const auto& e : cache)
      if (e.first == ctx) {
        *out = e.second;
        return WHALE_OK;
      }
  void* p = nullptr;
  CUCHECK(cudaGetSymbolAddress(&p, g_noalloc_scratch));  // initialises the runtime's context if needed
  if (!ctx) WCHECK(current_context(&ctx));
  if (ctx) cache.push_back({ctx, p});
  *out = p;
  return WHALE_OK;
}
}  // namespace

extern "C" {

whale_status whale_cross_attention_noalloc(const whale_config* cfg, const void* q, const void* kv,
                                           const int* seq_offsets, void* a, const whale_shape_hint* hint,
                                           whale_stream_t stream) {
  Shape s;
  WCHECK(validate(cfg, &s));
  WCHECK(check_hint(hint));
  if (hint->B == 0) return WHALE_OK;
  if (!q || !a || !seq_offsets || (hint->total_L > 0 && !kv)) return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!s.bf16) {
    WCHECK(debug_check(s, seq_offsets, *hint, st));
    return attention_f32(s, static_cast<const float*>(q), static_cast<const float*>(kv), seq_offsets,
                         static_cast<float*>(a), hint->B, hint->total_L, st);
  }
  // only the split-L kernel keeps partials in the scratch; the query-tiled kernel uses none
  const AttnPlan p = plan_attention(s, hint->B, hint->total_L);
  if (!attention_is_query_tiled(s) && p.bytes() > (size_t)WHALE_NOALLOC_SCRATCH_BYTES) return WHALE_ERR_WORKSPACE;
  void* scratch = nullptr;
  WCHECK(noalloc_scratch(&scratch));
  WCHECK(debug_check(s, seq_offsets, *hint, st));
  return attention_bf16(s, q, kv, seq_offsets, a, nullptr, hint->B, hint->total_L, scratch, st);
}

size_t whale_backward_workspace_size(const whale_config* cfg, const whale_shape_hint* hint) {
  Shape s;
  if (validate(cfg, &s) != WHALE_OK || check_hint(hint) != WHALE_OK || !backward_shape_ok(s) || s.prepared) return 0;
  return stack_bwd_bytes(s, *hint, nullptr);
}

whale_status whale_fusion_layer_backward(const whale_config* cfg, const void* tokens_in, const void* layer_states,
                                         const int* seq_offsets, const whale_layer_weights* w, const float* d_out,
                                         float* d_tokens, void* d_states, const whale_layer_grads* grads,
                                         const whale_shape_hint* hint, void* ws, size_t ws_bytes,
                                         whale_stream_t stream) {
  NvtxRange range("whale_fusion_layer_backward");
  Shape s;
  WCHECK(validate(cfg, &s));
  WCHECK(check_hint(hint));
  if (s.prepared) return WHALE_ERR_UNSUPPORTED;
  if (!backward_shape_ok(s)) return WHALE_ERR_UNSUPPORTED;
  if (!weights_ok(s, w) || !grads_ok(s, grads)) return WHALE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  BwdBufs b;
  const size_t need = bwd_buffers(s, *hint, nullptr, &b);  // the prefix of whale_backward_workspace_size
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return WHALE_ERR_WORKSPACE;
  if (hint->B == 0) {  // no examples: every gradient is zero
    const size_t d = s.d;
    const float* zs[] = {grads->g_q, grads->g_kv, grads->g_ffn};
    for (const float* z : zs) CUCHECK(cudaMemsetAsync(const_cast<float*>(z), 0, d * 4, st));
    CUCHECK(cudaMemsetAsync(grads->w_q, 0, d * d * 4, st));
    CUCHECK(cudaMemsetAsync(grads->w_kv, 0, (size_t)s.kvw * d * 4, st));
    if (s.Fh > 0) CUCHECK(cudaMemsetAsync(grads->w_f1, 0, (size_t)s.Fh * 2 * d * 4, st));
    CUCHECK(cudaMemsetAsync(grads->w_f2, 0, d * (size_t)(s.Fh > 0 ? s.Fh : 2 * s.d) * 4, st));
    CUCHECK(cudaMemsetAsync(grads->w_upgate, 0, (size_t)s.ugw * d * 4, st));
    CUCHECK(cudaMemsetAsync(grads->w_down, 0, d * (size_t)s.H * 4, st));
    if (hint->total_L > 0 && d_states)  // rows of no example
      CUCHECK(cudaMemsetAsync(d_states, 0, (size_t)hint->total_L * s.d * s.es, st));
    return WHALE_OK;
  }
  if (!tokens_in || !seq_offsets || !d_out || !d_tokens || (hint->total_L > 0 && (!layer_states || !d_states)))
    return WHALE_ERR_INVALID_ARG;
  if (!aligned16(tokens_in) || !aligned16(d_out) || !aligned16(d_tokens) ||
      (layer_states && !aligned16(layer_states)) || (d_states && !aligned16(d_states)))
    return WHALE_ERR_INVALID_ARG;
  bwd_buffers(s, *hint, static_cast<char*>(ws), &b);
  WCHECK(debug_check(s, seq_offsets, *hint, st));
  if (s.bf16) {
    WCHECK(pair_from_bf16(tokens_in, static_cast<float*>(b.x32), b.xlo, (long long)hint->B * s.N * s.d, st));
    const Stream3 in{static_cast<float*>(b.x32), const_cast<void*>(tokens_in), b.xlo};
    return layer_backward_bf16(s, in, layer_states, seq_offsets, *w, d_out, d_tokens, d_states, *grads, *hint, b, st);
  }
  return layer_backward_f32(s, static_cast<const float*>(tokens_in), static_cast<const float*>(layer_states),
                            seq_offsets, *w, d_out, d_tokens, static_cast<float*>(d_states), *grads, *hint, b, st);
}

whale_status whale_fusion_backward(const whale_config* cfg, const void* tokens, const void* seq_states,
                                   const int* seq_offsets, const whale_layer_weights* weights, const float* d_out,
                                   float* d_tokens, void* d_states, const whale_layer_grads* grads,
                                   const whale_shape_hint* hint, void* ws, size_t ws_bytes, whale_stream_t stream) {
  NvtxRange range("whale_fusion_backward");
  Shape s;
  WCHECK(validate(cfg, &s));
  WCHECK(check_hint(hint));
  if (s.prepared || !backward_shape_ok(s) || s.layers > 64) return WHALE_ERR_UNSUPPORTED;
  if (!weights || !grads) return WHALE_ERR_INVALID_ARG;
  for (int l = 0; l < s.layers; ++l)
    if (!weights_ok(s, &weights[l]) || !grads_ok(s, &grads[l])) return WHALE_ERR_INVALID_ARG;
  const size_t need = stack_bwd_bytes(s, *hint, nullptr);
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return WHALE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long rows = (long long)hint->B * s.N, T = hint->total_L;
  if (hint->B == 0) {
    for (int l = 0; l < s.layers; ++l)
      WCHECK(whale_fusion_layer_backward(cfg, nullptr, nullptr, nullptr, &weights[l], nullptr, nullptr,
                                         T > 0 && d_states ? static_cast<char*>(d_states) + l * T * s.d * s.es
                                                           : nullptr,
                                         &grads[l], hint, ws, ws_bytes, stream));
    return WHALE_OK;
  }
  if (!tokens || !seq_offsets || !d_out || !d_tokens || (T > 0 && (!seq_states || !d_states)))
    return WHALE_ERR_INVALID_ARG;
  if (!aligned16(tokens) || !aligned16(d_out) || !aligned16(d_tokens) || (seq_states && !aligned16(seq_states)) ||
      (d_states && !aligned16(d_states)))
    return WHALE_ERR_INVALID_ARG;
  StackBwd k;
  stack_bwd_bytes(s, *hint, static_cast<char*>(ws), &k);
  WCHECK(debug_check(s, seq_offsets, *hint, st));
  const size_t slab_bytes = (size_t)T * s.d * s.es;
  auto slab = [&](int l) { return T > 0 ? static_cast<const char*>(seq_states) + l * slab_bytes : nullptr; };
  // forward, keeping every layer's input (the residual stream: fp32 and, in bf16 mode, its pair)
  if (s.bf16) {
    // the recompute path of the backward (hi/lo pairs, raw weights, K|V as pairs), so that every
    // layer's input carries the precision its gradients need; each layer's activations stay in
    // lb[l] for its backward below
    WCHECK(pair_from_bf16(tokens, k.in[0].f32, k.in[0].lo, rows * s.d, st));
    CUCHECK(cudaMemcpyAsync(k.in[0].hi, tokens, (size_t)rows * s.d * 2, cudaMemcpyDeviceToDevice, st));
    for (int l = 0; l < s.layers; ++l) {
      WCHECK(recompute_bf16(s, k.in[l], slab(l), seq_offsets, weights[l], *hint, k.lb[l], st));
      if (l + 1 < s.layers) WCHECK(layer_output_bf16(s, weights[l], *hint, k.lb[l], k.in[l + 1], st));
    }
  } else {
    CUCHECK(cudaMemcpyAsync(k.in[0].f32, tokens, (size_t)rows * s.d * 4, cudaMemcpyDeviceToDevice, st));
    for (int l = 0; l + 1 < s.layers; ++l)
      WCHECK(layer_f32(s, k.in[l].f32, slab(l), seq_offsets, weights[l], k.in[l + 1].f32, *hint, k.fwd, k.fl, st));
  }
  // backward, last layer first: each layer's token gradient is the next one's upstream gradient
  const float* g = d_out;
  for (int l = s.layers - 1; l >= 0; --l) {
    float* dx = l == 0 ? d_tokens : k.g[l & 1];
    void* dsl = T > 0 ? static_cast<char*>(d_states) + l * slab_bytes : nullptr;
    if (s.bf16)
      WCHECK(layer_backward_bf16(s, k.in[l], slab(l), seq_offsets, weights[l], g, dx, dsl, grads[l], *hint, k.lb[l], st,
                                 false));
    else
      WCHECK(layer_backward_f32(s, k.in[l].f32, reinterpret_cast<const float*>(slab(l)), seq_offsets, weights[l], g, dx,
                                static_cast<float*>(dsl), grads[l], *hint, k.b, st));
    g = dx;
  }
  return WHALE_OK;
}

whale_status whale_test_bounded_waits(unsigned long long limit_ns, whale_stream_t stream) {
  if (limit_ns < 1000ull || limit_ns > kWaitLimitNs) return WHALE_ERR_INVALID_ARG;
  wait_selftest_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  CUCHECK(cudaGetLastError());
  return WHALE_OK;
}

whale_status whale_get_device_error(whale_stream_t stream, int* code) {
  if (!code) return WHALE_ERR_INVALID_ARG;
  CUCHECK(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  unsigned v = 0, zero = 0;
  CUCHECK(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)));
  CUCHECK(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)));
  *code = (int)v;
  return v ? WHALE_ERR_DEVICE_CHECK : WHALE_OK;
}

}  // extern "C"
