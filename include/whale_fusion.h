/*
 * whale_fusion.h — C ABI of the B200 (sm_100a) WHALE attention-fusion forward.
 *
 * What is computed. WHALE stacks layers; in each, a fusion module lets the Wukong
 * branch's interaction tokens query the HSTU branch's per-position behavior states
 * (gist.science technical summary of WHALE, section 2.1 "Core Architecture",
 * Attention-Based Fusion Module; pith.science verdict, "key_machinery"):
 *
 *   Q    = RMSNorm(H_w; g_q)  W_Q^T                     queries from Wukong tokens
 *   K|V  = RMSNorm(H_s; g_kv) [W_K ; W_V]^T             keys/values from HSTU states
 *   A    = per-head softmax(Q K^T / sqrt(d_head)) V      Eq. (4), over the example's own
 *                                                       jagged history, no mask, no bias
 *   F    = H_w + W_F2 SiLU(W_F1 [A ; H_w])              Eq. (5), residual Fusion MLP
 *   H_f  = F + W_down (SiLU(W_gate n) * (W_up n)),      pre-norm SwiGLU FFN, n = RMSNorm(F; g_ffn),
 *                                                       up|gate run as ONE concatenated GEMM
 *   H_f feeds the next layer's query side (identity Wukong stand-in); layer l reads its
 *   own H_s slab (section 2.1 "Propagation").
 *
 * Conventions (all entry points):
 *  - Matrices are row-major. Weights use the nn.Linear layout [out, in].
 *  - "device" pointers are CUDA global memory on the current device; "host" pointers
 *    are ordinary (preferably pinned) host memory. The caller owns every buffer and
 *    the stream. No entry point allocates device memory: scratch lives in the
 *    caller's workspace (size from whale_workspace_size).
 *  - Element type of tokens, states, weights and outputs is cfg->dtype (bf16 or fp32).
 *    Gains g_* are always fp32 [d]. Offsets are int32.
 *  - All GPU work is enqueued on `stream` and is asynchronous; return codes report
 *    host-detectable errors only (bad arguments, unsupported shapes, launch errors).
 *    Nothing inside a forward synchronises the device or copies device->host: the
 *    shape hint carries the sizes the host needs (the pages' "shape hint tensors",
 *    gist.science section 2.2, Inference Optimizations).
 *  - Offsets must satisfy offsets[0] = 0, offsets[b] <= offsets[b+1],
 *    offsets[B] <= hint->total_L and offsets[b+1]-offsets[b] <= hint->max_L. Kernels
 *    clamp every history row index to [0, total_L), so a violation never reads out of
 *    bounds, but it gives wrong results; with WHALE_DEBUG the forward also checks the
 *    offsets on the device and records WHALE_DEVERR_OFFSETS, read by
 *    whale_get_device_error.
 *  - Device-side waits are bounded; a wait that runs out records WHALE_DEVERR_TIMEOUT
 *    and the kernel returns.
 *  - The forward, backward, step and weight-preparation entry points each mark an NVTX range
 *    named after themselves, and every layer of a stack one named "whale layer <l>", for timeline
 *    tools; with no tool attached these cost nothing.
 */
#ifndef WHALE_FUSION_H_
#define WHALE_FUSION_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* whale_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  WHALE_OK = 0,
  WHALE_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, inconsistent config */
  WHALE_ERR_UNSUPPORTED = 2,   /* valid but not implemented shape (see whale_config) */
  WHALE_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (launch, encode) */
  WHALE_ERR_WORKSPACE = 4,     /* workspace null or smaller than whale_workspace_size */
  WHALE_ERR_DEVICE_CHECK = 5   /* whale_get_device_error found a recorded device error */
} whale_status;

typedef enum { WHALE_FP32 = 0, WHALE_BF16 = 1 } whale_dtype;

/* cfg->flags */
#define WHALE_SHARED_KV 1u  /* K = V: w_kv is W_K alone [d, d] (gist.science 2.2 "Shared Key-Value") */
#define WHALE_TIED_GATE 2u  /* W_gate = W_up: w_upgate is W_up alone [H, d] (gist.science 2.2 "Shared-Gate SwiGLU") */
#define WHALE_DEBUG 4u      /* validate offsets on the device before the forward */
#define WHALE_PREPARED_WEIGHTS 8u  /* bf16: w_q, w_kv, w_upgate (and w_kabs) come from
                                      whale_prepare_weights (gains already folded in, up|gate rows
                                      packed); g_* are not read */
#define WHALE_MATERIALIZED_KV 16u  /* bf16: always project K|V and attend over them, even where the
                                      absorbed path (below) applies */

/* device error bits (whale_get_device_error) */
#define WHALE_DEVERR_TIMEOUT 1
#define WHALE_DEVERR_OFFSETS 2

typedef struct {
  int n_layers;       /* stacked fusion layers (>= 1) */
  int d;              /* width of tokens and states */
  int n_heads;        /* attention heads; d_head = d / n_heads */
  int n_tokens;       /* N: Wukong tokens (queries) per example */
  int ffn_hidden;     /* SwiGLU hidden width H (4d in the pages' setting) */
  int fusion_hidden;  /* Fusion MLP hidden width (2d); 0 = one linear map W_F [d, 2d] */
  int dtype;          /* whale_dtype */
  unsigned flags;     /* WHALE_SHARED_KV | WHALE_TIED_GATE | WHALE_DEBUG | WHALE_PREPARED_WEIGHTS |
                         WHALE_MATERIALIZED_KV */
  float eps;          /* RMSNorm epsilon */
} whale_config;
/* Supported: fp32 — any d with d % n_heads == 0 and d_head in {8, 16, 32, 64, 128} (SIMT correctness path;
 *            its GEMMs take at most 65535 * 64 rows, so total_L and B * n_tokens up to 4 194 240).
 *            bf16 — d % 64 == 0, d_head in {32, 64}, n_heads 2, 4 or a multiple of 8 (the
 *            attention kernels take min(n_heads, 8) heads per CTA), ffn_hidden % 64 == 0,
 *            fusion_hidden % 64 == 0. Any n_tokens >= 1.
 *
 * Absorbed attention (bf16, the default where it applies: n_tokens * n_heads == 256, d_head == 64,
 * d in {256, 512}, WHALE_MATERIALIZED_KV not set). The key and value projections are folded into
 * the queries, which is exact algebra for Eq. (4) with RMSNorm'd states:
 *   q_j . K_t,j = r_t * (H_t . qa),  qa = diag(g_kv) W_K,j^T q_j;   sum_t p_t V_t,j = z W'_V,j^T,
 *   z = sum_t p_t r_t H_t,  W'_V = W_V diag(g_kv),
 * so the history states are read twice and no K|V tensor is formed: 2 (N h) d instead of 2 d^2
 * multiply-adds per history row. Results agree with the materialising path to bf16 rounding, not
 * bit for bit. It assumes finite states: the last 256-row unit of an example multiplies the zero
 * weights of its padding columns with the following rows of the slab. */

/* Per-layer weights: device pointers. Element type cfg->dtype, gains fp32. */
typedef struct {
  const float* g_q;      /* [d]   RMSNorm gain before W_Q */
  const float* g_kv;     /* [d]   RMSNorm gain before W_K, W_V */
  const void* w_q;       /* [d, d] */
  const void* w_kv;      /* [2d, d] = [W_K ; W_V]   ([d, d] with WHALE_SHARED_KV) */
  const void* w_f1;      /* [fusion_hidden, 2d], columns 0..d-1 read A, d..2d-1 read H_w (unused if fusion_hidden 0) */
  const void* w_f2;      /* [d, fusion_hidden]      ([d, 2d] = W_F if fusion_hidden 0) */
  const float* g_ffn;    /* [d]   RMSNorm gain before the SwiGLU FFN */
  const void* w_upgate;  /* [2H, d] = [W_up ; W_gate] ([H, d] with WHALE_TIED_GATE) */
  const void* w_down;    /* [d, H] */
  const void* w_kabs;    /* prepared weights only (may be null): per-head absorbed key weights from
                            whale_prepare_weights, [n_heads * d, d_head]; null = formed per call */
} whale_layer_weights;

/* Host-side sizes, so no device->host read is needed to launch.
 * B: examples; max_L: an upper bound of every history length; total_L: rows of each
 * H_s slab (>= offsets[B]). */
typedef struct {
  int B;
  int max_L;
  long long total_L;
} whale_shape_hint;

/* Human-readable name of a status code (static string). */
const char* whale_status_string(whale_status s);

/* Per-kernel timing, for profiling runs (no counterpart in the paper). Between
 * whale_profile_begin and whale_profile_end, every kernel of the bf16 path that the library
 * launches is followed by a CUDA event on its stream (at most max_kernels of them; the first
 * launch is also preceded by one), so that kernel k's time is the time between event k-1 and
 * event k. The events serialise the launches: a kernel no longer overlaps its prologue with its
 * predecessor's tail, so the sum can exceed an unprofiled run slightly. whale_profile_end waits
 * for the last event, writes up to `capacity` records {kernel name (owned by the CUDA runtime),
 * milliseconds} in launch order, sets *count to the number recorded, and releases the events.
 * Not thread-safe across concurrent forwards on different streams (one global record list). */
typedef struct {
  const char* kernel;
  float ms;
} whale_kernel_time;
whale_status whale_profile_begin(int max_kernels);
whale_status whale_profile_end(whale_kernel_time* out, int capacity, int* count);

/* Bytes of device workspace needed by every entry point below for this config and
 * shape (0 if cfg/hint are invalid or unsupported). The workspace holds one call's scratch
 * tensors and the words its kernels synchronise through (the order in which the absorbed
 * attention's first-pass CTA pairs finish, cleared by every call): calls in flight at the same
 * time, on different streams, need separate workspaces; calls ordered on one stream may share one. */
size_t whale_workspace_size(const whale_config* cfg, const whale_shape_hint* hint);

/* One-time weight preparation (bf16 mode). RMSNorm(x; g) W^T = r(x) * (x (W diag(g))^T), so the
 * gains can live in the weights: this folds g_q into W_Q, g_kv into [W_K ; W_V] and g_ffn into
 * [W_up ; W_gate], re-packing the up|gate rows in blocks of 32 (16 up rows, then the 16 matching
 * gate rows) for the fused SwiGLU epilogue. The results go to `prepared` (device, at least
 * whale_prepared_weights_size bytes, 256-byte aligned, owned by the caller), and `out_weights`
 * (host array of n_layers) receives the input pointers with w_q, w_kv, w_upgate replaced by the
 * prepared copies. Where the absorbed attention applies (see whale_config) it also forms the
 * per-head absorbed key weights w_kabs[j*d + n][k] = W_K[j*d_head + k][n] g_kv[n] log2(e)/sqrt(d_head)
 * and sets out_weights[l].w_kabs (null otherwise). Forwards given out_weights with
 * cfg->flags | WHALE_PREPARED_WEIGHTS skip the per-call fold. Asynchronous on `stream`; the inputs
 * must stay valid until it completes. */
size_t whale_prepared_weights_size(const whale_config* cfg);
whale_status whale_prepare_weights(const whale_config* cfg, const whale_layer_weights* weights, void* prepared,
                                   size_t prepared_bytes, whale_layer_weights* out_weights, whale_stream_t stream);

/* Whole stack (all n_layers) on device buffers.
 *   wukong_tokens  device [B, N, d]            H_w of layer 0
 *   seq_states     device [n_layers, total_L, d]  H_s slab of each layer
 *   seq_offsets    device int32 [B+1]
 *   weights        HOST array of n_layers whale_layer_weights (device pointers inside)
 *   out            device [B, N, d]            H_f of the last layer; must not alias inputs
 *   workspace      device, >= whale_workspace_size bytes, 256-byte aligned */
whale_status whale_fusion_forward(const whale_config* cfg, const void* wukong_tokens, const void* seq_states,
                                  const int* seq_offsets, const whale_layer_weights* weights, void* out,
                                  const whale_shape_hint* hint, void* workspace, size_t workspace_bytes,
                                  whale_stream_t stream);

/* Same computation from HOST buffers: copies each layer's inputs host->device inside the
 * call (overlapped with the previous layer's compute) and the result device->host.
 * host_tokens [B,N,d], host_seq_states [n_layers,total_L,d], host_offsets int32 [B+1],
 * host_out [B,N,d] are host pointers (pin them for asynchronous copies); weights as above.
 * The workspace must hold whale_host_workspace_size bytes. Returns after enqueueing;
 * synchronise `stream` before reading host_out. Calls on one device share one copy stream: calls
 * from several host threads take turns to enqueue (their GPU work may still overlap, each with its
 * own workspace). That stream and its events are created on the device's first call and kept, so
 * this entry point is not usable after cudaDeviceReset in the same process. At most 64 layers. */
size_t whale_host_workspace_size(const whale_config* cfg, const whale_shape_hint* hint);
whale_status whale_fusion_forward_host(const whale_config* cfg, const void* host_tokens,
                                       const void* host_seq_states, const int* host_offsets,
                                       const whale_layer_weights* weights, void* host_out,
                                       const whale_shape_hint* hint, void* workspace, size_t workspace_bytes,
                                       whale_stream_t stream);

/* One layer: tokens_in/out device [B, N, d], layer_states device [total_L, d]. */
whale_status whale_fusion_layer_forward(const whale_config* cfg, const void* tokens_in, const void* layer_states,
                                        const int* seq_offsets, const whale_layer_weights* layer_weights,
                                        void* tokens_out, const whale_shape_hint* hint, void* workspace,
                                        size_t workspace_bytes, whale_stream_t stream);

/* ---- single steps of one layer (for step-level tests and composition) ---------------- */

/* Q = RMSNorm(x; g_q) W_Q^T.  x, q: device [rows, d]. */
whale_status whale_project_queries(const whale_config* cfg, long long rows, const void* x, const float* g_q,
                                   const void* w_q, void* q, void* workspace, size_t workspace_bytes,
                                   whale_stream_t stream);

/* K|V = RMSNorm(s; g_kv) [W_K ; W_V]^T.  s: device [rows, d]; kv: device [rows, 2d]
 * (K in columns 0..d-1, V in d..2d-1; [rows, d] = K with WHALE_SHARED_KV). */
whale_status whale_project_kv(const whale_config* cfg, long long rows, const void* s, const float* g_kv,
                              const void* w_kv, void* kv, void* workspace, size_t workspace_bytes,
                              whale_stream_t stream);

/* Eq. (4): q device [B*N, d] (row b*N+n), kv device [total_L, 2d] (or [total_L, d] shared),
 * offsets device int32 [B+1] -> a device [B*N, d]. Empty histories give a = 0. */
whale_status whale_cross_attention(const whale_config* cfg, const void* q, const void* kv, const int* seq_offsets,
                                   void* a, const whale_shape_hint* hint, void* workspace, size_t workspace_bytes,
                                   whale_stream_t stream);

/* Eq. (5): f = x + W_F2 SiLU(W_F1 [a ; x]) (or x + W_F [a ; x]).  a, x, f: device [rows, d]. */
whale_status whale_fusion_mlp(const whale_config* cfg, long long rows, const void* a, const void* x,
                              const void* w_f1, const void* w_f2, void* f, void* workspace, size_t workspace_bytes,
                              whale_stream_t stream);

/* y = f + W_down (SiLU(W_gate n) * W_up n), n = RMSNorm(f; g_ffn).  f, y: device [rows, d]. */
whale_status whale_swiglu_ffn(const whale_config* cfg, long long rows, const void* f, const float* g_ffn,
                              const void* w_upgate, const void* w_down, void* y, void* workspace,
                              size_t workspace_bytes, whale_stream_t stream);

/* S2 + S3 in absorbed form (see whale_config): A from the projected queries and the raw history
 * states, without forming K|V. q device [B*N, d] bf16 (whale_project_queries), layer_states device
 * [total_L, d], offsets device int32 [B+1]; from `w` it reads g_kv and w_kv (raw), or with
 * WHALE_PREPARED_WEIGHTS the prepared w_kv and w_kabs (w_kabs may be null). a device [B*N, d] bf16.
 * Workspace: whale_workspace_size. WHALE_ERR_UNSUPPORTED where the absorbed path does not apply
 * (fp32, other shapes, WHALE_MATERIALIZED_KV). Empty histories give a = 0. */
whale_status whale_attend_states(const whale_config* cfg, const void* q, const void* layer_states,
                                 const int* seq_offsets, const whale_layer_weights* w, void* a,
                                 const whale_shape_hint* hint, void* workspace, size_t workspace_bytes,
                                 whale_stream_t stream);

/* Eq. (4) like whale_cross_attention, for callers that cannot allocate device memory.
 * No counterpart in the paper: this is a deployment convenience. Some callers cannot call
 * cudaMalloc or hand out a workspace: code embedded in a host framework that owns every byte of
 * device memory through its own allocator or a fixed pre-reserved pool, and latency-critical
 * serving loops where a cudaMalloc (which may synchronise the device) is not acceptable. This
 * entry point takes no workspace: the attention partials live in one file-scope device array of
 * WHALE_NOALLOC_SCRATCH_BYTES (32 MiB) that every GPU which loads this library holds until the
 * process exits. It allocates nothing itself.
 *  - Limit: where the split-L kernel runs (fewer than 128 queries per example, or d_head not 32
 *    or 64), its partials, (B * ceil(N / QB) + G) * n_heads * QB * (d_head + 2) * 4 bytes
 *    (QB = 16, 32 or 64 queries per block, G <= 148), must fit; a larger shape returns
 *    WHALE_ERR_WORKSPACE before any GPU work. The 15k-history stack (B 64, N 32, d 512, 8 heads)
 *    needs 14 MB. Shapes with 128 or more queries per example and d_head 32 or 64 (the serving
 *    shapes) take the query-tiled kernel, which keeps no partials: no limit applies to them.
 *  - The first call in a CUDA context looks up the array's device address (once per context, with
 *    that context's device current) and caches it under the context; make that first call before
 *    any stream capture.
 *  - Every call shares the one array and overwrites it; nothing in it needs to start at zero (each
 *    partial is written before it is read within the same call). Calls whose kernels overlap on
 *    the GPU (other streams, other host threads) race on the array: serialise them.
 *  - fp32 mode uses no scratch and simply runs the fp32 attention. */
#define WHALE_NOALLOC_SCRATCH_BYTES (32u << 20)
whale_status whale_cross_attention_noalloc(const whale_config* cfg, const void* q, const void* kv,
                                           const int* seq_offsets, void* a, const whale_shape_hint* hint,
                                           whale_stream_t stream);

/* ---- backward pass (training) -------------------------------------------------------------
 *
 * The gradients of one fusion layer for an upstream gradient d_out = dLoss/dH_f: the
 * vector-Jacobian product of the forward above, step by step in reverse (the pages give the
 * forward's steps, gist.science section 2.1, and name the backward's schedule, section 2.2
 * "Asymmetric Backward Variants": the attention's backward is KV-parallel here, since a few queries
 * per example meet thousands of history rows; paper-daily.com digest, section 2). The forward is
 * recomputed inside the call (with K|V materialised and the softmax's log-sum-exp kept), so the
 * caller passes only the layer's inputs.
 *
 *   tokens_in     device [B, N, d]    the layer's H_w (cfg->dtype)
 *   layer_states  device [total_L, d] the layer's H_s (cfg->dtype)
 *   seq_offsets   device int32 [B+1]
 *   w             the layer's RAW weights and gains (WHALE_PREPARED_WEIGHTS is not accepted)
 *   d_out         device fp32 [B, N, d]      dLoss/dH_f
 *   d_tokens      device fp32 [B, N, d]      dLoss/dH_w (written)
 *   d_states      device [total_L, d]        dLoss/dH_s in cfg->dtype (written; rows past offsets[B],
 *                                            which no example reads, get 0)
 *   grads         HOST struct of device fp32 pointers, each overwritten with dLoss/d(parameter),
 *                 summed over the batch, in the parameter's own layout (w_f1 may be null when
 *                 fusion_hidden is 0)
 *   workspace     device, >= whale_backward_workspace_size bytes, 256-byte aligned
 *
 * Supported: d <= 1024, d % 32 == 0 and ffn_hidden a multiple of 8; bf16 also with n_tokens <= 32,
 * d_head 32 or 64 and d % 128 == 0; fp32 with d_head 8, 16, 32 or 64 (the SIMT correctness mode). Other shapes return
 * WHALE_ERR_UNSUPPORTED (the many-candidate serving shape is an inference shape). Asynchronous on `stream`; no device-to-host reads. In bf16
 * mode dq is summed with fp32 atomics across history chunks, so repeated calls can differ in the
 * last bits of d_tokens and of the gradients downstream of it. */
typedef struct {
  float* g_q;      /* [d] */
  float* g_kv;     /* [d] */
  float* w_q;      /* [d, d] */
  float* w_kv;     /* [2d, d] ([d, d] with WHALE_SHARED_KV) */
  float* w_f1;     /* [fusion_hidden, 2d] (null if fusion_hidden 0) */
  float* w_f2;     /* [d, fusion_hidden] ([d, 2d] if fusion_hidden 0) */
  float* g_ffn;    /* [d] */
  float* w_upgate; /* [2H, d] ([H, d] with WHALE_TIED_GATE) */
  float* w_down;   /* [d, H] */
} whale_layer_grads;
/* Workspace of whale_fusion_backward for cfg->n_layers layers (also enough for
 * whale_fusion_layer_backward; 0 for unsupported shapes). */
size_t whale_backward_workspace_size(const whale_config* cfg, const whale_shape_hint* hint);
whale_status whale_fusion_layer_backward(const whale_config* cfg, const void* tokens_in, const void* layer_states,
                                         const int* seq_offsets, const whale_layer_weights* w, const float* d_out,
                                         float* d_tokens, void* d_states, const whale_layer_grads* grads,
                                         const whale_shape_hint* hint, void* workspace, size_t workspace_bytes,
                                         whale_stream_t stream);

/* The whole stack's backward: the forward is run once more, keeping every layer's input (the
 * residual stream between layers in fp32 and its hi/lo pair, as the forward carries it) and, in bf16
 * mode, every layer's forward activations (its K|V pair over the history above all, about 4 bytes per
 * K|V element), then each layer's backward, last layer first, each layer's d_tokens being the upstream
 * gradient of the layer below (the Wukong module between layers is the identity, as in the forward).
 * In bf16 mode each layer's forward thus runs once; the fp32 mode recomputes it inside the layer's
 * backward.
 *   wukong_tokens  device [B, N, d]               H_w of layer 0 (cfg->dtype)
 *   seq_states     device [n_layers, total_L, d]  H_s slab of each layer
 *   weights        HOST array of n_layers raw whale_layer_weights
 *   d_out          device fp32 [B, N, d]          dLoss/d(last layer's H_f)
 *   d_tokens       device fp32 [B, N, d]          dLoss/d(layer 0's H_w) (written)
 *   d_states       device [n_layers, total_L, d]  dLoss/dH_s of each layer, cfg->dtype (written)
 *   grads          HOST array of n_layers whale_layer_grads (device fp32 pointers, overwritten)
 *   workspace      device, >= whale_backward_workspace_size bytes, 256-byte aligned
 * Supported shapes as for whale_fusion_layer_backward, n_layers <= 64. */
whale_status whale_fusion_backward(const whale_config* cfg, const void* wukong_tokens, const void* seq_states,
                                   const int* seq_offsets, const whale_layer_weights* weights, const float* d_out,
                                   float* d_tokens, void* d_states, const whale_layer_grads* grads,
                                   const whale_shape_hint* hint, void* workspace, size_t workspace_bytes,
                                   whale_stream_t stream);

/* Failure detection. Every device-side wait of the library's kernels (a pipeline stage on an
 * mbarrier, one CTA pair waiting for another's published results) gives up after a time limit
 * (2 s in the kernels), records WHALE_DEVERR_TIMEOUT in the device error word and lets its kernel
 * return instead of hanging the GPU; results of that call are then invalid, and the timeout is seen
 * through whale_get_device_error (no entry point synchronises to check it on its own).
 * whale_test_bounded_waits exercises that mechanism with no pipeline around it: it enqueues one
 * small kernel whose two waits can never be satisfied (an mbarrier that no thread arrives on, a
 * flag that no thread sets), each bounded by limit_ns (1 us .. 2 s, else WHALE_ERR_INVALID_ARG).
 * Both give up after about limit_ns and record WHALE_DEVERR_TIMEOUT; the kernel returns and the
 * context stays usable. No counterpart in the paper: a health check of the failure detection. */
whale_status whale_test_bounded_waits(unsigned long long limit_ns, whale_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word of the current
 * device (bits WHALE_DEVERR_*). Returns WHALE_ERR_DEVICE_CHECK if any bit was set. */
whale_status whale_get_device_error(whale_stream_t stream, int* code);

#ifdef __cplusplus
}
#endif

#endif /* WHALE_FUSION_H_ */
