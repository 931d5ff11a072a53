// attention.cuh — Eq. (4) of WHALE: each Wukong query attends over its own example's
// jagged history (softmax(q k^T / sqrt(d_head)) v per head, no mask, no bias).
//
// Work decomposition (flattened split-L). A work item is (example b, query block qb) and owns
// the L_b history rows of example b. All items' rows are laid end to end in one index space of
// W = n_qblocks * sum_b L_b "work rows" (item-major), and CTA c of the G CTAs of a head group
// takes the contiguous slice [c*W/G, (c+1)*W/G). Every CTA therefore streams the same number of
// K|V rows whatever the length mix, in one wave; a slice that crosses item boundaries is cut
// into segments, one partial (m, l, o) per segment, at most (items + G) partials in total.
//
// Inside a CTA: the K|V rows of its head group stream through a STAGES-deep ring of shared-
// memory stages filled by TMA (64-column boxes, 128-byte swizzle; rows past the slab are
// zero-filled, rows past the segment masked). One warp per head keeps its queries' running max
// m, sum l and unnormalised output o in registers (online softmax in base 2), computing q k^T
// and p v with warp-level bf16 tensor-core MMAs fed by ldmatrix from the swizzled stages; row
// max / sum reductions are warp shuffles across the 4 threads that share a query row. A last
// warp issues the TMA. An item that lies inside one slice is finished in place; otherwise every
// slice writes a partial, counts itself done on the item's counter, and the CTA that completes
// the item merges the partials with log-sum-exp and writes A (no separate combine pass).
// At the workloads' query counts the path is HBM-bound (N flops per byte of K|V); the tensor
// cores only need to keep up with the stream.
#pragma once

#include "ptx.cuh"

namespace whale {

struct AttnArgs {
  const __nv_bfloat16* q;  // [B*N, d], row b*N + n, head j in columns [j*DH, (j+1)*DH)
  const int* offsets;      // [B+1]
  float* part_o;           // [slots, h, QB, DH], slots = B * n_qblocks + G
  float* part_ml;          // [slots, h, QB, 2]  (m in log2 units, l)
  int B;
  int N;                   // queries per example
  int QB;                  // queries per work item (16 * QT)
  int n_qblocks;           // ceil(N / QB)
  int d;                   // width (row stride of q)
  int n_heads;
  int v_col0;              // column where V starts inside a kv row (d, or 0 for shared K = V)
  int shared_kv;           // 1: V tiles are the K tiles
  int G;                   // CTAs per head group in the flattened schedule
  long long total_L;       // rows of the kv tensor
  float scale_log2;        // log2(e) / sqrt(DH)
  int* counters;           // [B * n_qblocks] finished-slice counts, zero at launch
  __nv_bfloat16* out;      // A [B*N, d] (bf16)
  __nv_bfloat16* out_lo;   // bf16 residue of A (may be null)
  float* lse;              // [B*N, h] log2 of each softmax denominator, in scaled units (may be null):
                           // p_t = 2^(s_t * scale_log2 - lse); the backward pass reuses it
};

// Offsets clamped into the slab [0, total_L]: example b owns rows [lo_b, hi_b).
__device__ __forceinline__ long long clamp_off(const AttnArgs& a, int b) {
  long long o = a.offsets[b];
  return o < 0 ? 0 : (o > a.total_L ? a.total_L : o);
}

// Flat work-row space: example b's items start at nqb * lo_b; P0 = start of example 0, W = size.
__device__ __forceinline__ void flat_extent(const AttnArgs& a, long long& P0, long long& W) {
  const long long lo = clamp_off(a, 0), hi = clamp_off(a, a.B);
  P0 = (long long)a.n_qblocks * lo;
  W = hi > lo ? (long long)a.n_qblocks * (hi - lo) : 0;
}

// Start of CTA c's slice.
__device__ __forceinline__ long long slice_start(long long P0, long long W, int G, int c) {
  return P0 + (W * c) / G;
}

// One segment of a slice: rows [t0, t1) of example b for query block qb (item = b*nqb + qb).
struct AttnSeg {
  int b, qb, item;
  long long t0, t1;
};

// Next segment at flat position p (< pend). Returns false at the end or on inconsistent offsets
// (which can only shorten the work: every row index stays inside [0, total_L)).
__device__ __forceinline__ bool attn_next_segment(const AttnArgs& a, long long& p, long long pend, AttnSeg& sg) {
  if (p >= pend) return false;
  // largest b in [0, B) with nqb * lo_b <= p
  int lo = 0, hi = a.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)a.n_qblocks * clamp_off(a, mid) <= p) lo = mid;
    else hi = mid - 1;
  }
  const int b = lo;
  const long long lo_b = clamp_off(a, b);
  long long hi_b = clamp_off(a, b + 1);
  if (hi_b < lo_b) hi_b = lo_b;
  const long long L = hi_b - lo_b;
  const long long rel = p - (long long)a.n_qblocks * lo_b;
  if (L <= 0 || rel < 0) return false;
  const long long qb = rel / L, t = rel % L;
  if (qb >= a.n_qblocks) return false;
  long long len = L - t;
  if (len > pend - p) len = pend - p;
  sg.b = b;
  sg.qb = (int)qb;
  sg.item = b * a.n_qblocks + (int)qb;
  sg.t0 = lo_b + t;
  sg.t1 = lo_b + t + len;
  p += len;
  return true;
}

// CTA whose slice contains flat position p.
__device__ __forceinline__ int attn_cta_of(long long p, long long P0, long long W, int G) {
  int c = (int)(((p - P0) * G) / W);
  if (c < 0) c = 0;
  if (c > G - 1) c = G - 1;
  while (c + 1 < G && slice_start(P0, W, G, c + 1) <= p) ++c;
  while (c > 0 && slice_start(P0, W, G, c) > p) --c;
  return c;
}

// Number of CTAs whose (non-empty) slices hold rows of an item that starts at flat position F and
// has L rows, and the first / last of them.
__device__ __forceinline__ int attn_item_ctas(long long F, long long L, long long P0, long long W, int G, int& c0,
                                              int& c1) {
  c0 = attn_cta_of(F, P0, W, G);
  c1 = attn_cta_of(F + L - 1, P0, W, G);
  int n = 0;
  for (int k = c0; k <= c1; ++k) n += slice_start(P0, W, G, k) < slice_start(P0, W, G, k + 1);
  return n;
}

template <int DH, int QT, int T, int HG>
struct AttnCfg {
  static constexpr int NBOX = HG * DH / 64;           // 64-column TMA boxes per K (or V) tile
  static constexpr uint32_t BOX_BYTES = T * 128;
  static constexpr uint32_t KV_BYTES = NBOX * BOX_BYTES;
  static constexpr int THREADS = 32 * (HG + 1);
  static_assert((HG * DH) % 64 == 0, "a head group must cover whole 64-column boxes");
  static_assert(T % 16 == 0 && DH % 16 == 0, "tile shape");
};

template <int DH, int QT, int T, int HG, int STAGES>
__global__ void __launch_bounds__(32 * (HG + 1), 1)
    attn_splitl_kernel(const __grid_constant__ CUtensorMap tmKV, const AttnArgs a) {
  using C = AttnCfg<DH, QT, T, HG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t stage_bytes = a.shared_kv ? C::KV_BYTES : 2 * C::KV_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * 2 * C::KV_BYTES);
  uint64_t* empty = full + STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + STAGES);

  volatile int* last_flag = reinterpret_cast<volatile int*>(empty + STAGES) + 1;

  const int cta = blockIdx.x, hg = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  long long P0, W;
  flat_extent(a, P0, W);
  // Items with an empty history get A = 0 here (no slice covers them).
  for (int item = cta; item < a.B * a.n_qblocks; item += a.G) {
    const int b = item / a.n_qblocks, qb = item % a.n_qblocks;
    if (clamp_off(a, b + 1) > clamp_off(a, b)) continue;
    for (int idx = threadIdx.x; idx < a.QB * HG * DH; idx += blockDim.x) {
      const int nl = idx / (HG * DH), col = hg * HG * DH + idx % (HG * DH);
      const int n = qb * a.QB + nl;
      if (n >= a.N) continue;
      const long long oi = ((long long)b * a.N + n) * a.d + col;
      a.out[oi] = __float2bfloat16_rn(0.f);
      if (a.out_lo) a.out_lo[oi] = __float2bfloat16_rn(0.f);
    }
  }
  const long long p_begin = slice_start(P0, W, a.G, cta), p_end = slice_start(P0, W, a.G, cta + 1);
  if (p_begin >= p_end) return;  // uniform across the CTA

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], HG);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  __syncthreads();

  if (warp == HG) {
    // ---------------- TMA producer: every tile of every segment of the slice ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmKV);
      const int col_k = hg * HG * DH;
      const int col_v = a.v_col0 + hg * HG * DH;
      int i = 0;
      bool stop = false;
      long long p = p_begin;
      AttnSeg sg;
      while (!stop && attn_next_segment(a, p, p_end, sg)) {
        for (long long row = sg.t0; row < sg.t1; row += T, ++i) {
          const int s = i % STAGES, u = i / STAGES;
          if (i >= STAGES && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag)) {
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(&full[s], stage_bytes);
          uint8_t* sk = smem + s * 2 * C::KV_BYTES;
#pragma unroll 1
          for (int bx = 0; bx < C::NBOX; ++bx) {
            tma_load_2d(sk + bx * C::BOX_BYTES, &tmKV, col_k + bx * 64, (int)row, &full[s]);
            if (!a.shared_kv)
              tma_load_2d(sk + C::KV_BYTES + bx * C::BOX_BYTES, &tmKV, col_v + bx * 64, (int)row, &full[s]);
          }
        }
      }
      if (*abort_flag) {
        volatile int quiet = 0;
        for (int k = (i > STAGES ? i - STAGES : 0); k < i; ++k) mbar_wait(&full[k % STAGES], (k / STAGES) & 1, &quiet);
      }
    }
    return;
  }

  // ---------------- compute warp: one head ----------------
  const int head = hg * HG + warp;
  const int g = lane >> 2, qd = lane & 3;
  const int hcol = (warp * DH) & 63;          // head's first column inside its 64-column box
  const int hbox = (warp * DH) >> 6;          // head's box
  const int mi = lane >> 3, r8 = lane & 7;
  int i = 0;
  long long p = p_begin;
  AttnSeg sg;
  bool ok = true;
  while (ok && attn_next_segment(a, p, p_end, sg)) {
    // Q fragments of this segment's query block (A operand, row-major [query][d_head]).
    uint32_t qa[QT][DH / 16][4];
#pragma unroll
    for (int mt = 0; mt < QT; ++mt) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int n = sg.qb * a.QB + mt * 16 + g + 8 * hr;
        const bool valid = n < a.N;
        const uint32_t* qrow =
            reinterpret_cast<const uint32_t*>(a.q + ((long long)sg.b * a.N + (valid ? n : 0)) * a.d + head * DH);
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          qa[mt][ks][hr] = valid ? qrow[ks * 8 + qd] : 0u;          // columns 16ks + 2qd, +1
          qa[mt][ks][2 + hr] = valid ? qrow[ks * 8 + 4 + qd] : 0u;  // columns 16ks + 8 + 2qd, +1
        }
      }
    }
    float o[QT][DH / 8][4];
    float m_run[QT][2], l_run[QT][2];
#pragma unroll
    for (int mt = 0; mt < QT; ++mt) {
#pragma unroll
      for (int nt = 0; nt < DH / 8; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[mt][nt][j] = 0.f;
      m_run[mt][0] = m_run[mt][1] = -INFINITY;
      l_run[mt][0] = l_run[mt][1] = 0.f;
    }

    for (long long trow0 = sg.t0; trow0 < sg.t1; trow0 += T, ++i) {
      const int s = i % STAGES, u = i / STAGES;
      if (!mbar_wait(&full[s], u & 1, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t kbase = smem_u32(smem + s * 2 * C::KV_BYTES + hbox * C::BOX_BYTES);
      const uint32_t vbase = a.shared_kv ? kbase : kbase + C::KV_BYTES;

      // S = Q K^T for this tile: [16*QT queries] x [T rows]
      float sc[QT][T / 8][4];
#pragma unroll
      for (int mt = 0; mt < QT; ++mt)
#pragma unroll
        for (int nt = 0; nt < T / 8; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) sc[mt][nt][j] = 0.f;
#pragma unroll
      for (int ks = 0; ks < DH / 16; ++ks) {
#pragma unroll
        for (int np = 0; np < T / 16; ++np) {
          // matrices: (rows 16np+0..7, k lo), (same rows, k hi), (rows 16np+8..15, k lo), (k hi)
          const int trow = 16 * np + 8 * (mi >> 1) + r8;
          const int chunk16 = (hcol + 16 * ks + 8 * (mi & 1)) >> 3;
          const uint32_t addr = kbase + trow * 128 + ((chunk16 ^ (trow & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
#pragma unroll
          for (int mt = 0; mt < QT; ++mt) {
            mma_bf16_16816(sc[mt][2 * np], qa[mt][ks][0], qa[mt][ks][1], qa[mt][ks][2], qa[mt][ks][3], b0, b1);
            mma_bf16_16816(sc[mt][2 * np + 1], qa[mt][ks][0], qa[mt][ks][1], qa[mt][ks][2], qa[mt][ks][3], b2, b3);
          }
        }
      }

      // online softmax (base 2); rows past the segment end are masked out. The reference max
      // m_run (scaled log2 units) moves only when some row's max exceeds it by more than 8, so the
      // O / l rescale is skipped on most tiles; p = 2^(s*scale - m_run) <= 2^8 stays exact in fp32
      // and well inside bf16 range. The decision is warp-uniform.
      const bool partial = trow0 + T > sg.t1;
      uint32_t pa[QT][T / 16][4];
      float mxs[QT][2];
      bool need = false;
#pragma unroll
      for (int mt = 0; mt < QT; ++mt) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          float mx = -INFINITY;
#pragma unroll
          for (int nt = 0; nt < T / 8; ++nt) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              if (partial && trow0 + nt * 8 + 2 * qd + j >= sg.t1) sc[mt][nt][2 * hr + j] = -INFINITY;
              mx = fmaxf(mx, sc[mt][nt][2 * hr + j]);
            }
          }
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          mxs[mt][hr] = mx * a.scale_log2;
          need |= mxs[mt][hr] > m_run[mt][hr] + 8.0f;
        }
      }
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int mt = 0; mt < QT; ++mt) {
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            const float m_new = fmaxf(m_run[mt][hr], mxs[mt][hr]);
            const float corr = fast_exp2(m_run[mt][hr] - m_new);
            m_run[mt][hr] = m_new;
            l_run[mt][hr] *= corr;
#pragma unroll
            for (int nt = 0; nt < DH / 8; ++nt) {
              o[mt][nt][2 * hr] *= corr;
              o[mt][nt][2 * hr + 1] *= corr;
            }
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < QT; ++mt) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const float neg_m = -m_run[mt][hr];
          float sum = 0.f;
#pragma unroll
          for (int nt = 0; nt < T / 8; ++nt) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float pv = fast_exp2(fmaf(sc[mt][nt][2 * hr + j], a.scale_log2, neg_m));
              sc[mt][nt][2 * hr + j] = pv;
              sum += pv;
            }
          }
          l_run[mt][hr] += sum;
        }
#pragma unroll
        for (int kt = 0; kt < T / 16; ++kt) {
          pa[mt][kt][0] = pack_bf16x2(sc[mt][2 * kt][0], sc[mt][2 * kt][1]);
          pa[mt][kt][1] = pack_bf16x2(sc[mt][2 * kt][2], sc[mt][2 * kt][3]);
          pa[mt][kt][2] = pack_bf16x2(sc[mt][2 * kt + 1][0], sc[mt][2 * kt + 1][1]);
          pa[mt][kt][3] = pack_bf16x2(sc[mt][2 * kt + 1][2], sc[mt][2 * kt + 1][3]);
        }
      }

      // O += P V
#pragma unroll
      for (int kt = 0; kt < T / 16; ++kt) {
#pragma unroll
        for (int cp = 0; cp < DH / 16; ++cp) {
          // matrices: (rows 16kt+0..7, cols 16cp+0..7), (rows +8..15, same), (rows 0..7, cols +8), (rows +8, cols +8)
          const int trow = 16 * kt + 8 * (mi & 1) + r8;
          const int chunk16 = (hcol + 16 * cp + 8 * (mi >> 1)) >> 3;
          const uint32_t addr = vbase + trow * 128 + ((chunk16 ^ (trow & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(addr, b0, b1, b2, b3);
#pragma unroll
          for (int mt = 0; mt < QT; ++mt) {
            mma_bf16_16816(o[mt][2 * cp], pa[mt][kt][0], pa[mt][kt][1], pa[mt][kt][2], pa[mt][kt][3], b0, b1);
            mma_bf16_16816(o[mt][2 * cp + 1], pa[mt][kt][0], pa[mt][kt][1], pa[mt][kt][2], pa[mt][kt][3], b2, b3);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (!ok) break;

    // ---- end of a segment: quad-reduced row sums, then either the final A (the item lies in this
    // CTA's slice alone) or a partial; the CTA that completes an item merges all of its partials.
    float lq[QT][2];
#pragma unroll
    for (int mt = 0; mt < QT; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        float l = l_run[mt][hr];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        lq[mt][hr] = l;
      }
    const long long lo_b = clamp_off(a, sg.b);
    const long long Lb = clamp_off(a, sg.b + 1) - lo_b;
    int c0, c1;
    const int nseg = attn_item_ctas((long long)a.n_qblocks * lo_b + (long long)sg.qb * Lb, Lb, P0, W, a.G, c0, c1);
    bool finish = nseg <= 1;
    if (!finish) {
      // partial of this segment: slot = item + cta (unique and increasing along the slices)
      const long long slot = (long long)sg.item + cta;
#pragma unroll
      for (int mt = 0; mt < QT; ++mt) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int nl = mt * 16 + g + 8 * hr;
          if (sg.qb * a.QB + nl >= a.N) continue;
          const long long base = (slot * a.n_heads + head) * a.QB + nl;
          if (qd == 0) {
            a.part_ml[2 * base] = m_run[mt][hr];
            a.part_ml[2 * base + 1] = lq[mt][hr];
          }
          float* po = a.part_o + base * DH;
#pragma unroll
          for (int nt = 0; nt < DH / 8; ++nt)
            *reinterpret_cast<float2*>(po + nt * 8 + 2 * qd) = make_float2(o[mt][nt][2 * hr], o[mt][nt][2 * hr + 1]);
        }
      }
      __threadfence();
      asm volatile("bar.sync 1, %0;" ::"n"(HG * 32) : "memory");  // compute warps only
      if (threadIdx.x == 0) {
        const int prev = atomicAdd(a.counters + sg.item, 1);
        *last_flag = (prev == nseg - 1);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(HG * 32) : "memory");
      finish = *last_flag != 0;
      if (finish) {
        __threadfence();
        // Merge every slice's partial (this CTA's own included, re-read) in slot order from an
        // empty state, so the result does not depend on which CTA finishes the item. Partials
        // written by other SMs are read through L2.
#pragma unroll
        for (int mt = 0; mt < QT; ++mt)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            m_run[mt][hr] = -INFINITY;
            lq[mt][hr] = 0.f;
#pragma unroll
            for (int nt = 0; nt < DH / 8; ++nt) o[mt][nt][2 * hr] = o[mt][nt][2 * hr + 1] = 0.f;
          }
        for (int k = c0; k <= c1; ++k) {
          if (slice_start(P0, W, a.G, k) >= slice_start(P0, W, a.G, k + 1)) continue;
          const long long slot_k = (long long)sg.item + k;
#pragma unroll
          for (int mt = 0; mt < QT; ++mt) {
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
              const int nl = mt * 16 + g + 8 * hr;
              if (sg.qb * a.QB + nl >= a.N) continue;
              const long long base = (slot_k * a.n_heads + head) * a.QB + nl;
              const float2 ml = __ldcg(reinterpret_cast<const float2*>(a.part_ml + 2 * base));
              const float m_new = fmaxf(m_run[mt][hr], ml.x);
              const float w_acc = fast_exp2(m_run[mt][hr] - m_new), w_k = fast_exp2(ml.x - m_new);
              m_run[mt][hr] = m_new;
              lq[mt][hr] = lq[mt][hr] * w_acc + ml.y * w_k;
              const float* po = a.part_o + base * DH;
#pragma unroll
              for (int nt = 0; nt < DH / 8; ++nt) {
                const float2 ov = __ldcg(reinterpret_cast<const float2*>(po + nt * 8 + 2 * qd));
                o[mt][nt][2 * hr] = o[mt][nt][2 * hr] * w_acc + ov.x * w_k;
                o[mt][nt][2 * hr + 1] = o[mt][nt][2 * hr + 1] * w_acc + ov.y * w_k;
              }
            }
          }
        }
      }
    }
    if (finish) {
      // A = o / l as bf16 (and its bf16 residue)
#pragma unroll
      for (int mt = 0; mt < QT; ++mt) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int nl = mt * 16 + g + 8 * hr;
          const int n = sg.qb * a.QB + nl;
          if (n >= a.N) continue;
          const float inv = 1.0f / lq[mt][hr];
          const long long row = ((long long)sg.b * a.N + n) * a.d + head * DH;
          if (a.lse != nullptr && qd == 0)
            a.lse[((long long)sg.b * a.N + n) * a.n_heads + head] = m_run[mt][hr] + __log2f(lq[mt][hr]);
#pragma unroll
          for (int nt = 0; nt < DH / 8; ++nt) {
            const float x0 = o[mt][nt][2 * hr] * inv, x1 = o[mt][nt][2 * hr + 1] * inv;
            const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
            *reinterpret_cast<__nv_bfloat162*>(a.out + row + nt * 8 + 2 * qd) = h;
            if (a.out_lo) {
              const float2 hf = __bfloat1622float2(h);
              *reinterpret_cast<uint32_t*>(a.out_lo + row + nt * 8 + 2 * qd) = pack_bf16x2(x0 - hf.x, x1 - hf.y);
            }
          }
        }
      }
    }
  }
}

}  // namespace whale
