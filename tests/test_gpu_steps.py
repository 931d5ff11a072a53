"""Step-level parity of the CUDA path against the fp64 oracle, through the C ABI:
S1 query projection, S2 K|V projection (tcgen05 GEMMs with the fused RMSNorm row factor),
S3 cross-attention (split-L kernel + combine, and the fp32 kernel), S4 Fusion MLP, S5 SwiGLU
FFN, and S2 + S3 in absorbed form (whale_attend_states). Shapes cross 128-row tiles with ragged
tails, several K/V splits, empty and one-row histories, query counts that are not multiples of 16,
and each BN tile width."""
import numpy as np
import pytest
import torch

from oracle import whale_oracle as O
from tests.gpu_util import assert_parity, bf16_randn
from wukong_hstu_cross_b200 import inputs as I

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from wukong_hstu_cross_b200 import build
    build.build()
    from wukong_hstu_cross_b200 import whale as W

DEV = "cuda"


def _t(a, dtype="bf16"):
    if dtype == "bf16":
        return torch.from_numpy(I.bf16_bits(a).view(np.int16)).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV)


def _g(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV)


def _cfg(d, h, N=16, H=None, Fh=None, dtype="bf16", flags=0, layers=1):
    return W.make_config(layers, d, h, N, H or 4 * d, 2 * d if Fh is None else Fh,
                         W.WHALE_BF16 if dtype == "bf16" else W.WHALE_FP32, flags, 1e-6)


def _ws(nbytes):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=DEV)


@pytest.mark.parametrize("rows,d", [(1, 64), (127, 128), (129, 256), (1000, 512), (5000, 128), (40000, 256)])
def test_project_queries_and_kv(rows, d):
    rng = np.random.default_rng(rows + d)
    x = bf16_randn(rng, rows, d)
    g = rng.uniform(0.5, 1.5, d).astype(np.float32)
    wq = I.bf16_round(I.xavier_uniform(rng, d, d))
    wkv = I.bf16_round(np.concatenate([I.xavier_uniform(rng, d, d), I.xavier_uniform(rng, d, d)]))
    cfg = _cfg(d, d // 64 if d >= 128 else 2)
    ws = _ws(64 << 20)
    q = torch.empty(rows, d, dtype=torch.bfloat16, device=DEV)
    kv = torch.empty(rows, 2 * d, dtype=torch.bfloat16, device=DEV)
    xt = _t(x)
    W.whale_project_queries(cfg, rows, xt, _g(g), _t(wq), q, ws)
    W.whale_project_kv(cfg, rows, xt, _g(g), _t(wkv), kv, ws)
    torch.cuda.synchronize()
    xn = O.rms_norm(x, g, 1e-6)
    assert_parity(q, O.linear(xn, wq), "bf16", rms_rel=1e-2, what="Q")
    assert_parity(kv, O.linear(xn, wkv), "bf16", rms_rel=1e-2, what="KV")


def test_project_kv_shared_and_fp32():
    rng = np.random.default_rng(7)
    rows, d = 300, 128
    x = bf16_randn(rng, rows, d)
    g = rng.uniform(0.5, 1.5, d).astype(np.float32)
    wk = I.bf16_round(I.xavier_uniform(rng, d, d))
    kv = torch.empty(rows, d, dtype=torch.bfloat16, device=DEV)
    W.whale_project_kv(_cfg(d, 4, flags=W.WHALE_SHARED_KV), rows, _t(x), _g(g), _t(wk), kv, _ws(1 << 20))
    torch.cuda.synchronize()
    assert_parity(kv, O.linear(O.rms_norm(x, g, 1e-6), wk), "bf16", rms_rel=1e-2, what="K (shared)")
    # fp32 mode
    x32 = rng.standard_normal((rows, 64)).astype(np.float32)
    g32 = rng.uniform(0.5, 1.5, 64).astype(np.float32)
    w32 = np.concatenate([I.xavier_uniform(rng, 64, 64), I.xavier_uniform(rng, 64, 64)])
    kv32 = torch.empty(rows, 128, dtype=torch.float32, device=DEV)
    W.whale_project_kv(_cfg(64, 2, dtype="fp32"), rows, _t(x32, "fp32"), _g(g32), _t(w32, "fp32"), kv32, _ws(1 << 20))
    torch.cuda.synchronize()
    assert_parity(kv32, O.linear(O.rms_norm(x32, g32, 1e-6), w32), "fp32", what="KV fp32")


ATTN_CASES = [
    # (N, d, heads, lengths)
    (16, 128, 4, [0, 1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 257, 1000, 3000]),
    (32, 512, 8, [1, 31, 32, 33, 127, 128, 129, 500, 5000]),
    (32, 256, 8, [3, 700, 4000, 0, 6000]),
    (8, 256, 8, [5, 300, 2000]),
    (1, 64, 2, [1, 17, 1000]),
    (100, 256, 8, [1, 90, 2500]),
    (64, 512, 8, [40, 300]),
]


def _attn_ref(q, kv, off, N, d, h, shared=False):
    out = np.zeros((len(off) - 1, N, d))
    for b in range(len(off) - 1):
        k = kv[off[b]:off[b + 1], :d]
        v = k if shared else kv[off[b]:off[b + 1], d:2 * d]
        out[b] = O.cross_attention(q[b * N:(b + 1) * N], k, v, h)
    return out.reshape(-1, d)


@pytest.mark.parametrize("N,d,h,lengths", ATTN_CASES)
def test_cross_attention_bf16(N, d, h, lengths):
    rng = np.random.default_rng(N * 1000 + d)
    L = np.array(lengths, dtype=np.int64)
    off = I.offsets_of(L)
    B, total = len(L), int(off[-1])
    q = bf16_randn(rng, B * N, d)
    kv = bf16_randn(rng, max(total, 1), 2 * d)
    cfg = _cfg(d, h, N=N)
    hint = W.make_hint(B, int(L.max()), total)
    a = torch.empty(B * N, d, dtype=torch.bfloat16, device=DEV)
    ws = _ws(W.whale_workspace_size(cfg, hint))
    W.whale_cross_attention(cfg, _t(q), _t(kv), torch.from_numpy(off).to(DEV), a, hint, ws)
    torch.cuda.synchronize()
    assert_parity(a, _attn_ref(q, kv, off, N, d, h), "bf16", rms_rel=1e-2, what="A")


QTILE_CASES = [
    # many queries per history: the query-tiled kernel (N >= 128); ragged query tiles, empty and
    # one-row histories, blocks of 128 history rows with ragged tails, d_head 32 and 64
    (128, 256, 8, [1, 127, 128, 129, 0, 700]),
    (160, 256, 8, [300, 1, 2049]),
    (256, 512, 8, [129, 0, 1500]),
    (200, 128, 2, [64, 1000]),
]


@pytest.mark.parametrize("N,d,h,lengths", QTILE_CASES)
@pytest.mark.parametrize("shared", [False, True])
def test_cross_attention_many_queries(N, d, h, lengths, shared):
    rng = np.random.default_rng(N * 1000 + d + shared)
    L = np.array(lengths, dtype=np.int64)
    off = I.offsets_of(L)
    B, total = len(L), int(off[-1])
    q = bf16_randn(rng, B * N, d)
    kv = bf16_randn(rng, max(total, 1), (1 if shared else 2) * d)
    cfg = _cfg(d, h, N=N, flags=W.WHALE_SHARED_KV if shared else 0)
    hint = W.make_hint(B, int(L.max()), total)
    ws = _ws(W.whale_workspace_size(cfg, hint))
    offs = torch.from_numpy(off).to(DEV)
    a = torch.empty(B * N, d, dtype=torch.bfloat16, device=DEV)
    W.whale_cross_attention(cfg, _t(q), _t(kv), offs, a, hint, ws)
    torch.cuda.synchronize()
    assert_parity(a, _attn_ref(q, kv, off, N, d, h, shared), "bf16", rms_rel=1e-2, what="A (query tiles)")


def test_cross_attention_shared_kv_and_fp32():
    rng = np.random.default_rng(99)
    N, d, h = 32, 256, 8
    L = np.array([1, 400, 2000, 77])
    off = I.offsets_of(L)
    B, total = len(L), int(off[-1])
    q = bf16_randn(rng, B * N, d)
    k = bf16_randn(rng, total, d)
    cfg = _cfg(d, h, N=N, flags=W.WHALE_SHARED_KV)
    hint = W.make_hint(B, int(L.max()), total)
    a = torch.empty(B * N, d, dtype=torch.bfloat16, device=DEV)
    W.whale_cross_attention(cfg, _t(q), _t(k), torch.from_numpy(off).to(DEV), a, hint,
                            _ws(W.whale_workspace_size(cfg, hint)))
    torch.cuda.synchronize()
    assert_parity(a, _attn_ref(q, k, off, N, d, h, shared=True), "bf16", rms_rel=1e-2, what="A shared")
    # fp32 kernel, d_head 32
    N, d, h = 8, 64, 2
    L = np.array([0, 1, 130, 256])
    off = I.offsets_of(L)
    B, total = len(L), int(off[-1])
    q = rng.standard_normal((B * N, d)).astype(np.float32)
    kv = rng.standard_normal((total, 2 * d)).astype(np.float32)
    cfg = _cfg(d, h, N=N, dtype="fp32")
    hint = W.make_hint(B, int(L.max()), total)
    a = torch.empty(B * N, d, dtype=torch.float32, device=DEV)
    W.whale_cross_attention(cfg, _t(q, "fp32"), _t(kv, "fp32"), torch.from_numpy(off).to(DEV), a, hint,
                            _ws(W.whale_workspace_size(cfg, hint)))
    torch.cuda.synchronize()
    assert_parity(a, _attn_ref(q, kv, off, N, d, h), "fp32", what="A fp32")


@pytest.mark.parametrize("rows,d,Fh", [(1000, 128, 256), (333, 512, 1024), (130, 256, 0)])
def test_fusion_mlp(rows, d, Fh):
    rng = np.random.default_rng(rows + Fh)
    a, x = bf16_randn(rng, rows, d), bf16_randn(rng, rows, d)
    if Fh:
        w1 = I.bf16_round(I.xavier_uniform(rng, Fh, 2 * d))
        w2 = I.bf16_round(I.xavier_uniform(rng, d, Fh))
    else:
        w1, w2 = None, I.bf16_round(I.xavier_uniform(rng, d, 2 * d))
    cfg = _cfg(d, d // 64, Fh=Fh)
    f = torch.empty(rows, d, dtype=torch.bfloat16, device=DEV)
    W.whale_fusion_mlp(cfg, rows, _t(a), _t(x), None if w1 is None else _t(w1), _t(w2), f, _ws(64 << 20))
    torch.cuda.synchronize()
    assert_parity(f, O.fusion_mlp(a, x, w1, w2), "bf16", rms_rel=1e-2, what="F")


@pytest.mark.parametrize("rows,d,tied", [(1000, 128, False), (257, 512, False), (300, 256, True)])
def test_swiglu_ffn(rows, d, tied):
    rng = np.random.default_rng(rows + d + tied)
    H = 4 * d
    f = bf16_randn(rng, rows, d)
    g = rng.uniform(0.5, 1.5, d).astype(np.float32)
    wu = I.bf16_round(I.xavier_uniform(rng, H, d))
    wug = wu if tied else np.concatenate([wu, I.bf16_round(I.xavier_uniform(rng, H, d))])
    wd = I.bf16_round(I.xavier_uniform(rng, d, H))
    cfg = _cfg(d, d // 64, flags=W.WHALE_TIED_GATE if tied else 0)
    y = torch.empty(rows, d, dtype=torch.bfloat16, device=DEV)
    W.whale_swiglu_ffn(cfg, rows, _t(f), _g(g), _t(wug), _t(wd), y, _ws(64 << 20))
    torch.cuda.synchronize()
    assert_parity(y, O.swiglu_ffn(f, g, wug, wd, 1e-6, tied_gate=tied), "bf16", rms_rel=1e-2, what="Y")


@pytest.mark.parametrize("rows,d,shared", [(70001, 512, False), (40000, 128, True)])
def test_project_kv_large(rows, d, shared):
    """The history-side K|V projection at sizes that take the persistent path: the 2-SM
    (cta_group::2, 256 x 256 tiles) kernel where the output width is a multiple of 256, the one-CTA
    kernel otherwise (shared K = V at d = 128: 128 output columns); ragged row counts."""
    rng = np.random.default_rng(rows + d)
    x = bf16_randn(rng, rows, d)
    g = rng.uniform(0.5, 1.5, d).astype(np.float32)
    wkv = I.bf16_round(I.xavier_uniform(rng, d, d)) if shared else \
        I.bf16_round(np.concatenate([I.xavier_uniform(rng, d, d), I.xavier_uniform(rng, d, d)]))
    kvw = wkv.shape[0]
    kv = torch.empty(rows, kvw, dtype=torch.bfloat16, device=DEV)
    W.whale_project_kv(_cfg(d, d // 64, flags=W.WHALE_SHARED_KV if shared else 0), rows, _t(x), _g(g), _t(wkv), kv,
                       _ws(64 << 20))
    torch.cuda.synchronize()
    sel = np.r_[0:300, rows // 2:rows // 2 + 300, rows - 300:rows]
    ref = O.linear(O.rms_norm(x[sel], g, 1e-6), wkv)
    assert_parity(kv[torch.from_numpy(sel).to(DEV)], ref, "bf16", rms_rel=1e-2, what="KV")


ABS_CASES = [
    # (N, d, heads, lengths): N * heads = 256 absorbed queries, d_head = 64
    (32, 512, 8, [1, 255, 256, 257, 0, 1024, 777, 3000]),
    (64, 256, 4, [300, 1, 2048, 129, 0]),
]


@pytest.mark.parametrize("N,d,h,lengths", ABS_CASES)
@pytest.mark.parametrize("shared", [False, True])
def test_attend_states_absorbed(N, d, h, lengths, shared):
    rng = np.random.default_rng(N * 7 + d + shared)
    L = np.array(lengths, dtype=np.int64)
    off = I.offsets_of(L)
    B, total = len(L), int(off[-1])
    q = bf16_randn(rng, B * N, d)
    s = bf16_randn(rng, max(total, 1), d)
    g = rng.uniform(0.5, 1.5, d).astype(np.float32)
    wkv = I.bf16_round(I.xavier_uniform(rng, d, d)) if shared else \
        np.concatenate([I.bf16_round(I.xavier_uniform(rng, d, d)), I.bf16_round(I.xavier_uniform(rng, d, d))])
    cfg = _cfg(d, h, N=N, flags=W.WHALE_SHARED_KV if shared else 0)
    hint = W.make_hint(B, int(L.max()), total)
    a = torch.empty(B * N, d, dtype=torch.bfloat16, device=DEV)
    ws = _ws(W.whale_workspace_size(cfg, hint))
    W.whale_attend_states(cfg, _t(q), _t(s), torch.from_numpy(off).to(DEV), {"g_kv": _g(g), "w_kv": _t(wkv)}, a,
                          hint, ws)
    torch.cuda.synchronize()
    k, v = O.project_kv(s[:total], g, wkv, 1e-6, shared_kv=shared)
    ref = np.zeros((B, N, d))
    for b in range(B):
        ref[b] = O.cross_attention(q[b * N:(b + 1) * N], k[off[b]:off[b + 1]], v[off[b]:off[b + 1]], h)
    assert_parity(a, ref.reshape(-1, d), "bf16", rms_rel=1e-2, what="A (absorbed)")
