"""Backward pass of one fusion layer through whale_fusion_layer_backward against the fp64 VJP oracle
(oracle/whale_backward.py, itself pinned by finite differences of the forward oracle): every
gradient, d_tokens, d_states and each parameter's, summed over the batch. Reduced copies of the
training workloads (d = 128 with 4 heads of 32, d = 512 with 8 heads of 64, ragged histories, an
empty one, 16 tokens with histories over several 1024-row chunks), every variant (shared K = V, tied
gate, single-map Fusion MLP) and the fp32 mode.
Every case's worst error over bound, per tensor, goes to the JSON-lines file named by
WHALE_PARITY_REPORT when it is set.

Tolerances. bf16: every element within 2e-2 (1 + |oracle|) and a relative RMS error of at most 3e-2
per tensor (many gradients are far below 1 in size, where the element bound alone says little).
fp32: every element within 1e-4 (1 + |oracle|) (the gradients are sums over the batch, so the bound
scales with their size) and a relative RMS error of 1e-4."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import whale_backward as OB
from tests.gpu_util import to_np
from wukong_hstu_cross_b200 import inputs as I

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from wukong_hstu_cross_b200 import build
    build.build()
    from wukong_hstu_cross_b200 import harness as Hn
    from wukong_hstu_cross_b200 import whale as W


def _check(name, g, ref, dtype):
    g = np.asarray(g, np.float64)
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (name, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{name}: non-finite"
    tol, rms_tol = (2e-2, 3e-2) if dtype == "bf16" else (1e-4, 1e-4)
    err = np.abs(g - ref)
    bound = tol * (1.0 + np.abs(ref))
    if err.size and (err > bound).any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{name}: |gpu-oracle| {err[i]:.3e} > {bound[i]:.3e} at {i} (gpu {g[i]:.5g}, "
                             f"oracle {ref[i]:.5g}); {int((err > bound).sum())} elements out")
    nrm = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    if nrm > 0:
        rel = np.sqrt(np.mean(err ** 2)) / nrm
        assert rel <= rms_tol, f"{name}: relative RMS error {rel:.3e} > {rms_tol}"


def _oracle(p, dy):
    w = p.w
    flags = p.flags
    lw = p.host_weights[0]
    d_tok = np.zeros((w.batch, w.n_tokens, w.d))
    d_st = np.zeros((p.total_L, w.d))
    d_w = {k: np.zeros(np.shape(v)) for k, v in lw.items() if v is not None}
    for b in range(w.batch):
        lo, hi = int(p.offsets[b]), int(p.offsets[b + 1])
        s = I.states_of_example(w, 0, b, hi - lo)
        dx, ds, dlw = OB.fusion_layer_backward(I.tokens_of_example(w, b), s, lw, w.n_heads, w.eps, dy[b], **flags)
        d_tok[b] = dx
        d_st[lo:hi] = ds
        for k, v in dlw.items():
            d_w[k] += v
    return d_tok, d_st, d_w


# The workloads' training shapes, reduced (c2: d = 128 with 4 heads of 32; c4: d = 512 with 8 heads of
# 64), and every variant on one of them; the fp32 mode on the tiny workload.
CASES = {
    "tiny_fp32": ("tiny_fp32", dict(batch=3), {}),
    "d128_reduced": ("stack_d128", dict(batch=6, n_layers=1, lengths=("uniform", 1, 700)), {}),
    "d512_reduced": ("hist15k_d512", dict(batch=3, n_layers=1, lengths=("lognormal", 1500.0, 0.5, 64, 3000)), {}),
    "d128_shared_kv": ("stack_d128", dict(batch=4, n_layers=1, lengths=("uniform", 1, 900)), {"shared_kv": True}),
    "d512_tied_gate": ("hist15k_d512", dict(batch=3, n_layers=1, lengths=("uniform", 1, 900)), {"tied_gate": True}),
    "d512_shared_kv": ("hist15k_d512", dict(batch=3, n_layers=1, lengths=("uniform", 1, 1300)), {"shared_kv": True}),
    "d512_n16_long": ("hist15k_d512", dict(batch=2, n_layers=1, n_tokens=16, lengths=("uniform", 1100, 2600)), {}),
    "d128_single_map": ("stack_d128", dict(batch=4, n_layers=1, lengths=("uniform", 1, 900), fusion_mult=0), {}),
    "fp32_variants": ("tiny_fp32", dict(batch=3, fusion_mult=0), {"shared_kv": True, "tied_gate": True}),
}


@pytest.mark.parametrize("case", list(CASES))
def test_layer_backward_matches_oracle(case):
    base, over, flags = CASES[case]
    w = I.WORKLOADS[base].replace(**over)
    L = I.draw_lengths(w)
    if case == "d128_reduced":
        L[2] = 0  # an empty history: its queries get dq = 0 and its tokens only the non-attention terms
    p = Hn.build_problem(w, gains="random", lengths=L, **flags)
    rng = np.random.default_rng(7)
    dy = rng.standard_normal((w.batch, w.n_tokens, w.d)).astype(np.float32)
    out = Hn.run_layer_backward(p, 0, torch.from_numpy(dy).cuda())
    torch.cuda.synchronize()
    assert W.whale_get_device_error() == 0
    d_tok, d_st, d_w = _oracle(p, dy)
    refs = {"d_tokens": (to_np(out["d_tokens"]), d_tok), "d_states": (to_np(out["d_states"][:p.total_L]), d_st)}
    refs.update({k: (to_np(out[k]), v) for k, v in d_w.items()})
    tol = 2e-2 if w.dtype == "bf16" else 1e-4
    path = os.environ.get("WHALE_PARITY_REPORT")
    if path:
        worst = {k: float((np.abs(g - r) / (tol * (1 + np.abs(r)))).max()) for k, (g, r) in refs.items()}
        with open(path, "a") as fh:
            fh.write(json.dumps({"backward": case, "bound": f"{tol}*(1+|oracle|)", "max_err_over_bound": worst}) + "\n")
    for k, (g, r) in refs.items():
        _check(k, g, r, w.dtype)


def test_layer_backward_is_repeatable():
    """Two calls give the same parameter and state gradients bitwise where no atomics are involved
    (every gradient but those downstream of dq: d_tokens, w_q and g_q)."""
    w = I.WORKLOADS["stack_d128"].replace(batch=4, n_layers=1, lengths=("uniform", 100, 900))
    p = Hn.build_problem(w, gains="random")
    dy = torch.from_numpy(np.random.default_rng(3).standard_normal((w.batch, w.n_tokens, w.d)).astype(np.float32))
    a = Hn.run_layer_backward(p, 0, dy.cuda())
    b = Hn.run_layer_backward(p, 0, dy.cuda())
    torch.cuda.synchronize()
    for k in ("d_states", "w_kv", "g_kv", "w_f1", "w_f2", "g_ffn", "w_upgate", "w_down"):
        assert torch.equal(a[k], b[k]), k
    for k in ("d_tokens", "w_q", "g_q"):
        x, y = a[k].float(), b[k].float()
        assert bool(((x - y).abs() <= 1e-4 * (1 + y.abs())).all()), k


STACK_CASES = {
    "tiny_fp32_2layers": ("tiny_fp32", dict(batch=3, n_layers=2), {}),
    "d128_3layers": ("stack_d128", dict(batch=4, n_layers=3, lengths=("uniform", 1, 600)), {}),
    "d512_2layers": ("hist15k_d512", dict(batch=3, n_layers=2, lengths=("lognormal", 1500.0, 0.5, 64, 3000)), {}),
}


@pytest.mark.parametrize("case", list(STACK_CASES))
def test_stack_backward_matches_oracle(case):
    """The whole stack's backward (whale_fusion_backward) against the oracle's stack VJP: every
    layer's state and weight gradients and the tokens' gradient through all layers."""
    from oracle import whale_oracle as O  # noqa: F401  (the stack VJP below re-runs its forward)
    base, over, flags = STACK_CASES[case]
    w = I.WORKLOADS[base].replace(**over)
    L = I.draw_lengths(w)
    if case == "d128_3layers":
        L[1] = 0
    p = Hn.build_problem(w, gains="random", lengths=L, **flags)
    dy = np.random.default_rng(11).standard_normal((w.batch, w.n_tokens, w.d)).astype(np.float32)
    out = Hn.run_stack_backward(p, torch.from_numpy(dy).cuda())
    torch.cuda.synchronize()
    assert W.whale_get_device_error() == 0
    tokens = I.make_tokens(w)
    states = np.stack([I.make_states_layer(w, l, L, threads=4) for l in range(w.n_layers)])
    d_tok, d_st, d_w = OB.fusion_stack_backward(tokens, states, p.offsets, p.host_weights, w.n_heads, w.eps, dy,
                                                **flags)
    _check("d_tokens", to_np(out["d_tokens"]), d_tok, w.dtype)
    for l in range(w.n_layers):
        _check(f"d_states[{l}]", to_np(out["d_states"][l, :p.total_L]), d_st[l], w.dtype)
        for k, v in d_w[l].items():
            _check(f"{k}[{l}]", to_np(out["grads"][l][k]), v, w.dtype)


def test_layer_backward_full_size():
    """The 15k-history layer at full size (B 64, 403 481 history rows, random gains) against the fp64
    VJP on every element: d_tokens and d_states example by example, and each parameter's gradient (a
    sum over all examples). The oracle runs per example in a process pool."""
    from tests import oracle_pool
    w_name = "hist15k_d512"
    w = I.WORKLOADS[w_name].replace(n_layers=1)
    p = Hn.build_problem(w, gains="random")
    dy = np.random.default_rng(17).standard_normal((w.batch, w.n_tokens, w.d)).astype(np.float32)
    out = Hn.run_layer_backward(p, 0, torch.from_numpy(dy).cuda())
    torch.cuda.synchronize()
    assert W.whale_get_device_error() == 0
    d_tok = to_np(out["d_tokens"])
    d_st = to_np(out["d_states"][:p.total_L])
    lw = p.host_weights[0]
    d_w = {k: np.zeros(np.shape(v)) for k, v in lw.items() if v is not None}
    worst = {}
    seen = 0
    for b, dx, ds, dlw in oracle_pool.oracle_layer_backward(w_name, p.lengths, dy, gains="random",
                                                            overrides=(("n_layers", 1),)):
        lo, hi = int(p.offsets[b]), int(p.offsets[b + 1])
        _check(f"d_tokens[{b}]", d_tok[b], dx, "bf16")
        _check(f"d_states[{b}]", d_st[lo:hi], ds, "bf16")
        for k, v in dlw.items():
            d_w[k] += v
        for name, g, r in (("d_tokens", d_tok[b], dx), ("d_states", d_st[lo:hi], ds)):
            if r.size:
                worst[name] = max(worst.get(name, 0.0), float((np.abs(g - r) / (2e-2 * (1 + np.abs(r)))).max()))
        seen += 1
    assert seen == w.batch
    for k, v in d_w.items():
        g = to_np(out[k])
        _check(k, g, v, "bf16")
        worst[k] = float((np.abs(g - v) / (2e-2 * (1 + np.abs(v)))).max())
    path = os.environ.get("WHALE_PARITY_REPORT")
    if path:
        with open(path, "a") as fh:
            fh.write(json.dumps({"backward": f"{w_name} full size (B 64, total_L {p.total_L})",
                                 "bound": "2e-2*(1+|oracle|)", "max_err_over_bound": worst}) + "\n")
