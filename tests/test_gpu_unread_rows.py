"""History rows that no example reads. The C ABI lets a slab hold more rows than the examples use
(offsets[B] < total_L). The forward never reads those rows: its output is the oracle's for the
examples' own rows, on the split-L, the query-tiled and the absorbed attention and in fp32 mode. Their
gradient is zero and they add nothing to the K|V weight and gain gradients: checked through
whale_fusion_layer_backward (bf16 with both attention backward kernels, d_head 32 and 64, and the
fp32 mode) and whale_fusion_backward (a two-layer stack, each layer's slab with its own unread rows)
against the fp64 VJP oracle. The unread rows hold random values. A batch of no examples over a
non-empty slab gets every gradient zero."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import whale_backward as OB
from oracle import whale_oracle as O
from tests.gpu_util import assert_parity, to_np
from tests.test_gpu_backward import _check, _oracle
from wukong_hstu_cross_b200 import inputs as I

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from wukong_hstu_cross_b200 import build
    build.build()
    from wukong_hstu_cross_b200 import harness as Hn
    from wukong_hstu_cross_b200 import whale as W

EXTRA = 300  # unread rows after the last example's


def _with_unread_rows(p, extra, seed):
    """The problem with `extra` random rows appended to every layer's slab, total_L raised to match
    (offsets unchanged) and the forward's workspace sized for it."""
    w = p.w
    T = p.total_L + extra
    tail = I.bf16_round(np.random.default_rng(seed).standard_normal((w.n_layers, extra, w.d)).astype(np.float32))
    states = torch.empty((w.n_layers, T, w.d), dtype=p.states.dtype, device=p.states.device)
    states[:, :p.total_L].copy_(p.states[:, :p.total_L])
    for l in range(w.n_layers):
        states[l, p.total_L:].copy_(Hn.to_device(tail[l], w, p.states.device))
    hint = W.make_hint(w.batch, int(p.lengths.max()), T)
    ws = torch.empty(W.whale_workspace_size(p.cfg, hint), dtype=torch.uint8, device=p.states.device)
    return dataclasses.replace(p, states=states, hint=hint, workspace=ws)


FORWARD_CASES = {
    "d128_splitl": ("stack_d128", dict(batch=4, n_layers=2, lengths=("uniform", 1, 500))),
    "d512_absorbed": ("hist15k_d512", dict(batch=3, n_layers=2, lengths=("uniform", 100, 900))),
    "d256_query_tiled": ("serve_15k", dict(n_tokens=16 * 16, n_layers=1, lengths=("fixed", 700))),
    "tiny_fp32": ("tiny_fp32", dict(batch=3)),
}


@pytest.mark.parametrize("case", list(FORWARD_CASES))
def test_forward_ignores_unread_rows(case):
    base, over = FORWARD_CASES[case]
    w = I.WORKLOADS[base].replace(**over)
    p = _with_unread_rows(Hn.build_problem(w, gains="random"), EXTRA, seed=4)
    out = Hn.run_forward(p).float().cpu().numpy()
    torch.cuda.synchronize()
    for b in range(w.batch):
        ref = O.fusion_stack_example(I.tokens_of_example(w, b), Hn.states_of_example_host(p, b), p.host_weights,
                                     w.n_heads, w.eps)
        assert_parity(out[b], ref, w.dtype, what=f"{case} example {b}")


LAYER_CASES = {
    "d128_bf16": ("stack_d128", dict(batch=3, n_layers=1, lengths=("uniform", 1, 400))),
    "d512_bf16": ("hist15k_d512", dict(batch=2, n_layers=1, lengths=("uniform", 100, 700))),
    "tiny_fp32": ("tiny_fp32", dict(batch=3)),
}


@pytest.mark.parametrize("case", list(LAYER_CASES))
def test_layer_backward_gives_unread_rows_zero_gradient(case):
    base, over = LAYER_CASES[case]
    w = I.WORKLOADS[base].replace(**over)
    p = Hn.build_problem(w, gains="random")
    q = _with_unread_rows(p, EXTRA, seed=5)
    dy = np.random.default_rng(9).standard_normal((w.batch, w.n_tokens, w.d)).astype(np.float32)
    out = Hn.run_layer_backward(q, 0, torch.from_numpy(dy).cuda())
    torch.cuda.synchronize()
    assert W.whale_get_device_error() == 0
    ds = to_np(out["d_states"])
    assert ds.shape == (p.total_L + EXTRA, w.d)
    assert np.all(ds[p.total_L:] == 0), float(np.abs(ds[p.total_L:]).max())
    d_tok, d_st, d_w = _oracle(p, dy)
    _check("d_tokens", to_np(out["d_tokens"]), d_tok, w.dtype)
    _check("d_states", ds[:p.total_L], d_st, w.dtype)
    for k, v in d_w.items():
        _check(k, to_np(out[k]), v, w.dtype)


def test_stack_backward_gives_unread_rows_zero_gradient():
    w = I.WORKLOADS["stack_d128"].replace(batch=3, n_layers=2, lengths=("uniform", 1, 400))
    p = Hn.build_problem(w, gains="random")
    q = _with_unread_rows(p, EXTRA, seed=6)
    dy = np.random.default_rng(10).standard_normal((w.batch, w.n_tokens, w.d)).astype(np.float32)
    out = Hn.run_stack_backward(q, torch.from_numpy(dy).cuda())
    torch.cuda.synchronize()
    assert W.whale_get_device_error() == 0
    tokens = I.make_tokens(w)
    states = np.stack([I.make_states_layer(w, l, p.lengths, threads=4) for l in range(w.n_layers)])
    d_tok, d_st, d_w = OB.fusion_stack_backward(tokens, states, p.offsets, p.host_weights, w.n_heads, w.eps, dy)
    _check("d_tokens", to_np(out["d_tokens"]), d_tok, w.dtype)
    for l in range(w.n_layers):
        ds = to_np(out["d_states"][l])
        assert np.all(ds[p.total_L:] == 0), (l, float(np.abs(ds[p.total_L:]).max()))
        _check(f"d_states[{l}]", ds[:p.total_L], d_st[l], w.dtype)
        for k, v in d_w[l].items():
            _check(f"{k}[{l}]", to_np(out["grads"][l][k]), v, w.dtype)


@pytest.mark.parametrize("base", ["stack_d128", "tiny_fp32"])
def test_backward_of_no_examples_is_zero(base):
    w = I.WORKLOADS[base].replace(batch=2, n_layers=1)
    p = Hn.build_problem(w, gains="random")
    cfg = Hn.config_of(w)
    T = p.total_L
    hint = W.make_hint(0, 0, T)   # no examples; the slab still has T rows
    lw = p.weights[0]
    grads = {k: torch.full(tuple(v.shape), float("nan"), dtype=torch.float32, device="cuda") for k, v in lw.items()
             if v is not None and k != "w_kabs"}
    d_states = torch.full((T, w.d), float("nan"), dtype=p.states.dtype, device="cuda")
    ws = torch.empty(max(W.whale_backward_workspace_size(cfg, hint), 256), dtype=torch.uint8, device="cuda")
    W.whale_fusion_layer_backward(cfg, None, p.states[0], p.offsets_t, lw, None, None, d_states, grads, hint, ws)
    torch.cuda.synchronize()
    assert bool((d_states.float() == 0).all())
    for k, g in grads.items():
        assert bool((g == 0).all()), k
