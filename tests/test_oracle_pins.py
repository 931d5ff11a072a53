"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
closed forms, a hand-derived worked example, the invariants the pages fix or imply
(softmax weights sum to 1, a single-key history returns its projected V, identical
keys reduce to the pages' average-pooling ablation, history order does not matter,
the concatenated up|gate SwiGLU equals the three-matmul form), brute force on tiny
inputs, and batch-composition invariance. CPU only.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import whale_oracle as O
from tests import bruteforce as BF
from wukong_hstu_cross_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _tiny_weights(rng, d, H, Fh, shared_kv=False, tied_gate=False, random_gain=True):
    def g():
        return rng.uniform(0.5, 1.5, d) if random_gain else np.ones(d)
    lw = {"g_q": g(), "g_kv": g(), "g_ffn": g(),
          "w_q": _rand(rng, d, d, scale=d ** -0.5),
          "w_kv": _rand(rng, d if shared_kv else 2 * d, d, scale=d ** -0.5),
          "w_f1": None if Fh == 0 else _rand(rng, Fh, 2 * d, scale=(2 * d) ** -0.5),
          "w_f2": _rand(rng, d, 2 * d if Fh == 0 else Fh, scale=0.3),
          "w_upgate": _rand(rng, H if tied_gate else 2 * H, d, scale=d ** -0.5),
          "w_down": _rand(rng, d, H, scale=H ** -0.5)}
    return lw


# ---------------------------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("c", [-3.0, 0.5, 7.25])
def test_rmsnorm_constant_row_closed_form(c):
    d, eps = 8, 1e-6
    g = np.linspace(0.5, 2.0, d)
    y = O.rms_norm(np.full((1, d), c), g, eps)
    np.testing.assert_allclose(y[0], g * c / math.sqrt(c * c + eps), rtol=1e-14)


def test_rmsnorm_unit_mean_square_and_scale_invariance():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 16))
    y = O.rms_norm(x, np.ones(16), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(O.rms_norm(3.5 * x, np.ones(16), 0.0), y, rtol=1e-13)


def test_linear_matches_triple_loop():
    rng = np.random.default_rng(1)
    x, w = rng.standard_normal((3, 5)), rng.standard_normal((4, 5))
    ref = [[sum(x[i, k] * w[o, k] for k in range(5)) for o in range(4)] for i in range(3)]
    np.testing.assert_allclose(O.linear(x, w), ref, rtol=1e-13)


def test_silu_identities():
    z = np.linspace(-6, 6, 25)
    np.testing.assert_allclose(O.silu(z) - O.silu(-z), z, atol=1e-14)   # z s(z) + z s(-z) = z
    assert O.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(O.silu(np.array([math.log(3.0)])), [0.75 * math.log(3.0)], rtol=1e-15)
    np.testing.assert_allclose(O.silu(np.array([40.0])), [40.0], rtol=1e-15)
    assert abs(O.silu(np.array([-40.0]))[0]) < 1e-15


# ---------------------------------------------------------------------------------------------
# attention invariants
# ---------------------------------------------------------------------------------------------
def test_softmax_weights_nonnegative_and_sum_to_one():
    rng = np.random.default_rng(2)
    q, k, v = rng.standard_normal((6, 8)), rng.standard_normal((11, 8)), rng.standard_normal((11, 8))
    _, probs = O.cross_attention(q * 4, k, v, n_heads=2, return_probs=True)
    for p in probs:
        assert p.shape == (6, 11)
        assert (p >= 0).all()
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)


def test_single_key_returns_projected_v():
    rng = np.random.default_rng(3)
    d, H = 8, 16
    lw = _tiny_weights(rng, d, H, 2 * d)
    x, s = rng.standard_normal((4, d)), rng.standard_normal((1, d))
    _, mid = O.fusion_layer(x, s, lw, n_heads=2, eps=1e-6, return_intermediates=True)
    # with one history row every query of every head returns that row's projected V exactly
    v1 = O.linear(O.rms_norm(s, lw["g_kv"], 1e-6), lw["w_kv"][d:])
    np.testing.assert_allclose(mid["a"], np.repeat(v1, 4, axis=0), rtol=1e-13, atol=1e-14)


def test_identical_keys_reduce_to_average_pooling():
    rng = np.random.default_rng(4)
    q, v = rng.standard_normal((5, 8)), rng.standard_normal((9, 8))
    k = np.repeat(rng.standard_normal((1, 8)), 9, axis=0)
    a = O.cross_attention(q, k, v, n_heads=4)
    np.testing.assert_allclose(a, np.repeat(v.mean(axis=0, keepdims=True), 5, axis=0), rtol=1e-13)


def test_zero_queries_layer_equals_average_pooling_ablation():
    """W_Q = 0 makes every score 0, so the layer equals the pages' ablation in which the
    attention is replaced by the mean of the history's value rows."""
    rng = np.random.default_rng(5)
    d, H, eps = 8, 16, 1e-6
    lw = _tiny_weights(rng, d, H, 2 * d)
    lw["w_q"] = np.zeros((d, d))
    x, s = rng.standard_normal((3, d)), rng.standard_normal((7, d))
    y = O.fusion_layer(x, s, lw, n_heads=2, eps=eps)
    v = O.rms_norm(s, lw["g_kv"], eps) @ lw["w_kv"][d:].T
    a_pool = np.repeat(v.mean(axis=0, keepdims=True), 3, axis=0)
    f = O.fusion_mlp(a_pool, x, lw["w_f1"], lw["w_f2"])
    np.testing.assert_allclose(y, O.swiglu_ffn(f, lw["g_ffn"], lw["w_upgate"], lw["w_down"], eps), rtol=1e-12)


def test_history_permutation_and_duplication_invariance():
    rng = np.random.default_rng(6)
    d, H = 8, 16
    lw = _tiny_weights(rng, d, H, 2 * d)
    x, s = rng.standard_normal((3, d)), rng.standard_normal((10, d))
    y = O.fusion_layer(x, s, lw, n_heads=2, eps=1e-6)
    perm = rng.permutation(10)
    np.testing.assert_allclose(O.fusion_layer(x, s[perm], lw, 2, 1e-6), y, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.fusion_layer(x, np.concatenate([s, s]), lw, 2, 1e-6), y, rtol=1e-12, atol=1e-13)


def test_hard_attention_limit_selects_argmax_row():
    rng = np.random.default_rng(7)
    q, k, v = rng.standard_normal((4, 4)), rng.standard_normal((6, 4)), rng.standard_normal((6, 4))
    a = O.cross_attention(q * 1e4, k, v, n_heads=1)
    expect = v[np.argmax(q @ k.T, axis=1)]
    np.testing.assert_allclose(a, expect, atol=1e-9)


def test_empty_history_gives_zero_attention():
    rng = np.random.default_rng(8)
    d = 8
    lw = _tiny_weights(rng, d, 16, 2 * d)
    x = rng.standard_normal((3, d))
    _, mid = O.fusion_layer(x, np.zeros((0, d)), lw, 2, 1e-6, return_intermediates=True)
    assert np.all(mid["a"] == 0.0)


# ---------------------------------------------------------------------------------------------
# Fusion MLP / SwiGLU
# ---------------------------------------------------------------------------------------------
def test_swiglu_concatenated_equals_three_matmul_form():
    rng = np.random.default_rng(9)
    d, H, eps = 8, 32, 1e-6
    f = rng.standard_normal((5, d))
    g = rng.uniform(0.5, 1.5, d)
    w_up, w_gate, w_down = rng.standard_normal((H, d)), rng.standard_normal((H, d)), rng.standard_normal((d, H))
    y = O.swiglu_ffn(f, g, np.concatenate([w_up, w_gate]), w_down, eps)
    n = f / np.sqrt((f * f).mean(-1, keepdims=True) + eps) * g
    up, gate = n @ w_up.T, n @ w_gate.T
    three = f + ((gate / (1 + np.exp(-gate))) * up) @ w_down.T
    np.testing.assert_allclose(y, three, rtol=1e-12)


def test_zero_output_projections_give_identities():
    rng = np.random.default_rng(10)
    d, H = 8, 32
    x, a, f = rng.standard_normal((3, d)), rng.standard_normal((3, d)), rng.standard_normal((3, d))
    np.testing.assert_array_equal(O.fusion_mlp(a, x, rng.standard_normal((16, 16)), np.zeros((d, 16))), x)
    np.testing.assert_array_equal(O.swiglu_ffn(f, np.ones(d), rng.standard_normal((2 * H, d)), np.zeros((d, H)), 1e-6), f)


def test_shared_kv_and_tied_gate_variants_equal_duplicated_weights():
    rng = np.random.default_rng(11)
    d, H = 8, 16
    lw = _tiny_weights(rng, d, H, 2 * d, shared_kv=True, tied_gate=True)
    dup = dict(lw, w_kv=np.concatenate([lw["w_kv"], lw["w_kv"]]),
               w_upgate=np.concatenate([lw["w_upgate"], lw["w_upgate"]]))
    x, s = rng.standard_normal((4, d)), rng.standard_normal((6, d))
    np.testing.assert_allclose(O.fusion_layer(x, s, lw, 2, 1e-6, shared_kv=True, tied_gate=True),
                               O.fusion_layer(x, s, dup, 2, 1e-6), rtol=1e-13)


# ---------------------------------------------------------------------------------------------
# whole layer: brute force, worked example, composition
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("n_heads,Fh,shared_kv,tied_gate,L", [
    (1, 16, False, False, 5), (2, 16, False, False, 3), (4, 0, False, False, 4),
    (2, 16, True, False, 2), (2, 16, False, True, 1), (2, 16, True, True, 6)])
def test_layer_matches_scalar_bruteforce(n_heads, Fh, shared_kv, tied_gate, L):
    rng = np.random.default_rng(100 + n_heads * 7 + Fh + L)
    d, H, eps = 8, 12, 1e-6
    lw = _tiny_weights(rng, d, H, Fh, shared_kv, tied_gate)
    x, s = rng.standard_normal((3, d)), rng.standard_normal((L, d))
    y = O.fusion_layer(x, s, lw, n_heads, eps, shared_kv=shared_kv, tied_gate=tied_gate)
    ref = BF.layer_one_example(x.tolist(), s.tolist(), BF.to_lists(lw), n_heads, eps, shared_kv, tied_gate)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


def _golden_value(v):
    if isinstance(v, str):
        return eval(v, {"__builtins__": {}}, {"ln3": math.log(3.0), "sqrt2": math.sqrt(2.0)})
    return float(v)


def _golden_array(a):
    return np.array([[_golden_value(v) for v in row] for row in a], dtype=np.float64)


@pytest.mark.parametrize("case", ["single_linear", "mlp"])
def test_hand_derived_worked_example(case):
    with open(os.path.join(GOLDEN, "worked_example_d2.json")) as fh:
        g = json.load(fh)
    c = g["cases"][case]
    lw = {"g_q": np.ones(2), "g_kv": np.ones(2), "g_ffn": np.ones(2),
          "w_q": _golden_array(c["w_q"]), "w_kv": _golden_array(c["w_kv"]),
          "w_f1": None if c["w_f1"] is None else _golden_array(c["w_f1"]),
          "w_f2": _golden_array(c["w_f2"]), "w_upgate": _golden_array(c["w_upgate"]),
          "w_down": _golden_array(c["w_down"])}
    x, s = np.array(g["x"]), np.array(g["s"])
    y, mid = O.fusion_layer(x, s, lw, g["n_heads"], g["eps"], return_intermediates=True)
    _, probs = O.cross_attention(mid["q"], mid["k"], mid["v"], 1, return_probs=True)
    np.testing.assert_allclose(probs[0][0], g["expected_probs"], rtol=1e-13)
    np.testing.assert_allclose(mid["a"][0], g["expected_a"], rtol=1e-13)
    np.testing.assert_allclose(y, _golden_array(c["expected_y"]), rtol=1e-13)


def test_stack_is_composition_of_layers_and_batch_invariant():
    w = I.small_workload("stack_d128", batch=4, n_tokens=3, d=16, n_heads=2, n_layers=2,
                         lengths=("uniform", 0, 5), dtype="fp32")
    lengths = I.draw_lengths(w)
    lengths[1] = 0                                        # one empty history in the batch
    off = I.offsets_of(lengths)
    toks = I.make_tokens(w)
    slabs = np.stack([I.make_states_layer(w, l, lengths, threads=1) for l in range(2)])
    lws = I.make_all_weights(w, gains="random")
    out = O.fusion_stack(toks, slabs, off, lws, w.n_heads, w.eps)
    for b in range(4):
        s0 = slabs[0][off[b]:off[b + 1]]
        s1 = slabs[1][off[b]:off[b + 1]]
        y = O.fusion_layer(O.fusion_layer(toks[b], s0, lws[0], 2, w.eps), s1, lws[1], 2, w.eps)
        np.testing.assert_allclose(out[b], y, rtol=1e-13)
    # reorder the batch: each example's output follows it
    perm = np.array([2, 0, 3, 1])
    L2 = lengths[perm]
    off2 = I.offsets_of(L2)
    slabs2 = np.stack([np.concatenate([slabs[l][off[p]:off[p + 1]] for p in perm]) for l in range(2)])
    out2 = O.fusion_stack(toks[perm], slabs2, off2, lws, 2, w.eps)
    np.testing.assert_allclose(out2, out[perm], rtol=1e-13)
