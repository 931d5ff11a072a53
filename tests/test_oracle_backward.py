"""Pins of the fp64 backward oracle (oracle/whale_backward.py) against facts that do not come
from the backward oracle itself:

  * central finite differences of the forward oracle (pinned on its own in test_oracle_pins.py)
    for every input and every parameter of a fusion layer, in every variant (Fusion MLP with a
    hidden layer or the single linear map, shared K = V, tied gate), and of a two-layer stack;
  * closed forms of the attention's backward: a one-row history (a = v, so dq = dk = 0 and dV is
    the sum of the upstream gradients); an empty history (dq = 0);
  * invariants: adding one vector to every key leaves the softmax unchanged, so the keys'
    gradients sum to zero per head; the softmax weights of a query sum to one, so the value
    rows' gradients sum to the queries' upstream gradients; RMSNorm is scale invariant, so the
    states' gradient is orthogonal to the states (eps = 0).
CPU only.
"""
import numpy as np
import pytest

from oracle import whale_backward as BW
from oracle import whale_oracle as O


def _weights(rng, d, H, Fh, shared_kv=False, tied_gate=False):
    lw = {"g_q": rng.uniform(0.5, 1.5, d), "g_kv": rng.uniform(0.5, 1.5, d), "g_ffn": rng.uniform(0.5, 1.5, d),
          "w_q": rng.standard_normal((d, d)) * d ** -0.5,
          "w_kv": rng.standard_normal((d if shared_kv else 2 * d, d)) * d ** -0.5,
          "w_f1": None if Fh == 0 else rng.standard_normal((Fh, 2 * d)) * (2 * d) ** -0.5,
          "w_f2": rng.standard_normal((d, 2 * d if Fh == 0 else Fh)) * 0.3,
          "w_upgate": rng.standard_normal((H if tied_gate else 2 * H, d)) * d ** -0.5,
          "w_down": rng.standard_normal((d, H)) * H ** -0.5}
    return lw


def _fd(fun, arr, h=1e-6):
    """Central differences of the scalar fun() with respect to every element of arr (in place)."""
    g = np.zeros_like(arr)
    it = np.nditer(arr, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = arr[i]
        arr[i] = old + h
        fp = fun()
        arr[i] = old - h
        fm = fun()
        arr[i] = old
        g[i] = (fp - fm) / (2 * h)
    return g


def _close(got, want, tol=2e-6):
    scale = max(1.0, float(np.max(np.abs(want))))
    np.testing.assert_allclose(got, want, rtol=0, atol=tol * scale)


# ---------------------------------------------------------------------------------------------
# pieces
# ---------------------------------------------------------------------------------------------
def test_rms_norm_backward_finite_differences():
    rng = np.random.default_rng(10)
    x, g, dy = rng.standard_normal((3, 7)), rng.uniform(0.5, 1.5, 7), rng.standard_normal((3, 7))
    eps = 1e-3
    dx, dg = BW.rms_norm_backward(x, g, eps, dy)
    fun = lambda: float(np.sum(O.rms_norm(x, g, eps) * dy))
    _close(dx, _fd(fun, x))
    _close(dg, _fd(fun, g))


def test_silu_grad_finite_differences():
    z = np.linspace(-30.0, 30.0, 121)
    h = 1e-6
    _close(BW.silu_grad(z), (O.silu(z + h) - O.silu(z - h)) / (2 * h))
    assert BW.silu_grad(np.array([0.0]))[0] == 0.5  # sigmoid(0) (1 + 0)


@pytest.mark.parametrize("L", [1, 6])
def test_attention_backward_finite_differences(L):
    rng = np.random.default_rng(11 + L)
    n, d, heads = 3, 8, 2
    q, k, v = rng.standard_normal((n, d)), rng.standard_normal((L, d)), rng.standard_normal((L, d))
    da = rng.standard_normal((n, d))
    dq, dk, dv = BW.cross_attention_backward(q, k, v, heads, da)
    fun = lambda: float(np.sum(O.cross_attention(q, k, v, heads) * da))
    _close(dq, _fd(fun, q))
    _close(dk, _fd(fun, k))
    _close(dv, _fd(fun, v))


# ---------------------------------------------------------------------------------------------
# closed forms and invariants of the attention's backward
# ---------------------------------------------------------------------------------------------
def test_attention_backward_one_row_history_closed_form():
    rng = np.random.default_rng(12)
    n, d, heads = 4, 8, 2
    q, k, v, da = (rng.standard_normal(s) for s in ((n, d), (1, d), (1, d), (n, d)))
    dq, dk, dv = BW.cross_attention_backward(q, k, v, heads, da)
    assert np.all(dq == 0.0) and np.all(dk == 0.0)  # p = 1 whatever the scores
    np.testing.assert_allclose(dv[0], da.sum(axis=0), rtol=1e-14)


def test_attention_backward_empty_history():
    rng = np.random.default_rng(13)
    q, da = rng.standard_normal((3, 8)), rng.standard_normal((3, 8))
    dq, dk, dv = BW.cross_attention_backward(q, np.zeros((0, 8)), np.zeros((0, 8)), 2, da)
    assert dq.shape == (3, 8) and np.all(dq == 0.0) and dk.shape == (0, 8) and dv.shape == (0, 8)


def test_attention_backward_key_shift_and_value_sum_invariants():
    rng = np.random.default_rng(14)
    n, L, d, heads = 5, 9, 12, 3
    q, k, v, da = (rng.standard_normal(s) for s in ((n, d), (L, d), (L, d), (n, d)))
    dq, dk, dv = BW.cross_attention_backward(q, k, v, heads, da)
    # a is unchanged when one vector is added to every key row: sum_t dk_t = 0
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)
    # dv_t = sum_n p_nt da_n and sum_t p_nt = 1: sum_t dv_t = sum_n da_n
    np.testing.assert_allclose(dv.sum(axis=0), da.sum(axis=0), rtol=1e-12)
    # a is linear in v: <dv, v> = <da, a>
    a = O.cross_attention(q, k, v, heads)
    np.testing.assert_allclose(np.sum(dv * v), np.sum(da * a), rtol=1e-12)


def test_attention_backward_schedules_agree():
    """The KV-parallel and Q-parallel schedules are two orders of the same sums: splitting the
    queries into blocks (Q-parallel: dK, dV reduced over the blocks) or the history into blocks
    (KV-parallel: dQ reduced over the blocks, each block's softmax taken with the full row's
    normaliser) gives the unsplit gradients."""
    rng = np.random.default_rng(15)
    n, L, d, heads = 6, 10, 8, 2
    q, k, v, da = (rng.standard_normal(s) for s in ((n, d), (L, d), (L, d), (n, d)))
    dq, dk, dv = BW.cross_attention_backward(q, k, v, heads, da)
    # Q-parallel: every query block on its own, dK and dV summed over the blocks
    dk_q, dv_q = np.zeros_like(dk), np.zeros_like(dv)
    for lo in range(0, n, 4):
        bq, bk, bv = BW.cross_attention_backward(q[lo:lo + 4], k, v, heads, da[lo:lo + 4])
        np.testing.assert_allclose(bq, dq[lo:lo + 4], rtol=1e-12, atol=1e-14)
        dk_q += bk
        dv_q += bv
    np.testing.assert_allclose(dk_q, dk, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv_q, dv, rtol=1e-12, atol=1e-14)
    # KV-parallel: history blocks, each with the whole row's softmax statistics
    dh = d // heads
    dq_kv = np.zeros_like(dq)
    for j in range(heads):
        sl = slice(j * dh, (j + 1) * dh)
        s = q[:, sl] @ k[:, sl].T / np.sqrt(dh)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        delta = np.sum(da[:, sl] * (p @ v[:, sl]), axis=1, keepdims=True)  # rowsum(p * dp)
        for lo in range(0, L, 3):
            pb = p[:, lo:lo + 3]
            dsb = pb * (da[:, sl] @ v[lo:lo + 3, sl].T - delta)
            dq_kv[:, sl] += dsb @ k[lo:lo + 3, sl] / np.sqrt(dh)
            np.testing.assert_allclose(dsb.T @ q[:, sl] / np.sqrt(dh), dk[lo:lo + 3, sl], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(pb.T @ da[:, sl], dv[lo:lo + 3, sl], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dq_kv, dq, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------------------------
# whole layer and stack
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("Fh,shared_kv,tied_gate", [(6, False, False), (0, False, False), (6, True, False),
                                                    (6, False, True), (0, True, True)])
def test_layer_backward_finite_differences(Fh, shared_kv, tied_gate):
    rng = np.random.default_rng(20 + Fh + 2 * shared_kv + 4 * tied_gate)
    n, L, d, heads, H, eps = 3, 5, 8, 2, 12, 1e-3
    x, s, dy = rng.standard_normal((n, d)), rng.standard_normal((L, d)), rng.standard_normal((n, d))
    lw = _weights(rng, d, H, Fh, shared_kv, tied_gate)
    flags = {"shared_kv": shared_kv, "tied_gate": tied_gate}
    dx, ds, dlw = BW.fusion_layer_backward(x, s, lw, heads, eps, dy, **flags)
    fun = lambda: float(np.sum(O.fusion_layer(x, s, lw, heads, eps, **flags) * dy))
    _close(dx, _fd(fun, x))
    _close(ds, _fd(fun, s))
    keys = [key for key, val in lw.items() if val is not None]
    assert sorted(dlw) == sorted(keys)
    for key in keys:
        assert dlw[key].shape == lw[key].shape, key
        _close(dlw[key], _fd(fun, lw[key]))


def test_layer_backward_states_scale_invariance():
    """With eps = 0 the layer sees H_s only through RMSNorm(H_s), which is invariant to scaling
    each history row: every row of dH_s is orthogonal to that row of H_s."""
    rng = np.random.default_rng(30)
    n, L, d, heads, H = 4, 7, 8, 2, 12
    x, s, dy = rng.standard_normal((n, d)), rng.standard_normal((L, d)), rng.standard_normal((n, d))
    lw = _weights(rng, d, H, 6)
    _, ds, _ = BW.fusion_layer_backward(x, s, lw, heads, 0.0, dy)
    np.testing.assert_allclose(np.sum(ds * s, axis=1), 0.0, atol=1e-12)
    assert np.max(np.abs(ds)) > 1e-3


def test_stack_backward_finite_differences():
    rng = np.random.default_rng(31)
    B, n, d, heads, H, eps = 3, 2, 8, 2, 8, 1e-3
    lengths = [4, 0, 3]
    offsets = np.concatenate([[0], np.cumsum(lengths)])
    tokens = rng.standard_normal((B, n, d))
    states = rng.standard_normal((2, int(offsets[-1]), d))
    layers = [_weights(rng, d, H, 5), _weights(rng, d, H, 0)]
    dy = rng.standard_normal((B, n, d))
    dt, dst, dws = BW.fusion_stack_backward(tokens, states, offsets, layers, heads, eps, dy)
    fun = lambda: float(np.sum(O.fusion_stack(tokens, states, offsets, layers, heads, eps) * dy))
    _close(dt, _fd(fun, tokens))
    _close(dst, _fd(fun, states))
    for l, lw in enumerate(layers):
        for key, val in lw.items():
            if val is not None:
                _close(dws[l][key], _fd(fun, val))
