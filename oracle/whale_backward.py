"""Float64 CPU oracle of the WHALE attention-fusion BACKWARD pass (vector-Jacobian products).

TEST INFRASTRUCTURE ONLY, like the forward oracle beside it: only tests/, smoke() and the
benchmark's CPU-baseline leg may import it; the product path never does, and it shares no code
with the CUDA path.

What it states. For one fusion layer (the forward in whale_oracle.fusion_layer) and an upstream
gradient dY = dLoss/dH_f, the gradients of the loss with respect to the layer's inputs (H_w, H_s)
and to every parameter (g_q, W_Q, g_kv, [W_K ; W_V], W_F1, W_F2, g_ffn, [W_up ; W_gate], W_down),
obtained by running the forward's steps in reverse, each step's derivative written out by hand.

Sources:
  [G] gist.science technical summary of WHALE, section 2.2 "Efficiency Optimizations",
      "Asymmetric Backward Variants": few queries against a long history, so the training path
      picks a KV-parallel or a Q-parallel schedule for the attention's backward to cut the cost of
      reducing gradients.
  [D] paper-daily.com digest, section 2: the backward computation is split along the query
      dimension to save intermediate tensors and synchronisation.
Both schedules compute the same sums (dK and dV are sums over queries, dQ a sum over history
rows); they differ only in which of those sums is split across workers and reduced afterwards,
i.e. in the order of floating-point additions. The oracle therefore states the gradients once,
by their definition; a kernel with either schedule must match it up to rounding.

Readings: the same as the forward oracle's (RMSNorm with gain, no mask or bias, contiguous heads,
no output projection, Fusion MLP with SiLU hidden layer or the single linear map, identity between
layers). The loss is not part of the path: dY is an input.

Parity pins: tests/test_oracle_backward.py checks every gradient against central finite
differences of the (independently pinned) forward oracle, and the attention's gradients against
closed forms and invariants (one history row; shift of all keys; column sums of dV).
"""
from __future__ import annotations

import numpy as np

from .whale_oracle import F64, cross_attention, fusion_layer, fusion_mlp, linear, rms_norm, silu, softmax_rows


def rms_norm_backward(x: np.ndarray, g: np.ndarray, eps: float, dy: np.ndarray):
    """y = x * r * g with r = (mean(x^2) + eps)^(-1/2) over the last axis.

    dx_j = r (dy*g)_j - x_j r^3 / d * sum_i (dy*g)_i x_i ;  dg = sum over rows of dy * x * r.
    """
    x, g, dy = np.asarray(x, F64), np.asarray(g, F64), np.asarray(dy, F64)
    d = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    u = dy * g
    dx = r * u - x * (r ** 3) / d * np.sum(u * x, axis=-1, keepdims=True)
    dg = np.sum(dy * x * r, axis=tuple(range(x.ndim - 1)))
    return dx, dg


def linear_backward(x: np.ndarray, w: np.ndarray, dy: np.ndarray):
    """y = x W^T (W [out, in]): dx = dy W, dW = dy^T x."""
    x, w, dy = np.asarray(x, F64), np.asarray(w, F64), np.asarray(dy, F64)
    return dy @ w, dy.T @ x


def silu_grad(z: np.ndarray) -> np.ndarray:
    """d/dz [z sigmoid(z)] = sigmoid(z) (1 + z (1 - sigmoid(z)))."""
    z = np.asarray(z, F64)
    with np.errstate(over="ignore"):
        sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


def cross_attention_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, n_heads: int, da: np.ndarray):
    """Backward of Eq. (4) per head j (s = q_j k_j^T / sqrt(d_h), p = softmax_rows(s), a_j = p v_j):

      dp = da_j v_j^T,  dv_j = p^T da_j,  ds = p * (dp - rowsum(p * dp)),
      dq_j = ds k_j / sqrt(d_h),  dk_j = ds^T q_j / sqrt(d_h).

    dk and dv sum over the N queries (the reduction a Q-parallel schedule splits), dq over the L
    history rows (the one a KV-parallel schedule splits). An empty history has a = 0: dq = 0.
    """
    q, k, v, da = (np.asarray(t, F64) for t in (q, k, v, da))
    n, d = q.shape
    L = k.shape[0]
    dh = d // n_heads
    dq = np.zeros((n, d), F64)
    dk = np.zeros((L, d), F64)
    dv = np.zeros((L, d), F64)
    if L == 0:
        return dq, dk, dv
    for j in range(n_heads):
        sl = slice(j * dh, (j + 1) * dh)
        p = softmax_rows(q[:, sl] @ k[:, sl].T / np.sqrt(dh))
        dp = da[:, sl] @ v[:, sl].T
        dv[:, sl] = p.T @ da[:, sl]
        ds = p * (dp - np.sum(p * dp, axis=-1, keepdims=True))
        dq[:, sl] = ds @ k[:, sl] / np.sqrt(dh)
        dk[:, sl] = ds.T @ q[:, sl] / np.sqrt(dh)
    return dq, dk, dv


def fusion_mlp_backward(a: np.ndarray, x: np.ndarray, w_f1, w_f2: np.ndarray, dF: np.ndarray):
    """Backward of Eq. (5), F = H_w + FusionMLP([A ; H_w]). Returns (da, dx, dW_F1 or None, dW_F2);
    dx holds both the residual's and the concatenated operand's share."""
    a, x, dF = np.asarray(a, F64), np.asarray(x, F64), np.asarray(dF, F64)
    d = a.shape[-1]
    c = np.concatenate([a, x], axis=-1)
    if w_f1 is None:
        dc, dwf2 = linear_backward(c, w_f2, dF)
        dwf1 = None
    else:
        z = linear(c, w_f1)
        ds, dwf2 = linear_backward(silu(z), w_f2, dF)
        dz = ds * silu_grad(z)
        dc, dwf1 = linear_backward(c, w_f1, dz)
    return dc[:, :d], dF + dc[:, d:], dwf1, dwf2


def swiglu_ffn_backward(f: np.ndarray, g_ffn: np.ndarray, w_upgate: np.ndarray, w_down: np.ndarray,
                        eps: float, dy: np.ndarray, tied_gate: bool = False):
    """Backward of Y = F + W_down (SiLU(gate) * up), [up ; gate] = W_upgate RMSNorm(F; g_ffn).
    Tied gate: up = gate = W_up n, so both branches' gradients flow into the one matrix.
    Returns (dF, dg_ffn, dW_upgate, dW_down)."""
    f, dy = np.asarray(f, F64), np.asarray(dy, F64)
    nrm = rms_norm(f, g_ffn, eps)
    h = np.asarray(w_down).shape[1]
    ug = linear(nrm, w_upgate)
    up, gate = (ug, ug) if tied_gate else (ug[:, :h], ug[:, h:])
    m = silu(gate) * up
    dm, dwdown = linear_backward(m, w_down, dy)
    dup = dm * silu(gate)
    dgate = dm * up * silu_grad(gate)
    dug = dup + dgate if tied_gate else np.concatenate([dup, dgate], axis=-1)
    dn, dwug = linear_backward(nrm, w_upgate, dug)
    df_n, dg = rms_norm_backward(f, g_ffn, eps, dn)
    return dy + df_n, dg, dwug, dwdown


def project_kv_backward(s: np.ndarray, g_kv: np.ndarray, w_kv: np.ndarray, eps: float, dk: np.ndarray,
                        dv: np.ndarray, shared_kv: bool = False):
    """Backward of [K ; V] = RMSNorm(H_s; g_kv) [W_K ; W_V]^T (shared: V = K = RMSNorm(H_s) W_K^T).
    Returns (dH_s, dg_kv, dW_kv)."""
    sn = rms_norm(s, g_kv, eps)
    dkv = np.asarray(dk, F64) + np.asarray(dv, F64) if shared_kv else np.concatenate([dk, dv], axis=-1)
    dsn, dwkv = linear_backward(sn, w_kv, dkv)
    ds, dg = rms_norm_backward(s, g_kv, eps, dsn)
    return ds, dg, dwkv


def fusion_layer_backward(x: np.ndarray, s: np.ndarray, lw: dict, n_heads: int, eps: float, dy: np.ndarray,
                          shared_kv: bool = False, tied_gate: bool = False):
    """Gradients of one fusion layer (one example) for the upstream gradient dy = dLoss/dH_f.

    Returns (dx, ds, dlw): dx = dLoss/dH_w [N, d], ds = dLoss/dH_s [L, d], dlw the gradient of
    every entry of lw under the same key (w_f1 only when the layer has one).
    """
    x, s = np.asarray(x, F64), np.asarray(s, F64)
    # forward, keeping what the reverse steps need
    xn = rms_norm(x, lw["g_q"], eps)
    q = linear(xn, lw["w_q"])
    sn = rms_norm(s, lw["g_kv"], eps)
    kv = linear(sn, lw["w_kv"])
    d = x.shape[-1]
    k, v = (kv, kv) if shared_kv else (kv[:, :d], kv[:, d:])
    a = cross_attention(q, k, v, n_heads)
    f = fusion_mlp(a, x, lw.get("w_f1"), lw["w_f2"])
    # reverse
    dlw = {}
    df, dlw["g_ffn"], dlw["w_upgate"], dlw["w_down"] = swiglu_ffn_backward(
        f, lw["g_ffn"], lw["w_upgate"], lw["w_down"], eps, dy, tied_gate)
    da, dx, dwf1, dlw["w_f2"] = fusion_mlp_backward(a, x, lw.get("w_f1"), lw["w_f2"], df)
    if dwf1 is not None:
        dlw["w_f1"] = dwf1
    dq, dk, dv = cross_attention_backward(q, k, v, n_heads, da)
    dxn, dlw["w_q"] = linear_backward(xn, lw["w_q"], dq)
    dx_q, dlw["g_q"] = rms_norm_backward(x, lw["g_q"], eps, dxn)
    ds, dlw["g_kv"], dlw["w_kv"] = project_kv_backward(s, lw["g_kv"], lw["w_kv"], eps, dk, dv, shared_kv)
    return dx + dx_q, ds, dlw


def fusion_stack_backward(tokens: np.ndarray, seq_states: np.ndarray, offsets: np.ndarray, layer_weights,
                          n_heads: int, eps: float, dy: np.ndarray, **flags):
    """Whole batch and every layer: tokens [B, N, d], seq_states [n_layers, sum L, d], offsets
    [B + 1], dy [B, N, d] = dLoss/d(last layer's H_f). Layer l + 1's query-side input is layer l's
    H_f; each layer has its own H_s slab and weights.

    Returns (d_tokens [B, N, d], d_states [n_layers, sum L, d], d_weights: one dict per layer, the
    sum over the batch's examples)."""
    tokens = np.asarray(tokens, F64)
    seq_states = np.asarray(seq_states, F64)
    n_layers = len(layer_weights)
    d_tokens = np.zeros(tokens.shape, F64)
    d_states = np.zeros(seq_states.shape, F64)
    d_weights = [{key: np.zeros(np.shape(val), F64) for key, val in lw.items() if val is not None}
                 for lw in layer_weights]
    for b in range(tokens.shape[0]):
        lo, hi = int(offsets[b]), int(offsets[b + 1])
        xs = [tokens[b]]  # query-side input of every layer
        for l in range(n_layers - 1):
            xs.append(fusion_layer(xs[-1], seq_states[l][lo:hi], layer_weights[l], n_heads, eps, **flags))
        g = np.asarray(dy[b], F64)
        for l in reversed(range(n_layers)):
            g, ds, dlw = fusion_layer_backward(xs[l], seq_states[l][lo:hi], layer_weights[l], n_heads, eps, g,
                                               **flags)
            d_states[l][lo:hi] = ds
            for key, val in dlw.items():
                d_weights[l][key] += val
        d_tokens[b] = g
    return d_tokens, d_states, d_weights
