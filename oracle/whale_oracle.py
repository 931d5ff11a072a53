"""Float64 CPU oracle of the WHALE attention-fusion forward.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain statement of what the CUDA
path computes. Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg
may import it; the product path never does. It shares no code with the CUDA path.

Sources (the pages print no equations and no code; every step below is read from
their prose):

  [G] gist.science technical summary of WHALE, section 2.1 "Core Architecture"
      (Attention-Based Fusion Module: mechanism, refinement, propagation) and
      section 2.2 "Efficiency Optimizations" (shared key/value, shared-gate SwiGLU,
      BF16 backbone).
  [V] pith.science verdict, "key_machinery": the Wukong output is normalized and
      projected into queries; the HSTU output is normalized and projected into keys
      and values; a softmax attention yields one history vector per interaction
      representation; a fusion MLP concatenates that vector with the Wukong output
      and adds a residual; then a pre-norm SwiGLU FFN. Referee minor comments name
      the attention output Eq. (4) and the fused output Eq. (5), and say the Fusion
      MLP of Eq. (5) is a single linear projection of the concatenated vectors.
  [P] pith.science paper page, "What carries the argument" (Wukong queries attend
      over HSTU keys and values; residual Fusion MLP and pre-norm SwiGLU FFN blend
      the attended history with the interaction features) and the referee's major
      comment 1, which names the fusion parameters W_Q, W_K, W_V, W_F and the
      SwiGLU matrices.
  [D] paper-daily.com digest, section 2 (the attention output goes through the
      fusion MLP and the SwiGLU FFN and feeds the next layer; the shared gate cuts
      the FFN's three matmuls to two).

Readings taken where the pages are silent (each is also listed in the design notes):
  * "normalized" is RMSNorm with a gain g and eps (stats in float64 here);
  * no attention mask and no positional bias in the fusion attention: each query
    sees its own example's whole history (the relative bias belongs to HSTU);
  * scale 1/sqrt(d_head), multi-head split of the d columns into contiguous heads;
  * no output projection after the attention, no biases anywhere;
  * the Fusion MLP is (d+d) -> fusion_hidden -> d with SiLU on the hidden layer and
    the raw H_w as both the concatenated operand and the residual; fusion_hidden 0
    gives the pages' single linear projection;
  * between stacked layers the Wukong module is the identity: H_f of layer l is the
    query-side input of layer l+1, and each layer takes its own H_s slab;
  * an empty history (L_b = 0) attends to nothing: A = 0 for that example.

Parity pins for every function live in tests/test_oracle_pins.py. The paper's exact
Fusion MLP shape and norm type cannot be pinned from the pages: parity unpinned for
those two readings only.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g.   [V] "normalized"."""
    x = np.asarray(x, F64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, F64)


def linear(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y = x W^T with W stored [out, in] (no bias)."""
    return np.asarray(x, F64) @ np.asarray(w, F64).T


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z), written as z / (1 + exp(-z))."""
    z = np.asarray(z, F64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax, max-subtracted."""
    s = np.asarray(s, F64)
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def cross_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, n_heads: int,
                    return_probs: bool = False):
    """Eq. (4) as [G] 2.1 and [V] describe it: every query (a projected Wukong token)
    takes a softmax-weighted sum of its own example's value rows.

    q [N, d], k [L, d], v [L, d] -> a [N, d]. Heads split d into n_heads contiguous
    blocks of d/n_heads columns; head j uses q[:, j], k[:, j], v[:, j] only.
    Scores s = q_j k_j^T / sqrt(d_head); no mask, no bias. L = 0 gives a = 0.
    """
    q, k, v = np.asarray(q, F64), np.asarray(k, F64), np.asarray(v, F64)
    n, d = q.shape
    L = k.shape[0]
    dh = d // n_heads
    a = np.zeros((n, d), F64)
    probs = []
    for j in range(n_heads):
        sl = slice(j * dh, (j + 1) * dh)
        if L == 0:
            probs.append(np.zeros((n, 0), F64))
            continue
        p = softmax_rows(q[:, sl] @ k[:, sl].T / np.sqrt(dh))
        a[:, sl] = p @ v[:, sl]
        probs.append(p)
    return (a, probs) if return_probs else a


def fusion_mlp(a: np.ndarray, x: np.ndarray, w_f1, w_f2: np.ndarray) -> np.ndarray:
    """Eq. (5): F = H_w + FusionMLP([A ; H_w]).   [G] 2.1 "Refinement", [V] key_machinery.

    With w_f1 given: FusionMLP(c) = W_F2 SiLU(W_F1 c), W_F1 [Fh, 2d], W_F2 [d, Fh].
    With w_f1 None:  FusionMLP(c) = W_F c, W_F = w_f2 [d, 2d] (the pages' single linear map).
    """
    c = np.concatenate([np.asarray(a, F64), np.asarray(x, F64)], axis=-1)
    if w_f1 is None:
        return np.asarray(x, F64) + linear(c, w_f2)
    return np.asarray(x, F64) + linear(silu(linear(c, w_f1)), w_f2)


def swiglu_ffn(f: np.ndarray, g_ffn: np.ndarray, w_upgate: np.ndarray, w_down: np.ndarray,
               eps: float, tied_gate: bool = False) -> np.ndarray:
    """Pre-norm SwiGLU FFN with residual.   [G] 2.1 "Refinement", 2.2 shared-gate SwiGLU.

    n = RMSNorm(F; g_ffn);  Y = F + W_down (SiLU(W_gate n) * (W_up n)).
    w_upgate = [W_up ; W_gate] ([2H, d]) is applied as ONE matmul and split after it.
    tied_gate: w_upgate is W_up alone ([H, d]) and W_gate = W_up (two matmuls instead of three).
    """
    f = np.asarray(f, F64)
    nrm = rms_norm(f, g_ffn, eps)
    h = np.asarray(w_down).shape[1]
    ug = linear(nrm, w_upgate)
    if tied_gate:
        up, gate = ug, ug
    else:
        up, gate = ug[:, :h], ug[:, h:]
    return f + linear(silu(gate) * up, w_down)


def project_kv(s: np.ndarray, g_kv: np.ndarray, w_kv: np.ndarray, eps: float, shared_kv: bool = False):
    """K = RMSNorm(H_s) W_K^T, V = RMSNorm(H_s) W_V^T from one concatenated [W_K ; W_V].
    shared_kv: w_kv is W_K alone and V = K ([G] 2.2 "Shared Key-Value")."""
    sn = rms_norm(s, g_kv, eps)
    kv = linear(sn, w_kv)
    d = np.asarray(s).shape[-1]
    if shared_kv:
        return kv, kv
    return kv[:, :d], kv[:, d:]


def fusion_layer(x: np.ndarray, s: np.ndarray, lw: dict, n_heads: int, eps: float,
                 shared_kv: bool = False, tied_gate: bool = False, return_intermediates: bool = False):
    """One fusion module for one example.   [G] 2.1, [V] key_machinery, [P].

    x = H_w [N, d] (Wukong tokens), s = H_s [L, d] (that example's HSTU states).
      Q = RMSNorm(H_w; g_q) W_Q^T
      K, V = RMSNorm(H_s; g_kv) [W_K ; W_V]^T
      A = attention(Q, K, V)                          (Eq. 4)
      F = H_w + FusionMLP([A ; H_w])                  (Eq. 5)
      H_f = F + W_down(SiLU(W_gate n) * W_up n),  n = RMSNorm(F; g_ffn)
    """
    x = np.asarray(x, F64)
    q = linear(rms_norm(x, lw["g_q"], eps), lw["w_q"])
    k, v = project_kv(s, lw["g_kv"], lw["w_kv"], eps, shared_kv)
    a = cross_attention(q, k, v, n_heads)
    f = fusion_mlp(a, x, lw.get("w_f1"), lw["w_f2"])
    y = swiglu_ffn(f, lw["g_ffn"], lw["w_upgate"], lw["w_down"], eps, tied_gate)
    if return_intermediates:
        return y, {"q": q, "k": k, "v": v, "a": a, "f": f}
    return y


def fusion_stack_example(x: np.ndarray, slabs, layer_weights, n_heads: int, eps: float, **flags) -> np.ndarray:
    """Stacked layers for one example ([G] 2.1 "Propagation"): H_f of layer l is the
    query-side input of layer l+1; slabs[l] is this example's H_s for layer l."""
    y = np.asarray(x, F64)
    for l, lw in enumerate(layer_weights):
        y = fusion_layer(y, slabs[l], lw, n_heads, eps, **flags)
    return y


def fusion_stack(tokens: np.ndarray, seq_states: np.ndarray, offsets: np.ndarray, layer_weights,
                 n_heads: int, eps: float, **flags) -> np.ndarray:
    """Whole batch: tokens [B, N, d], seq_states [n_layers, sum L, d], offsets [B+1].
    Examples are independent; example b's history rows are [offsets[b], offsets[b+1])."""
    tokens = np.asarray(tokens)
    out = np.zeros(tokens.shape, F64)
    for b in range(tokens.shape[0]):
        lo, hi = int(offsets[b]), int(offsets[b + 1])
        slabs = [seq_states[l][lo:hi] for l in range(len(layer_weights))]
        out[b] = fusion_stack_example(tokens[b], slabs, layer_weights, n_heads, eps, **flags)
    return out
