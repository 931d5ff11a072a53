"""The absorbed form of the attention's backward, checked against the fp64 backward oracle.

The CUDA forward never forms K or V: with r_t the RMSNorm row factor of history row t and g the
states' gain, the score of query (head j, token n) is s = r_t (H_t . qa) with
qa = diag(g) W_K,j^T q_j / sqrt(d_h), and the attention output is z W'_V,j^T with
z = sum_t p_t r_t H_t and W'_V,j = W_V,j diag(g). Differentiating that form gives the quantities
a backward kernel in the same layout would compute, per example:

  dz  = dA_j W'_V,j                       dW'_V,j = dA_j^T z
  dp  = r_t (dz . H_t)                    delta   = dz . z   (= sum_t p dp)
  ds  = p (dp - delta)                    dqa     = sum_t ds r_t H_t
  dH_t = r_t sum_q (ds qa + p dz) - (r_t^2 H_t / d) sum_q (ds s + p dp)   (the second term: r_t;
         its row sum equals H_t . (the first term), so it needs no reduction over queries)

and the weight and gain gradients from dqa, q, dA and z alone (no pass over the history). This
test states those formulas in plain numpy and checks them against oracle/whale_backward.py (which
differentiates the K|V form and is pinned to finite differences), so the layout the backward
kernels will use is fixed before they are written. CPU only.
"""
import numpy as np
import pytest

from oracle import whale_backward as BW
from oracle import whale_oracle as O


def _absorbed_backward(q, H, g, w_k, w_v, dA, n_heads, eps):
    n, d = q.shape
    dh = d // n_heads
    r = 1.0 / np.sqrt(np.mean(H * H, axis=1) + eps)  # [L]
    dq = np.zeros_like(q)
    dH = np.zeros_like(H)
    dwk, dwv, dg = np.zeros_like(w_k), np.zeros_like(w_v), np.zeros(d)
    A = np.zeros_like(q)
    for j in range(n_heads):
        sl = slice(j * dh, (j + 1) * dh)
        wk, wv = w_k[sl], w_v[sl]  # [d_h, d]
        qk = q[:, sl] @ wk / np.sqrt(dh)  # [N, d]: W_K,j^T q_j / sqrt(d_h)
        qa = qk * g
        s = r[None, :] * (qa @ H.T)  # [N, L]
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        z = (p * r[None, :]) @ H  # [N, d]
        wpv = wv * g[None, :]  # W'_V,j
        A[:, sl] = z @ wpv.T
        # backward
        dz = dA[:, sl] @ wpv
        dwpv = dA[:, sl].T @ z
        dwv[sl] = dwpv * g[None, :]
        dg += np.sum(dwpv * wv, axis=0)
        dp = r[None, :] * (dz @ H.T)
        delta = np.sum(dz * z, axis=1, keepdims=True)
        ds = p * (dp - delta)
        dqa = (ds * r[None, :]) @ H
        dq[:, sl] = (dqa * g) @ wk.T / np.sqrt(dh)
        dwk[sl] = q[:, sl].T @ (dqa * g) / np.sqrt(dh)
        dg += np.sum(qk * dqa, axis=0)
        colsum = np.sum(ds * s + p * dp, axis=0)  # [L]
        dH += r[:, None] * (ds.T @ qa + p.T @ dz) - (r * r / d)[:, None] * H * colsum[:, None]
    return A, dq, dH, dwk, dwv, dg


@pytest.mark.parametrize("shared_kv", [False, True])
def test_absorbed_backward_matches_oracle(shared_kv):
    rng = np.random.default_rng(40 + shared_kv)
    n, L, d, heads, eps = 6, 11, 16, 4, 1e-3
    q = rng.standard_normal((n, d))
    H = rng.standard_normal((L, d)) * rng.uniform(0.5, 2.0, (L, 1))
    g = rng.uniform(0.5, 1.5, d)
    w_kv = rng.standard_normal((d if shared_kv else 2 * d, d)) * d ** -0.5
    w_k, w_v = (w_kv, w_kv) if shared_kv else (w_kv[:d], w_kv[d:])
    dA = rng.standard_normal((n, d))
    # oracle: K|V form
    k, v = O.project_kv(H, g, w_kv, eps, shared_kv)
    a_ref = O.cross_attention(q, k, v, heads)
    dq_ref, dk, dv = BW.cross_attention_backward(q, k, v, heads, dA)
    dH_ref, dg_ref, dwkv_ref = BW.project_kv_backward(H, g, w_kv, eps, dk, dv, shared_kv)
    # absorbed form
    A, dq, dH, dwk, dwv, dg = _absorbed_backward(q, H, g, w_k, w_v, dA, heads, eps)
    np.testing.assert_allclose(A, a_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dq, dq_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dH, dH_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dg, dg_ref, rtol=1e-10, atol=1e-12)
    dwkv = dwk + dwv if shared_kv else np.concatenate([dwk, dwv], axis=0)
    np.testing.assert_allclose(dwkv, dwkv_ref, rtol=1e-10, atol=1e-12)


def test_absorbed_backward_split_history_sums():
    """A history split between two CTA pairs: with the example's final softmax statistics, each
    part's ds, dqa and dH are its own rows' terms; dqa adds over the parts and dH needs no
    reduction (every query of the example is in the pair)."""
    rng = np.random.default_rng(42)
    n, L, d, heads, eps = 4, 9, 8, 2, 1e-3
    q, H = rng.standard_normal((n, d)), rng.standard_normal((L, d))
    g = rng.uniform(0.5, 1.5, d)
    w_k, w_v = rng.standard_normal((d, d)) * d ** -0.5, rng.standard_normal((d, d)) * d ** -0.5
    dA = rng.standard_normal((n, d))
    _, dq, dH, _, _, _ = _absorbed_backward(q, H, g, w_k, w_v, dA, heads, eps)
    dh = d // heads
    r = 1.0 / np.sqrt(np.mean(H * H, axis=1) + eps)
    dq_parts = np.zeros_like(dq)
    dH_parts = np.zeros_like(dH)
    for j in range(heads):
        sl = slice(j * dh, (j + 1) * dh)
        qk = q[:, sl] @ w_k[sl] / np.sqrt(dh)
        qa = qk * g
        s_full = r[None, :] * (qa @ H.T)
        m = s_full.max(axis=1, keepdims=True)
        l = np.exp(s_full - m).sum(axis=1, keepdims=True)  # final statistics of the example
        z = (np.exp(s_full - m) / l * r[None, :]) @ H
        dz = dA[:, sl] @ (w_v[sl] * g[None, :])
        delta = np.sum(dz * z, axis=1, keepdims=True)
        for lo, hi in ((0, 4), (4, L)):  # the two pairs' rows
            Hp, rp = H[lo:hi], r[lo:hi]
            s = rp[None, :] * (qa @ Hp.T)
            p = np.exp(s - m) / l
            dp = rp[None, :] * (dz @ Hp.T)
            ds = p * (dp - delta)
            dq_parts[:, sl] += ((ds * rp[None, :]) @ Hp * g) @ w_k[sl].T / np.sqrt(dh)
            colsum = np.sum(ds * s + p * dp, axis=0)
            dH_parts[lo:hi] += rp[:, None] * (ds.T @ qa + p.T @ dz) - (rp * rp / d)[:, None] * Hp * colsum[:, None]
    np.testing.assert_allclose(dq_parts, dq, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dH_parts, dH, rtol=1e-10, atol=1e-12)


def test_rmsnorm_term_from_the_dH_product_rows():
    """The RMSNorm term of dH needs no reduction over queries in the scoring pass: with
    dH_raw_t = r_t sum_q (ds qa + p dz) (the dH product itself), sum_q (ds s + p dp) = H_t . dH_raw_t,
    so dH_t = dH_raw_t - (r_t^2 / d) H_t (H_t . dH_raw_t): one dot product per history row in that
    product's epilogue."""
    rng = np.random.default_rng(43)
    n, L, d, heads, eps = 5, 8, 16, 2, 1e-3
    q, H = rng.standard_normal((n, d)), rng.standard_normal((L, d))
    g = rng.uniform(0.5, 1.5, d)
    w_k, w_v = rng.standard_normal((d, d)) * d ** -0.5, rng.standard_normal((d, d)) * d ** -0.5
    dA = rng.standard_normal((n, d))
    _, _, dH, _, _, _ = _absorbed_backward(q, H, g, w_k, w_v, dA, heads, eps)
    dh = d // heads
    r = 1.0 / np.sqrt(np.mean(H * H, axis=1) + eps)
    raw = np.zeros_like(H)
    for j in range(heads):
        sl = slice(j * dh, (j + 1) * dh)
        qa = q[:, sl] @ w_k[sl] / np.sqrt(dh) * g
        s = r[None, :] * (qa @ H.T)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        z = (p * r[None, :]) @ H
        dz = dA[:, sl] @ (w_v[sl] * g[None, :])
        dp = r[None, :] * (dz @ H.T)
        ds = p * (dp - np.sum(dz * z, axis=1, keepdims=True))
        raw_j = r[:, None] * (ds.T @ qa + p.T @ dz)
        np.testing.assert_allclose(np.sum(H * raw_j, axis=1), np.sum(ds * s + p * dp, axis=0), rtol=1e-10, atol=1e-12)
        raw += raw_j
    np.testing.assert_allclose(raw - (r * r / d)[:, None] * H * np.sum(H * raw, axis=1, keepdims=True), dH,
                               rtol=1e-10, atol=1e-12)
