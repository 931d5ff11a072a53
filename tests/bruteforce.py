"""A second, independent formulation of one WHALE fusion layer for tiny inputs.

Pure-Python scalar loops over lists (math.exp, math.sqrt): per query, per head, per
history position, with the softmax written as exp(s) / sum exp(s) (no max shift) and
the concatenation [A ; H_w] written as explicit index arithmetic. It shares nothing
with oracle/whale_oracle.py (no numpy, no matmul, no helper in common), so a dropped
term, transposed operand or wrong index in either one shows up as a mismatch.
Only usable for tiny sizes (d <= 16, L <= 8).
"""
import math


def _dot(u, v):
    s = 0.0
    for i in range(len(u)):
        s += u[i] * v[i]
    return s


def _matvec(w, x):
    # w is a list of rows [out][in] (nn.Linear convention); returns w x
    return [_dot(row, x) for row in w]


def _rmsnorm(x, g, eps):
    ms = 0.0
    for xi in x:
        ms += xi * xi
    ms /= len(x)
    r = 1.0 / math.sqrt(ms + eps)
    return [x[i] * r * g[i] for i in range(len(x))]


def _silu(z):
    return z / (1.0 + math.exp(-z))


def layer_one_example(x, s, lw, n_heads, eps, shared_kv=False, tied_gate=False):
    """x: list of N rows (d floats); s: list of L rows; lw: dict of nested lists."""
    d = len(x[0])
    dh = d // n_heads
    wq, wkv = lw["w_q"], lw["w_kv"]
    wk = wkv[:d]
    wv = wkv[:d] if shared_kv else wkv[d:2 * d]
    keys, vals = [], []
    for t in range(len(s)):
        sn = _rmsnorm(s[t], lw["g_kv"], eps)
        keys.append(_matvec(wk, sn))
        vals.append(_matvec(wv, sn))
    out = []
    for n in range(len(x)):
        xn = _rmsnorm(x[n], lw["g_q"], eps)
        q = _matvec(wq, xn)
        a = [0.0] * d
        for j in range(n_heads):
            if not s:
                continue
            w = []
            for t in range(len(s)):
                sc = 0.0
                for c in range(j * dh, (j + 1) * dh):
                    sc += q[c] * keys[t][c]
                w.append(math.exp(sc / math.sqrt(dh)))
            z = sum(w)
            for c in range(j * dh, (j + 1) * dh):
                acc = 0.0
                for t in range(len(s)):
                    acc += (w[t] / z) * vals[t][c]
                a[c] = acc
        # Fusion MLP on the concatenation [a ; x]: index i < d reads a[i], i >= d reads x[n][i - d]
        cat = [a[i] if i < d else x[n][i - d] for i in range(2 * d)]
        if lw.get("w_f1") is None:
            mix = _matvec(lw["w_f2"], cat)
        else:
            hid = [_silu(v) for v in _matvec(lw["w_f1"], cat)]
            mix = _matvec(lw["w_f2"], hid)
        f = [x[n][i] + mix[i] for i in range(d)]
        nf = _rmsnorm(f, lw["g_ffn"], eps)
        hdim = len(lw["w_down"][0])
        up = _matvec(lw["w_upgate"][:hdim], nf)
        gate = up if tied_gate else _matvec(lw["w_upgate"][hdim:2 * hdim], nf)
        hh = [_silu(gate[i]) * up[i] for i in range(hdim)]
        dn = _matvec(lw["w_down"], hh)
        out.append([f[i] + dn[i] for i in range(d)])
    return out


def to_lists(lw):
    return {k: (None if v is None else (v.tolist() if hasattr(v, "tolist") else v)) for k, v in lw.items()}
