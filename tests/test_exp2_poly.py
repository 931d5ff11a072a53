"""The FMA-pipe exponential of the query-tiled attention's softmax (exp2_fma in
csrc/attention_qtile.cuh: a Cody-Waite reduction x = n + f with |f| <= 1/2, a degree-3 polynomial
for 2^f fitted for this kernel, 2^n put into the exponent bits). Its stated bound, relative error
at most 7.51e-5, is pinned by evaluating the same coefficients, read from the kernel source, with
the same float32 steps on the CPU against exact 2^x, over the softmax's whole range of arguments.
(The bound first stated, 7.5e-5, was a rounding of the true maximum, 7.502e-5 near f = 1/2: this
pin found it.)"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "wukong_hstu_cross_b200", "csrc",
                   "attention_qtile.cuh")
F32 = np.float32


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("float exp2_fma(float x)"):]
    body = body[:body.index("\n}")]
    c = [float(v) for v in re.findall(r"(-?\d+\.\d+)f", body)]
    # clamp, 1.5 * 2^23, then the four polynomial coefficients (highest degree first)
    assert c[0] == -125.0 and c[1] == 12582912.0, c
    return c[2:6]


def _fma(a, b, c):
    # float32 fused multiply-add: the float64 product of two float32 values is exact
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(F32)


def exp2_fma_host(x):
    c3, c2, c1, c0 = (F32(v) for v in _coefficients())
    xc = np.maximum(x.astype(F32), F32(-125.0))
    big = F32(12582912.0)
    t = (xc + big).astype(F32)
    f = (xc - (t - big).astype(F32)).astype(F32)
    p = _fma(_fma(_fma(np.full_like(f, c3), f, np.full_like(f, c2)), f, np.full_like(f, c1)), f, np.full_like(f, c0))
    n = t.view(np.int32) - big.view(np.int32)
    out = (p.view(np.int32) + (n << 23)).view(F32)
    return out, f


def test_reduction_keeps_the_fraction_in_half_open_unit():
    x = np.linspace(-125.0, 0.0, 2_000_001, dtype=np.float64).astype(F32)
    _, f = exp2_fma_host(x)
    assert np.all(np.abs(f) <= 0.5)
    # the reduction is exact: n + f reproduces x
    n = x - f
    assert np.all(n == np.round(n))


def test_relative_error_below_the_stated_bound():
    rng = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-125.0, 0.0, 4_000_001), rng.uniform(-40.0, 0.0, 1_000_000),
                        np.arange(-125, 1, dtype=np.float64)]).astype(F32)
    y, _ = exp2_fma_host(x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) - exact) / exact
    assert rel.max() < 7.51e-5, rel.max()
    # and it is a good fit, not a loose one: the error is not far below the bound either
    assert rel.max() > 1e-5


def test_integer_arguments_are_nearly_exact():
    x = np.arange(-125, 1, dtype=F32)
    y, f = exp2_fma_host(x)
    assert np.all(f == 0)
    rel = np.abs(y.astype(np.float64) - np.exp2(x.astype(np.float64))) / np.exp2(x.astype(np.float64))
    assert rel.max() < 1e-4
