"""The FMA-pipe exponential (ex2_poly2 in csrc/pa_ptx.cuh; no kernel calls it, it
measured slower than ex2.approx in the prefill softmax), checked on
the CPU: its coefficients are read out of the header, its steps (range reduction by the
1.5 * 2^23 shift, degree-3 polynomial by fused multiply-adds, exponent added to the
bits) are replayed in float32, and the result is compared with the exact 2^x.

The bound it must meet: relative error below 2^-13 (the probabilities it produces are
rounded to bf16 afterwards, relative 2^-9), and the polynomial must be within 1e-6 of
a fresh near-minimax fit, so that the committed constants are the fit they claim."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "paged_kv_cache_442_b200", "csrc", "pa_ptx.cuh")


def coefficients():
    src = open(HDR).read()
    body = src[src.index("ex2_poly2"):]
    m = re.search(r"c0 = ([0-9.e+-]+)f, c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f, c3 = ([0-9.e+-]+)f",
                  body)
    assert m, "coefficients not found"
    return [np.float32(float(g)) for g in m.groups()]


def fma32(a, b, c):
    """float32 fused multiply-add: the exact product of two float32 fits a float64, so
    one float64 add followed by one rounding to float32 models it (double rounding is
    possible in rare ties, far below the bound tested)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_poly_emulated(x):
    c0, c1, c2, c3 = coefficients()
    shift = np.float32(12582912.0)
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = fma32(p, f, np.full_like(f, c1))
    p = fma32(p, f, np.full_like(f, c0))
    bits = (t.view(np.int32).astype(np.int64) << 23) + p.view(np.int32).astype(np.int64)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.int32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001),
                        rng.uniform(-20.0, 8.0, 400000),
                        np.arange(-125, 9)]).astype(np.float32)
    got = ex2_poly_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 2.0 ** -13, rel.max()


def test_integers_and_clamp():
    got = ex2_poly_emulated(np.array([0.0, 1.0, 8.0, -1.0, -60.0], np.float32))
    assert np.allclose(got, [1.0, 2.0, 256.0, 0.5, 2.0 ** -60], rtol=2.0 ** -13)
    tiny = ex2_poly_emulated(np.array([-np.inf, -1000.0, -127.0], np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 2.0 ** -125)


def test_coefficients_are_the_near_minimax_fit():
    n = 20000
    f = 0.5 * np.cos(np.pi * (np.arange(n) + 0.5) / n)
    y = np.exp2(f)
    w = np.ones(n)
    for _ in range(60):
        a = np.vander(f, 4, increasing=True) / y[:, None]
        c, *_ = np.linalg.lstsq(a * w[:, None], w, rcond=None)
        err = (np.vander(f, 4, increasing=True) @ c) / y - 1
        w = w * (1 + 4 * np.abs(err) / np.abs(err).max())
    assert np.allclose([float(v) for v in coefficients()], c, atol=1e-6)
