"""The soft-cap's polynomial tanh (csrc/tanh_poly.cuh): the committed coefficients are what
the generator computes, and the polynomial meets its error bound against numpy's tanh, both
as fitted (float32 Horner steps in y^2, times y) and as the kernel evaluates it (coefficients
folded into the raw score, Horner's scheme in float32 multiply-adds, the reference max
subtracted in the last one) -- where a masked score, -inf, must stay -inf."""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "io_aware_softmax_b200", "csrc")


def _generator():
    spec = importlib.util.spec_from_file_location("gen_tanh_poly",
                                                  os.path.join(CSRC, "gen_tanh_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _committed():
    text = open(os.path.join(CSRC, "tanh_poly.cuh")).read()
    body = text[text.index("kTanhPoly[kTanhPolyTerms] = {"):]
    return np.array([float(x) for x in re.findall(r"(-?\d\.\d+(?:e-?\d+)?)f,", body)],
                    dtype=np.float32)


def test_header_holds_the_generated_fit():
    gen = _generator()
    assert np.array_equal(_committed(), gen.fit().astype(np.float32))


def test_polynomial_tanh_error_bound():
    c = _committed()
    y = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    w = y * y
    acc = np.full_like(w, c[-1])
    for ci in c[-2::-1]:
        acc = acc * w + ci
    err = np.abs((y * acc).astype(np.float64) - np.tanh(y.astype(np.float64)))
    assert err.max() < 1e-7
    assert np.all(np.sign(y * acc) == np.sign(y))          # odd, no sign flips near 0


def _fma(a, b, c):
    # float32 fused multiply-add: the exact product plus c, rounded once (float64 holds the
    # product of two float32 values exactly; the sum is rounded to float64 first, which
    # agrees with a single rounding except in ties far below the bounds checked here)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _horner(b, s):
    # the kernel's steps: w = s^2, t = b4 w + b3, then t w + b_i for i = 2, 1, 0
    w = (s * s).astype(np.float32)
    t = _fma(np.full_like(w, b[4]), w, np.full_like(w, b[3]))
    for i in (2, 1, 0):
        t = _fma(t, w, np.full_like(w, b[i]))
    return t


def test_folded_coefficients_in_the_raw_score():
    # The kernel evaluates c log2(e) tanh(s cs) as s (b0 + w (b1 + w (b2 + w (b3 + w b4)))),
    # w = s^2, b_i = c log2(e) a_i cs^(2i+1) rounded to float32, all in float32 with fused
    # multiply-adds (Horner's scheme); the last step also subtracts the row's reference max
    # m, t s - m in one multiply-add.  Over |s cs| <= 1/2 the base-2 capped score must stay
    # within 1e-5 plus 2.4e-7 of its own size (about four float32 roundings), for caps from 1
    # to 1000 at d = 64 and 128 (LSE is checked to 1e-3).
    a = _committed().astype(np.float64)
    assert a[-1] > 0        # a masked score, -inf, must come out of the polynomial as -inf
    for d in (64, 128):
        for cap in (1.0, 5.0, 50.0, 1000.0):
            cs = np.float32((1.0 / np.sqrt(d)) / cap)
            L = cap * np.log2(np.e)
            b = np.array([a[i] * L * float(cs) ** (2 * i + 1) for i in range(len(a))],
                         dtype=np.float32)
            assert np.all(np.abs(b) >= np.finfo(np.float32).tiny)   # all normal: path taken
            s = np.linspace(-0.5 / float(cs), 0.5 / float(cs), 200001).astype(np.float32)
            t = _horner(b, s)
            ref = L * np.tanh(s.astype(np.float64) * float(cs))
            x = (t * s).astype(np.float64)
            assert np.all(np.abs(x - ref) <= 1e-5 + 2.4e-7 * np.abs(ref)), (
                d, cap, np.abs(x - ref).max())
            m = np.float32(L * 0.3)                                  # a reference max
            xm = _fma(t, s, np.full_like(s, -m)).astype(np.float64)
            assert np.all(np.abs(xm - (ref - float(m))) <=
                          1e-5 + 2.4e-7 * (np.abs(ref) + float(m))), (
                d, cap, np.abs(xm - (ref - float(m))).max())
            with np.errstate(invalid="ignore", over="ignore"):
                neg_inf = np.array([-np.inf], dtype=np.float32)
                x_masked = _fma(_horner(b, neg_inf), neg_inf, np.array([-m], np.float32))
            assert x_masked[0] == -np.inf
