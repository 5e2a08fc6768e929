"""The soft-cap's polynomial tanh (csrc/tanh_poly.cuh): the committed coefficients are what
the generator computes, and the polynomial meets its error bound against numpy's tanh, both
as fitted (float32 Horner steps in y^2, times y) and as the kernel evaluates it (coefficients
folded into the raw score, Estrin's order, float32)."""
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


def test_folded_coefficients_in_the_raw_score():
    # The kernel evaluates c log2(e) tanh(s cs) as s (b0 + b1 w + (b2 + b3 w + b4 w^2) w^2),
    # w = s^2, b_i = c log2(e) a_i cs^(2i+1) rounded to float32, all in float32 (Estrin's
    # order).  The base-2 capped score must stay within 1e-5 plus four float32 roundings of
    # its own size (2.4e-7 relative) over |s cs| <= 1/2 (LSE is checked to 1e-3), for caps
    # from 1 to 1000 at d = 64 and 128.
    a = _committed().astype(np.float64)
    for d in (64, 128):
        for cap in (1.0, 5.0, 50.0, 1000.0):
            cs = np.float32((1.0 / np.sqrt(d)) / cap)
            L = cap * np.log2(np.e)
            b = np.array([a[i] * L * float(cs) ** (2 * i + 1) for i in range(len(a))],
                         dtype=np.float32)
            assert np.all(np.abs(b) >= np.finfo(np.float32).tiny)   # all normal: path taken
            s = np.linspace(-0.5 / float(cs), 0.5 / float(cs), 200001).astype(np.float32)
            w = s * s
            u = b[1] * w + b[0]
            v = b[3] * w + b[2]
            z = w * w
            v = b[4] * z + v
            u = v * z + u
            x = (u * s).astype(np.float64)
            ref = L * np.tanh(s.astype(np.float64) * float(cs))
            assert np.all(np.abs(x - ref) <= 1e-5 + 2.4e-7 * np.abs(ref)), (
                d, cap, np.abs(x - ref).max())
