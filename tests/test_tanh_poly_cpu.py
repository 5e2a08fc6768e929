"""The soft-cap's polynomial tanh (csrc/tanh_poly.cuh): the committed coefficients are what
the generator computes, and the polynomial meets its error bound against numpy's tanh when it
is evaluated the way the kernel evaluates it (float32 Horner steps in y^2, times y)."""
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
    y = np.linspace(-1.0, 1.0, 400001).astype(np.float32)
    w = y * y
    acc = np.full_like(w, c[-1])
    for ci in c[-2::-1]:
        acc = acc * w + ci
    err = np.abs((y * acc).astype(np.float64) - np.tanh(y.astype(np.float64)))
    # the soft-cap multiplies tanh by c log2(e) (72 for c = 50): 1.5e-7 in tanh is 1.1e-5 in
    # the base-2 score, far inside the 1e-3 LSE tolerance
    assert err.max() < 1.5e-7
    assert np.all(np.sign(y * acc) == np.sign(y))          # odd, no sign flips near 0
