"""Helpers shared by the GPU parity tests: tolerances, conversions, comparisons.

Tolerances (bf16 inputs, fp32 accumulation, bf16 output, against the fp64 oracle):
O max-abs 2e-2 and mean-abs 2e-3; LSE max-abs 1e-3.  Tile maps are compared bit-exactly.

Every case is held to these fixed bounds.  Stress cases that need large scores draw Q and
K with a wider spread (std 2-3) and V from N(0,1), so the softmax is stressed while |O|
stays near 1.

The packed-document soft-cap workload draws Q, K and V from N(0,1)*2, and its scores (std
about 4) concentrate a row's weight on a few keys, so |O| reaches 6-8.  There the bf16
arithmetic alone can exceed 2e-2: rounding to bf16 (8-bit significand, round to nearest
even) errs by at most 2^-8 relative, once for each weight of P before the P V product and
once for O itself, so |O - O_ref| <= 2^-8 (|O_ref| + sum_j P_j |V_j|) per element, and the
fp32 accumulation and exponentials add orders of magnitude less.  ``o_bound`` passes that
derived per-element bound (with sum_j P_j |V_j| from the oracle on |V|); an element is
accepted when it is within 2e-2 or within its derived bound.  The mean and LSE bounds do
not change.
"""
import numpy as np
import torch

BF16_UNIT_ROUNDOFF = 2.0 ** -8

TOL_O_MAX = 2e-2
TOL_O_MEAN = 2e-3
TOL_LSE = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what="", o_bound=None):
    o = f64(o_gpu) if isinstance(o_gpu, torch.Tensor) else o_gpu
    l = f64(lse_gpu) if isinstance(lse_gpu, torch.Tensor) else lse_gpu
    assert o.shape == o_ref.shape, (what, o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite O"
    err = np.abs(o - o_ref)
    # rows with no visible key: O = 0 and LSE = -inf on both sides
    inf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(l), inf_ref), f"{what}: -inf LSE pattern differs"
    lerr = np.abs(np.where(inf_ref, 0.0, l - np.where(inf_ref, 0.0, lse_ref)))
    msg = (f"{what}: O max {err.max():.3e} mean {err.mean():.3e}; "
           f"LSE max {lerr.max() if lerr.size else 0:.3e}")
    if o_bound is None:
        assert err.max() <= TOL_O_MAX, msg
    else:
        assert np.all(err <= np.maximum(TOL_O_MAX, o_bound)), msg + (
            f" (derived bound at the worst element {o_bound.flat[np.argmax(err)]:.3e})")
    assert err.mean() <= TOL_O_MEAN, msg
    assert lerr.size == 0 or lerr.max() <= TOL_LSE, msg
    return err.max(), err.mean(), (lerr.max() if lerr.size else 0.0)


def sample_rows(N: int, rng: np.random.Generator, extra: int = 8) -> np.ndarray:
    base = [0, 1, 2, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1]
    rows = [r for r in base if 0 <= r < N] + list(rng.integers(0, N, size=extra))
    return np.unique(np.array(rows, dtype=np.int64))
