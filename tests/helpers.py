"""Shared helpers for the GPU parity tests: tolerances and comparisons.

Tolerances (stated once, used everywhere):
  O (bf16)          |O - O_ref| <= 1e-2 + half a bf16 ulp of O_ref, elementwise
                    (the arithmetic budget is 1e-2; rounding the exact value to
                    the bf16 output adds up to half an ulp, which alone exceeds
                    1e-2 for |O| >= 4)
  dQ, dK, dV (fp32) max |G - G_ref| <= 1e-2
  L (fp32)          |L - L_ref| <= 1e-3 * max(|L_ref|, 1)
  FP8 path          5e-2 in place of 1e-2 for O, 5e-2 relative for L
Indexing (causal mask, block table) is checked bit-exactly elsewhere.
"""

import numpy as np
import torch

O_TOL = 1e-2
GRAD_TOL = 1e-2
LSE_RTOL = 1e-3
FP8_TOL = 5e-2


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def max_abs(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - b)))


def assert_close_abs(got, ref, tol, what):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = max_abs(got, ref)
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"
    return err


def bf16_half_ulp(x):
    """Half the spacing of bf16 values at |x| (8 significant bits)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(np.where(a > 0, a, 1.0))      # a = f * 2^e, f in [0.5, 1)
    return np.where(a > 0, np.exp2(e.astype(np.float64) - 9.0), 0.0)


def assert_bf16_close(got, ref, tol, what):
    """bf16 outputs: |got - ref| <= tol + half a bf16 ulp of ref, elementwise.

    The arithmetic budget is ``tol``; rounding the exact result to bf16 can by
    itself move it by half an ulp (0.0078 for |x| in [2, 4), 0.0156 in
    [4, 8)), which no bf16 output can avoid. Returns the plain max abs error."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    diff = np.abs(got - ref)
    bound = tol + bf16_half_ulp(ref)
    bad = diff > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements exceed tol+half-ulp; worst "
                           f"excess {float((diff - bound).max()):.3e}, max abs err {float(diff.max()):.3e}")
    return float(diff.max()) if diff.size else 0.0


def assert_lse_close(got, ref, rtol=LSE_RTOL, what="L"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref) / np.maximum(np.abs(ref), 1.0)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= rtol, f"{what}: max rel err {worst:.3e} > {rtol:.1e}"
    return worst
