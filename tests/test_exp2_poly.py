"""The exp2 polynomial of the bf16 kernel, emulated in float32 on the CPU.

A third of the kernel's exponentials take 2^x on the FMA pipe instead of the MUFU
(``exp2_poly2`` in ``csrc/ptx.cuh``): Cody-Waite range reduction x = n + f with
n = rint(x) (the 1.5 * 2^23 shift) and f in [-1/2, 1/2], a degree-3 polynomial for
2^f whose coefficients minimise the maximum relative error (Remez exchange,
``csrc/fit_exp2_poly.py``), and 2^n added to the exponent field.  Here the same
float32 operation sequence is replayed in numpy and checked against ``np.exp2``:

* the relative error stays within the fitted bound (7.5e-5) wherever the result is a
  normal float, and the result is finite, non-negative and tiny below that;
* the kernel's hex constants are the ones the fit produces today (re-run here).
"""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "flash_attention_varlen_b200", "csrc", "ptx.cuh")
FIT = os.path.join(ROOT, "flash_attention_varlen_b200", "csrc", "fit_exp2_poly.py")
BOUND = 7.5e-5


def _kernel_source():
    src = open(PTX).read()
    body = src[src.index("float2 exp2_poly2("):]
    return body[:body.index("\n}\n")]


def _kernel_constants():
    """(clamp, [c3, c2, c1, c0]) as written in exp2_poly2, in Horner order."""
    body = _kernel_source()
    clamp = float(re.search(r"fmaxf\(x\.x, (-?[0-9.]+)f\)", body).group(1))
    hexes = re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", body)
    coef = []
    for h in hexes:  # each constant appears twice (both lanes of the pair)
        v = float.fromhex(h)
        if not coef or coef[-1] != v:
            coef.append(v)
    return clamp, coef


def _fma32(a, b, c):
    """float32 fused multiply-add: the f32 x f32 product is exact in float64."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_emulated(x, clamp, coef):
    """The kernel's operation sequence, lane by lane, in float32."""
    c3, c2, c1, c0 = (np.float32(c) for c in coef)
    x = np.maximum(np.asarray(x, np.float32), np.float32(clamp))
    shift = np.float32(12582912.0)
    xi = (x + shift).astype(np.float32)
    n = (xi - shift).astype(np.float32)
    f = _fma32(n, np.float32(-1.0), x)
    p = _fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.uint32) + (xi.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_within_the_fitted_bound():
    clamp, coef = _kernel_constants()
    assert len(coef) == 4
    # the kernel's arguments are s * c - m <= the rescale threshold (3), and as low as
    # the scores go; every float32 in [-120, 3] at a fine spacing plus the half-integers
    x = np.concatenate([np.linspace(-120.0, 3.0, 2_000_001, dtype=np.float32),
                        np.arange(-120.0, 3.5, 0.5, dtype=np.float32)])
    got = exp2_poly_emulated(x, clamp, coef).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= BOUND, f"max relative error {rel.max():.3e} at x = {x[rel.argmax()]}"


def test_far_below_the_running_max_gives_a_tiny_nonnegative_value():
    """Scores many binades below the row's running max (large scales, extreme logits):
    the result must stay finite, >= 0 and negligible next to the 1 at the max."""
    clamp, coef = _kernel_constants()
    x = np.concatenate([np.linspace(-1e4, -120.0, 200_001, dtype=np.float32),
                        np.array([-np.inf, -127.0, -126.99995, -126.5, -126.0, -125.5],
                                 np.float32)])
    got = exp2_poly_emulated(x, clamp, coef)
    assert np.all(np.isfinite(got)) and np.all(got >= 0.0)
    assert got.max() <= 2.0 ** -119


def test_kernel_constants_are_the_fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", FIT)
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c, err = fit.remez_exp2(3)
    c32 = [float(np.float32(v)) for v in c]
    _, coef = _kernel_constants()
    assert coef[::-1] == c32, (coef[::-1], c32)
    assert err <= BOUND
    assert fit.max_rel_err_f32(np.array(c32, np.float32)) <= BOUND


@pytest.mark.parametrize("clamp", [-127.0])
def test_the_old_clamp_is_caught(clamp):
    """A clamp at -127 lets n = -127 meet a polynomial value just below 1, and the
    exponent add then borrows into the sign bit (a NaN): the check above must see it."""
    _, coef = _kernel_constants()
    got = exp2_poly_emulated(np.array([-127.0], np.float32), clamp, coef)
    assert not (np.isfinite(got).all() and (got >= 0).all())
