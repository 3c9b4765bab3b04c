"""Error bound of the attention kernel's software exp2 (optional FMA-pipe path).

The kernel's exp2_poly2() computes 2^x as 2^n * p(f) with n = round(x) (1.5*2^23 shifter),
f = x - n and a degree-3 polynomial p. Its coefficients come from exp2_poly_fit.py
(Chebyshev-node least squares of the relative error on [-1/2, 1/2]). This test re-derives
the fit, checks the constants in the kernel source match it, and emulates the kernel's
float32 steps to bound the relative error against the exact 2^x over the range the
softmax uses (x <= 8; arguments below -125 are clamped).
"""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "block_sparse_attention_tok_b200", "csrc")


def _kernel_coeffs():
    src = open(os.path.join(CSRC, "attn_sm100.cuh")).read()
    m = re.search(r"constexpr float c1 = ([0-9.e-]+)f, c2 = ([0-9.e-]+)f, c3 = ([0-9.e-]+)f;", src)
    assert m, "coefficients not found"
    return [np.float32(float(x)) for x in m.groups()]


def _fit():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(os.path.dirname(__file__), "exp2_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.fit(3)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly_emulated(x):
    c1, c2, c3 = _kernel_coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = _fma32(n, np.float32(-1.0) * np.ones_like(n), x)
    q = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    q = _fma32(q, f, np.full_like(f, c1))
    q = _fma32(q, f, np.ones_like(f))
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23)))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_kernel_coefficients_match_the_fit():
    coeffs, err = _fit()
    assert coeffs[0] == 1.0
    np.testing.assert_allclose(_kernel_coeffs(), np.float32(coeffs[1:]), rtol=0, atol=0)
    assert err < 1.5e-4


def test_emulated_exp2_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 9) + 0.5]).astype(np.float32)
    got = _exp2_poly_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 2e-4, rel.max()          # far below bf16's 2^-9 rounding of P
    assert _exp2_poly_emulated(np.float32([0.0]))[0] == 1.0
    assert np.all(_exp2_poly_emulated(np.float32([-1e30, -200.0])) < 1e-37)
