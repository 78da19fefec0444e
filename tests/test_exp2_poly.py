"""The FMA-pipe exp2 of the tensor-core kernels (exp2_poly.h, ex2_poly2 in
tc_common.cuh): its constants are the committed fit, and its float32
evaluation, emulated here step by step as the kernel does it (round-to-
nearest split by the 1.5 * 2^23 magic add, Horner with fused multiply-adds,
exponent insertion), matches 2^x to the accuracy of the MUFU ex2."""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(__file__), "..", "block_sparse_attention_sas_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_coeffs():
    text = open(os.path.join(CSRC, "exp2_poly.h")).read()
    vals = dict((int(k), float(v)) for k, v in re.findall(r"kExp2C(\d) = ([-+0-9.e]+)f;", text))
    return np.array([vals[i] for i in range(len(vals))], np.float32)


def _fma32(a, b, c):
    # a*b of two float32 values is exact in float64; one rounding to float32 after the add.
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _ex2_poly(x, c):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t + np.float32(-12582912.0)).astype(np.float32)
    f = _fma32(n, np.float32(-1.0) * np.ones_like(n), x)
    p = _fma32(np.full_like(f, c[5]), f, np.full_like(f, c[4]))
    for k in (3, 2, 1, 0):
        p = _fma32(p, f, np.full_like(f, c[k]))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_header_holds_the_fit():
    fit = _gen().coefficients().astype(np.float32)
    np.testing.assert_array_equal(_header_coeffs(), fit)
    assert fit[0] == 1.0


def test_relative_error_against_exp2():
    c = _header_coeffs()
    x = np.linspace(-124.9, 8.0, 400_001, dtype=np.float32)
    got = _ex2_poly(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - want) / want) < 5e-7


def test_integers_exact_and_clamp():
    c = _header_coeffs()
    k = np.arange(-124, 100, dtype=np.float32)
    np.testing.assert_array_equal(_ex2_poly(k, c), np.exp2(k.astype(np.float64)).astype(np.float32))
    tiny = _ex2_poly(np.array([-np.inf, -1e30, -200.0], np.float32), c)
    assert np.all(tiny > 0) and np.all(tiny <= 2.0 ** -124)


def test_halfway_points_continuous():
    # f flips from +1/2 to -1/2 across x = n + 1/2: both sides agree with 2^x.
    c = _header_coeffs()
    x = np.array([0.5, 1.5, -0.5, -3.5, 6.5], np.float32)
    for d in (-1e-6, 0.0, 1e-6):
        xx = (x + np.float32(d)).astype(np.float32)
        got = _ex2_poly(xx, c).astype(np.float64)
        want = np.exp2(xx.astype(np.float64))
        assert np.max(np.abs(got - want) / want) < 5e-7
