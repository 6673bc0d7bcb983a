"""The attention kernels' FMA-pipe exponential (exp2_fma2 in csrc/attn_common.cuh), checked on
the CPU: its coefficients are those csrc/exp2_poly.py derives (Chebyshev interpolation of 2^f on
[-1/2, 1/2]), and the whole algorithm, replayed in numpy with fp32 roundings (the 1.5 * 2^23
shifter, Horner by fused multiply-adds, the exponent added as an integer), stays within 1.2e-4
relative error of 2^x for x in [-125, 0] and gives exactly 0 below -125."""

import os
import re

import numpy as np

from block_sparse_masked_segment_b200.csrc import exp2_poly

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "block_sparse_masked_segment_b200", "csrc", "attn_common.cuh")


def _kernel_coefficients():
    text = open(HEADER).read()
    m = re.search(r"kC0 = ([0-9.e+-]+)f, kC1 = ([0-9.e+-]+)f, kC2 = ([0-9.e+-]+)f, kC3 = ([0-9.e+-]+)f", text)
    assert m, "coefficients not found in attn_common.cuh"
    return np.array([float(g) for g in m.groups()], dtype=np.float32)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_fma(x):
    """exp2_fma2 step by step in fp32 (each fused multiply-add rounds once)."""
    c = _kernel_coefficients()
    x = x.astype(np.float32)
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = _fma32(n, np.float32(-1.0), x)
    p = _fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    p = _fma32(p, f, np.full_like(f, c[1]))
    p = _fma32(p, f, np.full_like(f, c[0]))
    with np.errstate(over="ignore"):
        bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    r = (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    return np.where(x >= -125.0, r, np.float32(0.0))


def test_coefficients_are_the_derived_ones():
    np.testing.assert_array_equal(_kernel_coefficients(), exp2_poly.coefficients())


def test_polynomial_error_on_the_reduced_interval():
    f = np.linspace(-0.5, 0.5, 100001)
    err = np.abs(exp2_poly.evaluate_fp32(_kernel_coefficients(), f) / np.exp2(f) - 1).max()
    assert err < 1.2e-4


def test_exp2_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 0.0, 400001), -np.random.default_rng(0).exponential(3.0, 100000)])
    x = x[x >= -125.0].astype(np.float32)
    got = _exp2_fma(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1.2e-4, rel.max()


def test_exp2_below_the_normal_range_and_minus_infinity_give_zero():
    x = np.array([-125.01, -126.0, -127.0, -150.0, -1e30, -np.inf], dtype=np.float32)
    np.testing.assert_array_equal(_exp2_fma(x), np.zeros_like(x))
