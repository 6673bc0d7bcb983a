"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on f in [-1/2, 1/2]
used by the attention kernels' FMA-pipe exponential (exp2_fma2 in attn_common.cuh).

Method: Chebyshev interpolation (the degree-3 interpolant at the 4 Chebyshev nodes of
[-1/2, 1/2], a near-minimax fit), converted to monomial form and rounded to fp32.  The
exponential's argument x is split as x = n + f with n = rint(x) (Cody and Waite's
additive range reduction), so 2^x = 2^n 2^f.

    python -m block_sparse_masked_segment_b200.csrc.exp2_poly   # prints the coefficients
"""

from __future__ import annotations

import numpy as np


def coefficients(degree: int = 3) -> np.ndarray:
    """Monomial coefficients (c0 .. c_degree) of the Chebyshev interpolant of 2^f on [-1/2, 1/2], as fp32."""
    k = np.arange(degree + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (degree + 1)))  # Chebyshev nodes on [-1/2, 1/2]
    vander = np.vander(nodes, degree + 1, increasing=True)
    c = np.linalg.solve(vander, np.exp2(nodes))
    return c.astype(np.float32)


def evaluate_fp32(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    """Horner evaluation in fp32 (each step one fused multiply-add, as the kernels do)."""
    f = f.astype(np.float32)
    acc = np.full_like(f, c[-1])
    for ci in c[-2::-1]:
        acc = (acc.astype(np.float64) * f + ci).astype(np.float32)  # fma: one rounding per step
    return acc


if __name__ == "__main__":
    c = coefficients()
    for i, x in enumerate(c):
        print(f"c{i} = {float(x):.9e}f  ({np.float32(x).view(np.uint32):#010x})")
    f = np.linspace(-0.5, 0.5, 200001)
    err = np.abs(evaluate_fp32(c, f) / np.exp2(f) - 1).max()
    print(f"max relative error on [-1/2, 1/2]: {err:.3e}")
