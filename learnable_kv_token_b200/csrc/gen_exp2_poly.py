"""Fits the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the prefill softmax
to evaluate part of its exponentials on the FMA pipe instead of the special
function unit.

Method: argument reduction 2^x = 2^n * 2^f with n = round(x), f = x - n in
[-1/2, 1/2] (the integer part goes straight into the exponent field), and a
degree-3 least-squares fit of 2^f on 64 Chebyshev nodes, weighted by 1/2^f so
that it minimises the relative error (close to minimax), with the constant
term pinned to 1 so that 2^0 is exact.  Prints the
coefficients (highest degree first, as the Horner loop uses them) and the
maximum and mean relative error of the polynomial (fp32 coefficients,
evaluated in fp64) on a dense grid.
Run: python learnable_kv_token_b200/csrc/gen_exp2_poly.py
"""
import numpy as np

DEG = 3
k = np.arange(64)
f = 0.5 * np.cos((2 * k + 1) * np.pi / 128)          # Chebyshev nodes on [-1/2, 1/2]
wt = 1.0 / 2.0 ** f                                    # relative-error weights
A = np.stack([f ** i for i in range(1, DEG + 1)], axis=1) * wt[:, None]
c, *_ = np.linalg.lstsq(A, (2.0 ** f - 1.0) * wt, rcond=None)
coef = np.float32(np.concatenate([[1.0], c]))          # c0 = 1, c1..cDEG
grid = np.linspace(-0.5, 0.5, 200001)
rel = np.polyval(coef[::-1].astype(np.float64), grid) / 2.0 ** grid - 1.0
print(f"coefficients c{DEG}..c0:", ", ".join(f"{float(x):.9e}f" for x in coef[::-1]))
print(f"relative error: max {np.abs(rel).max():.3e}, mean {rel.mean():.3e}")
