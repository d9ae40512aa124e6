"""Fits the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the prefill softmax
to evaluate part of its exponentials on the FMA pipe instead of the special
function unit.

Method: argument reduction 2^x = 2^n * 2^f with n = round(x), f = x - n in
[-1/2, 1/2] (the integer part goes straight into the exponent field), and a
degree-5 least-squares fit of 2^f on 64 Chebyshev nodes (close to minimax),
with the constant term pinned to 1 so that 2^0 is exact.  Prints the
coefficients (highest degree first, as the Horner loop uses them) and the
maximum relative error of the fp64 polynomial on a dense grid.
Run: python learnable_kv_token_b200/csrc/gen_exp2_poly.py
"""
import numpy as np

DEG = 5
k = np.arange(64)
f = 0.5 * np.cos((2 * k + 1) * np.pi / 128)          # Chebyshev nodes on [-1/2, 1/2]
A = np.stack([f ** i for i in range(1, DEG + 1)], axis=1)
c, *_ = np.linalg.lstsq(A, 2.0 ** f - 1.0, rcond=None)
coef = np.concatenate([[1.0], c])                      # c0 = 1, c1..c5
grid = np.linspace(-0.5, 0.5, 200001)
approx = np.polyval(coef[::-1], grid)
rel = np.max(np.abs(approx / 2.0 ** grid - 1.0))
print("coefficients c5..c0:", ", ".join(f"{float(np.float32(x)):.9e}f" for x in coef[::-1]))
print(f"max relative error (fp64 polynomial): {rel:.3e}")
