"""Coefficients of the cubic that approximates 2^f on [-1/2, 1/2] in the
attention softmax's software exp2 (Cody-Waite style split x = n + f, n the
nearest integer; 2^x = 2^n * p(f)).

Method: weighted least squares on 4096 Chebyshev nodes of [-1/2, 1/2] with
weight 2^-f (so the fit minimises the relative error), which is close to the
minimax cubic.  Prints the float32 coefficients and the largest relative
error over a dense grid.  Run: python gen_exp2_poly.py
"""
import numpy as np

n = 4096
k = np.arange(n)
f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * n))          # Chebyshev nodes in [-1/2, 1/2]
y = np.exp2(f)
V = np.vander(f, 4, increasing=True)                       # 1, f, f^2, f^3
w = 1.0 / y
c, *_ = np.linalg.lstsq(V * w[:, None], y * w, rcond=None)
c32 = c.astype(np.float32)
g = np.linspace(-0.5, 0.5, 200001)
p = ((c32[3] * g + c32[2]) * g + c32[1]) * g + c32[0]
print("c0..c3 =", ", ".join(f"{v:.9e}f" for v in c32))
print("max relative error", np.max(np.abs(p / np.exp2(g) - 1)))
