"""Coefficients of the cubic that approximates 2^f on [-1/2, 1/2] in the attention
kernel's FMA-pipe exp2 (the rest of exp2(x) is an exponent shift by round(x)).

Weighted least squares for the relative error on 2001 Chebyshev points, then one
exchange-style refinement pass is unnecessary for the precision needed here: the codes
are FP4 and the row sum tolerates ~1e-4 relative error. Prints the coefficients (as
float32 hex) and the maximum relative error of the float32 evaluation.
"""
import numpy as np

k = np.arange(2001)
f = 0.5 * np.cos(np.pi * (k + 0.5) / 2001)           # Chebyshev points in [-1/2, 1/2]
target = np.exp2(f)
A = np.stack([np.ones_like(f), f, f ** 2, f ** 3], 1) / target[:, None]   # relative error
c, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
c32 = c.astype(np.float32)
ff = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
p = ((c32[3] * ff + c32[2]) * ff + c32[1]) * ff + c32[0]
err = np.abs(p.astype(np.float64) / np.exp2(ff.astype(np.float64)) - 1).max()
for i, v in enumerate(c32):
    print(f"c{i} = {float(v).hex()}  ({v!r})")
print("max relative error:", err)
