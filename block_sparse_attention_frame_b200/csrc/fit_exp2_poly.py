"""Derives the cubic used by the attention kernel's FMA-pipe exp2 (kExp2C0..kExp2C3).

p(f) ~ 2^f on f in [-1/2, 1/2], fitted by iteratively reweighted least squares on the
relative error (a Lawson-style approximation of the minimax fit), rounded to float32
and checked in float32 Horner form.  Run: python fit_exp2_poly.py
"""
import numpy as np
deg = 3
f = np.linspace(-0.5, 0.5, 20001)
y = np.exp2(f)
w = np.ones_like(f)
for it in range(200):
    A = np.vander(f, deg + 1, increasing=True) / y[:, None]
    c, *_ = np.linalg.lstsq(A * w[:, None], w, rcond=None)
    err = (np.vander(f, deg + 1, increasing=True) @ c) / y - 1
    w = w * (1 + 5 * np.abs(err) / np.abs(err).max())
    w /= w.mean()
c32 = c.astype(np.float32)
print("coeffs", [float(x) for x in c32], [x.hex() for x in map(float, c32)])
ff = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
p = np.float32(c32[3])
for k in (2, 1, 0):
    p = (p * ff + c32[k]).astype(np.float32)
rel = np.abs(p.astype(np.float64) / np.exp2(ff.astype(np.float64)) - 1)
print("max rel err (float32 Horner):", rel.max(), "bf16 half-ulp:", 2.0**-9)
