"""Fits the degree-3 polynomial for 2^f on [-0.5, 0.5] that the softmax
kernels use on the FMA pipes (constants kExp2P0..kExp2P3 in ptx.cuh).

Method: Lawson's iteratively reweighted least squares towards the minimax
polynomial for relative error, on Chebyshev nodes; the coefficients are then
rounded to fp32 and the error re-measured with fp32 Horner evaluation.
Run: python fit_exp2_poly.py  (prints degree, coefficients, max rel error).
"""
import numpy as np
for deg in (3, 4):
    f = np.cos(np.linspace(0, np.pi, 4001)) * 0.5
    y = np.exp2(f)
    A = np.vander(f, deg + 1, increasing=True)
    w = np.ones_like(f)
    for it in range(300):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * (sw / y)[:, None], sw, rcond=None)
        err = (A @ c - y) / y
        w = w * np.abs(err); w /= w.sum()
    c32 = c.astype(np.float32)
    ff = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.full_like(ff, c32[-1])
    for k in range(deg - 1, -1, -1):
        p = (p * ff + c32[k]).astype(np.float32)
    rel = np.max(np.abs(p.astype(np.float64) / np.exp2(ff.astype(np.float64)) - 1))
    print(deg, [float(x) for x in c32], "max rel err fp32 horner:", rel)
