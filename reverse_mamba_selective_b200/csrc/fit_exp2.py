# Fits the polynomial used by the software exp2 of the scan kernel (scan_kernels.cuh, exp2_poly).
# Method: Cody-Waite style split x = n + f (n = round(x), |f| <= 1/2), 2^x = 2^n * p(f), with p a
# degree-5 polynomial whose max relative error on [-1/2, 1/2] is minimised by Lawson iteratively
# reweighted least squares.  Run: python fit_exp2.py  (prints the fp32 coefficients).
# Fit p(f) ~ 2^f on [-0.5, 0.5] minimising max relative error (Lawson IRLS), degree 5 and 6.
import numpy as np
f = np.cos(np.linspace(0, np.pi, 4001)) * 0.5
target = np.exp2(f)
for deg in (4, 5, 6):
    V = np.vander(f, deg + 1, increasing=True)
    w = np.ones_like(f)
    for it in range(400):
        sw = np.sqrt(w)[:, None]
        c, *_ = np.linalg.lstsq(V * sw / target[:, None], np.sqrt(w) * 1.0, rcond=None)
        err = (V @ c - target) / target
        w = w * np.abs(err); w /= w.sum()
    c32 = c.astype(np.float32).astype(np.float64)
    # evaluate with fp32 coefficients, fp64 arithmetic
    ff = np.linspace(-0.5, 0.5, 200001)
    p = np.zeros_like(ff)
    for k in range(deg, -1, -1):
        p = p * ff + c32[k]
    rel = np.max(np.abs(p / np.exp2(ff) - 1))
    # fp32 Horner with fma emulation via fp64 then round each step
    p32 = np.full_like(ff, np.float32(c32[deg]), dtype=np.float64)
    ff32 = ff.astype(np.float32).astype(np.float64)
    for k in range(deg - 1, -1, -1):
        p32 = (p32 * ff32 + c32[k]).astype(np.float32).astype(np.float64)
    rel32 = np.max(np.abs(p32 / np.exp2(ff32) - 1))
    print(deg, "coef-only rel err %.3g (2^%.1f), fp32 horner %.3g (2^%.1f)" % (rel, np.log2(rel), rel32, np.log2(rel32)))
    print("  ", [float(np.float32(v)) for v in c], [np.float32(v).view(np.uint32).item() for v in c])
