# Fits the polynomial used by the softplus of the scan kernel (scan_kernels.cuh, softplus_f).
# log1p(w) = w * q(w) on w in (0, 1]; q of degree 5..9 minimising the max relative error by
# Lawson iteratively reweighted least squares; the kernel uses degree 7.  Run: python fit_log1p.py
import numpy as np
w = (1 - np.cos(np.linspace(0, np.pi, 6001))) / 2  # [0,1] chebyshev-ish
w[0] = 1e-12
target = np.log1p(w) / w
for deg in (5, 6, 7, 8, 9):
    V = np.vander(w, deg + 1, increasing=True)
    wt = np.ones_like(w)
    for it in range(300):
        sw = np.sqrt(wt)[:, None]
        c, *_ = np.linalg.lstsq(V * sw / target[:, None], np.sqrt(wt), rcond=None)
        err = (V @ c - target) / target
        wt = wt * np.abs(err); wt /= wt.sum()
    c32 = c.astype(np.float32)
    ww = np.linspace(0, 1, 400001).astype(np.float32); ww[0] = np.float32(1e-30)
    p = np.full_like(ww, c32[deg], dtype=np.float32)
    for k in range(deg - 1, -1, -1):
        p = (p.astype(np.float64) * ww + c32[k]).astype(np.float32)
    res = (ww.astype(np.float64) * p.astype(np.float64))
    rel = np.max(np.abs(res / np.log1p(ww.astype(np.float64)) - 1))
    print(deg, "rel err %.3g" % rel, [float(x) for x in c32])
