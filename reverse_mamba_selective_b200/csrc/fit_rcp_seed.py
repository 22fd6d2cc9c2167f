# Fits the integer seed of the FMA-pipe reciprocal used by the scan kernel's SiLU
# (scan_kernels.cuh, rcp_fma): r0 = bits^-1(M - bits(d)) treats the float bit pattern as a
# piecewise-linear log2, so M - bits(d) approximates the pattern of 1/d.  M is chosen to minimise
# the maximum relative error of r0 over one binade (the error is the same in every binade), and
# the relative error left after 1, 2, 3 Newton steps r <- r + r (1 - d r) is printed.
import numpy as np

d = np.linspace(1.0, 2.0, 200001, dtype=np.float32)
bits = d.view(np.uint32).astype(np.int64)
best = None
for M in range(0x7EE00000, 0x7F000000, 0x400):
    r0 = (M - bits).astype(np.uint32).view(np.float32).astype(np.float64)
    err = np.max(np.abs(r0 * d - 1))
    if best is None or err < best[1]:
        best = (M, err)
M = best[0]
for M2 in range(M - 0x400, M + 0x400):
    r0 = (M2 - bits).astype(np.uint32).view(np.float32).astype(np.float64)
    err = np.max(np.abs(r0 * d - 1))
    if err < best[1]:
        best = (M2, err)
M, e0 = best
r = (M - bits).astype(np.uint32).view(np.float32).astype(np.float64)
errs = []
for _ in range(3):
    r = r + r * (1 - d * r)
    errs.append(np.max(np.abs(r * d - 1)))
print(f"seed 0x{M:08X}: seed error {e0:.3e}; after Newton steps: " + ", ".join(f"{x:.3e}" for x in errs))
