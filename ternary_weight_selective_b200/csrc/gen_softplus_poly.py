"""Coefficients of the softplus polynomial used by the selective-scan kernel.

softplus(z) = max(z, 0) + log1p(t), t = exp(-|z|) in (0, 1].  log1p(t) is
evaluated as t * p(t), with p a degree-8 least-squares fit (on Chebyshev
nodes) of log1p(t) / t over [0, 1]; t * p(t) has relative error ~3e-8 over
(0, 1] in exact arithmetic.  Run to print the coefficients (low order
first) pasted into kernel_scan.cuh.
"""
import numpy as np

t = np.cos(np.pi * (np.arange(4000) + 0.5) / 4000) * 0.5 + 0.5
f = np.log1p(t) / t
c = np.polynomial.chebyshev.Chebyshev.fit(t, f, 8, domain=[0, 1])
p = c.convert(kind=np.polynomial.Polynomial, domain=[0, 1], window=[0, 1])
tt = np.linspace(0, 1, 200001)[1:]
err = np.abs(tt * p(tt) - np.log1p(tt)) / np.log1p(tt)
print("max rel err", err.max())
print(", ".join(f"{v:.9e}f" for v in p.coef))
