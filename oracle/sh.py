"""Oracle for the real spherical-harmonics direction encoding (bands l = 0..3,
16 values). Test infrastructure only.

The pages name no direction encoding for the hash-grid scene function beyond
the positional encoding; the degree-4 spherical-harmonics reading is written
here from the textbook definition:

  Y_l^0      = K_l^0 P_l^0(cos th)
  Y_l^m      = sqrt(2) K_l^m P_l^m(cos th) cos(m ph)      m > 0
  Y_l^{-m}   = sqrt(2) K_l^m P_l^m(cos th) sin(m ph)      m > 0
  K_l^m      = sqrt((2l+1)/(4 pi) * (l-m)!/(l+m)!)

with associated Legendre functions P_l^m WITHOUT the Condon-Shortley phase,
cos th = z and ph = atan2(y, x) for a unit direction (x, y, z). Output order:
index l*l + l + m for m = -l..l.
"""
from __future__ import annotations

import math

import numpy as np


def assoc_legendre(l: int, m: int, x):
    """P_l^m(x), m >= 0, no Condon-Shortley phase, by the standard recurrences:
    P_m^m = (2m-1)!! (1-x^2)^(m/2); P_{m+1}^m = x (2m+1) P_m^m;
    (l-m) P_l^m = x (2l-1) P_{l-1}^m - (l+m-1) P_{l-2}^m."""
    x = np.asarray(x, dtype=np.float64)
    pmm = np.ones_like(x)
    if m > 0:
        s = np.sqrt(np.maximum(0.0, 1.0 - x * x))
        fact = 1.0
        for _ in range(m):
            pmm = pmm * fact * s
            fact += 2.0
    if l == m:
        return pmm
    pm1 = x * (2 * m + 1) * pmm
    if l == m + 1:
        return pm1
    p_prev, p = pmm, pm1
    for ll in range(m + 2, l + 1):
        p_prev, p = p, (x * (2 * ll - 1) * p - (ll + m - 1) * p_prev) / (ll - m)
    return p


def sh_norm(l: int, m: int) -> float:
    return math.sqrt((2 * l + 1) / (4 * math.pi) * math.factorial(l - m) / math.factorial(l + m))


def real_sh(d, bands: int = 4):
    """Real SH of unit directions d [P,3] -> [P, bands^2] fp64."""
    d = np.asarray(d, dtype=np.float64)
    x, y, z = d[:, 0], d[:, 1], d[:, 2]
    ph = np.arctan2(y, x)
    out = np.zeros((d.shape[0], bands * bands))
    for l in range(bands):
        for m in range(0, l + 1):
            p = assoc_legendre(l, m, z)
            k = sh_norm(l, m)
            if m == 0:
                out[:, l * l + l] = k * p
            else:
                out[:, l * l + l + m] = math.sqrt(2.0) * k * p * np.cos(m * ph)
                out[:, l * l + l - m] = math.sqrt(2.0) * k * p * np.sin(m * ph)
    return out
