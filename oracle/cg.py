"""Clebsch-Gordan coefficients in float64 (oracle side; test infrastructure only).

e3nn course, "Curriculum at a glance", lesson 03a: x (x) y decomposes by Clebsch-Gordan
coefficients into irreps l3 with |l1-l2| <= l3 <= l1+l2, and the three paths of 1 (x) 1 are the
dot, cross and symmetric traceless products.  The E3J summary (section G.2) builds the same
coefficients by a ladder construction; the oracle deliberately uses a different route:

1. complex (Condon-Shortley) coefficients <l1 m1 l2 m2 | l3 m3> from the Racah closed form,
   evaluated in exact integer/rational arithmetic and rounded once;
2. the change to the real basis of ``oracle.sh`` (Y_real = U Y_complex):
       C_R[m1,m2,m3] = sum_{a,b,c} conj(U1[m1,a]) conj(U2[m2,b]) U3[m3,c] <l1 a l2 b | l3 c>
   which is either purely real or purely imaginary; the nonzero part is kept;
3. the normalisation and sign fixed for this build (the sources leave both open):
   * each path tensor has Frobenius norm 1 over (m1, m2, m3);
   * if l1+l2+l3 is even, C_R[0,0,0] (all m = 0) is positive; if odd, the first nonzero entry in
     lexicographic (m1, m2, m3) order, each m ascending from -l, is positive.
   These give +dot/sqrt(3), +cross/sqrt(6) and a positive symmetric-traceless path for 1 (x) 1.
"""

from fractions import Fraction
from functools import lru_cache
from math import factorial, sqrt

import numpy as np


def complex_cg(j1, m1, j2, m2, J, M):
    """<j1 m1 j2 m2 | J M> by the Racah formula (integer spins), Condon-Shortley phase."""
    if M != m1 + m2:
        return 0.0
    if not (abs(j1 - j2) <= J <= j1 + j2):
        return 0.0
    if abs(m1) > j1 or abs(m2) > j2 or abs(M) > J:
        return 0.0
    f = factorial
    pre = Fraction((2 * J + 1) * f(J + j1 - j2) * f(J - j1 + j2) * f(j1 + j2 - J), f(j1 + j2 + J + 1))
    pre *= f(J + M) * f(J - M) * f(j1 - m1) * f(j1 + m1) * f(j2 - m2) * f(j2 + m2)
    s = Fraction(0)
    kmin = max(0, j2 - J - m1, j1 - J + m2)
    kmax = min(j1 + j2 - J, j1 - m1, j2 + m2)
    for k in range(kmin, kmax + 1):
        den = f(k) * f(j1 + j2 - J - k) * f(j1 - m1 - k) * f(j2 + m2 - k) * f(J - j2 + m1 + k) * f(J - j1 - m2 + k)
        s += Fraction((-1) ** k, den)
    if s == 0:
        return 0.0
    # s * sqrt(pre): square exactly, take one rounded square root, restore the sign.
    val = sqrt(float(s * s * pre))
    return val if s > 0 else -val


def real_basis_change(l):
    """U with Y_real = U @ Y_complex (rows: real m = -l..l, columns: complex m = -l..l)."""
    U = np.zeros((2 * l + 1, 2 * l + 1), dtype=np.complex128)
    r2 = 1.0 / sqrt(2.0)
    for m in range(-l, l + 1):
        i = m + l
        if m > 0:
            U[i, -m + l] = r2
            U[i, m + l] = (-1) ** m * r2
        elif m == 0:
            U[i, l] = 1.0
        else:
            k = -m
            U[i, -k + l] = 1j * r2
            U[i, k + l] = -1j * (-1) ** k * r2
    return U


@lru_cache(maxsize=None)
def _real_cg_cached(l1, l2, l3):
    cc = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    for a in range(-l1, l1 + 1):
        for b in range(-l2, l2 + 1):
            c = a + b
            if abs(c) <= l3:
                cc[a + l1, b + l2, c + l3] = complex_cg(l1, a, l2, b, l3, c)
    U1, U2, U3 = real_basis_change(l1), real_basis_change(l2), real_basis_change(l3)
    cr = np.einsum("ia,jb,kc,abc->ijk", U1.conj(), U2.conj(), U3, cc)
    re, im = np.abs(cr.real).max(), np.abs(cr.imag).max()
    t = cr.real if re >= im else cr.imag
    t = t / np.sqrt(np.sum(t * t))
    if (l1 + l2 + l3) % 2 == 0:
        ref = t[l1, l2, l3]
    else:
        ref = t.reshape(-1)[np.flatnonzero(np.abs(t.reshape(-1)) > 1e-12)[0]]
    if ref < 0:
        t = -t
    # the discarded part must vanish: the change of basis is exact up to rounding
    assert min(re, im) < 1e-12 * max(re, im), (l1, l2, l3)
    t[np.abs(t) < 1e-15] = 0.0
    t.setflags(write=False)
    return t


def real_cg(l1, l2, l3):
    """Real-basis CG tensor [2l1+1, 2l2+1, 2l3+1]; Frobenius norm 1, sign rule above."""
    if not (abs(l1 - l2) <= l3 <= l1 + l2):
        raise ValueError(f"triangle rule violated for ({l1}, {l2}, {l3})")
    return _real_cg_cached(l1, l2, l3)
