"""Clebsch-Gordan coefficients, complex and real basis (oracle; test infrastructure).

LunaTP §2.1 Eq. 1 writes the degree-l output of the CG tensor product as
    [x^(l1) (x) y^(l2)]^(l)_m = sum_{m1,m2} C^{(l,m)}_{(l1,m1)(l2,m2)} x_{m1} y_{m2},
nonzero only when |l1-l2| <= l <= l1+l2. Sobek §4.2 Eq. 32 uses the same sparse
coefficient c^pi_{mi,my,mo} (with the path normalisation folded in) in the real
spherical-harmonic basis that the features live in.

Readings taken here (the pages name no convention):
* complex CG: Racah's closed formula with Condon-Shortley phases, evaluated in
  exact rational arithmetic (the coefficient is +-sqrt(rational));
* real basis: the standard complex->real change of basis U (m<0 <-> sine-type,
  m=0, m>0 <-> cosine-type; l=1 orders as (y, z, x)), giving
  R[a,b,c] = sum_{i,j,k} conj(U1[a,i]) conj(U2[b,j]) U3[c,k] C[i,j,k];
  R is purely real or purely imaginary; the non-zero part is kept;
* orthonormal coupling sum_{a,b} R[a,b,c] R[a,b,c'] = delta_{cc'};
* overall sign: the first non-zero entry in lexicographic (m1, m2, m3) order is
  positive;
* path normalisation factor 1 (A is learned and absorbs any scale).
"""
from __future__ import annotations

import decimal
from fractions import Fraction
from functools import lru_cache
from math import factorial

import numpy as np

_NONZERO = 1e-12


def _f(n: int) -> int:
    return factorial(n)


@lru_cache(maxsize=None)
def complex_cg_exact(j1: int, m1: int, j2: int, m2: int, J: int, M: int):
    """<j1 m1; j2 m2 | J M> as (sign, square) with square an exact Fraction.

    Racah's formula:
      delta(M, m1+m2) * sqrt((2J+1)(J+j1-j2)!(J-j1+j2)!(j1+j2-J)!/(j1+j2+J+1)!)
      * sqrt((J+M)!(J-M)!(j1-m1)!(j1+m1)!(j2-m2)!(j2+m2)!)
      * sum_k (-1)^k / (k!(j1+j2-J-k)!(j1-m1-k)!(j2+m2-k)!(J-j2+m1+k)!(J-j1-m2+k)!)
    """
    if M != m1 + m2:
        return 0, Fraction(0)
    if not (abs(j1 - j2) <= J <= j1 + j2):
        return 0, Fraction(0)
    if abs(m1) > j1 or abs(m2) > j2 or abs(M) > J:
        return 0, Fraction(0)
    pre = Fraction((2 * J + 1) * _f(J + j1 - j2) * _f(J - j1 + j2) * _f(j1 + j2 - J),
                   _f(j1 + j2 + J + 1))
    pre *= (_f(J + M) * _f(J - M) * _f(j1 - m1) * _f(j1 + m1) * _f(j2 - m2) * _f(j2 + m2))
    s = Fraction(0)
    for k in range(0, j1 + j2 - J + 1):
        a = [k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k]
        if min(a) < 0:
            continue
        d = 1
        for v in a:
            d *= _f(v)
        s += Fraction((-1) ** k, d)
    if s == 0:
        return 0, Fraction(0)
    return (1 if s > 0 else -1), pre * s * s


def _sqrt_fraction(q: Fraction) -> float:
    """Correctly rounded float of sqrt(q) for a non-negative Fraction."""
    if q == 0:
        return 0.0
    with decimal.localcontext() as ctx:
        ctx.prec = 50
        return float((decimal.Decimal(q.numerator) / decimal.Decimal(q.denominator)).sqrt())


def complex_cg_value(j1, m1, j2, m2, J, M) -> float:
    sgn, sq = complex_cg_exact(j1, m1, j2, m2, J, M)
    return sgn * _sqrt_fraction(sq)


@lru_cache(maxsize=None)
def complex_cg(l1: int, l2: int, l3: int) -> np.ndarray:
    """C[i, j, k] = <l1 (i-l1); l2 (j-l2) | l3 (k-l3)>, fp64."""
    C = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    for i in range(2 * l1 + 1):
        for j in range(2 * l2 + 1):
            k = (i - l1) + (j - l2) + l3
            if 0 <= k <= 2 * l3:
                C[i, j, k] = complex_cg_value(l1, i - l1, l2, j - l2, l3, k - l3)
    return C


@lru_cache(maxsize=None)
def real_basis_U(l: int) -> np.ndarray:
    """Rows: real index (m=-l..l); columns: complex index (m'=-l..l).

    Y_real[m] = sum_{m'} U[m, m'] Y_complex[m'] with
      m > 0: (Y^{-m} + (-1)^m Y^{m}) / sqrt2
      m = 0: Y^0
      m < 0: i (Y^{m} - (-1)^m Y^{-m}) / sqrt2
    """
    n = 2 * l + 1
    U = np.zeros((n, n), dtype=np.complex128)
    r = 1.0 / np.sqrt(2.0)
    for m in range(-l, l + 1):
        row = m + l
        if m > 0:
            U[row, -m + l] = r
            U[row, m + l] = (-1) ** m * r
        elif m == 0:
            U[row, l] = 1.0
        else:
            U[row, m + l] = 1j * r
            U[row, -m + l] = -1j * (-1) ** m * r
    return U


@lru_cache(maxsize=None)
def real_cg(l1: int, l2: int, l3: int) -> np.ndarray:
    """Real-basis coupling tensor R[m1, m2, m3] (indices 0..2l), see module doc."""
    if not (abs(l1 - l2) <= l3 <= l1 + l2):
        raise ValueError(f"triangle rule violated for ({l1},{l2},{l3})")
    C = complex_cg(l1, l2, l3)
    U1, U2, U3 = real_basis_U(l1), real_basis_U(l2), real_basis_U(l3)
    R = np.einsum("ai,bj,ck,ijk->abc", U1.conj(), U2.conj(), U3, C)
    re, im = np.abs(R.real).max(), np.abs(R.imag).max()
    if im > re:
        assert re < _NONZERO, (l1, l2, l3, re, im)
        T = R.imag.copy()
    else:
        assert im < _NONZERO, (l1, l2, l3, re, im)
        T = R.real.copy()
    T[np.abs(T) < _NONZERO] = 0.0
    flat = T.reshape(-1)
    first = flat[np.nonzero(flat)[0][0]]
    if first < 0:
        T = -T
    T = T + 0.0                      # no negative zeros
    T.setflags(write=False)
    return T


def real_cg_sparse(l1: int, l2: int, l3: int):
    """Non-zero entries of real_cg as a list of (m1, m2, m3, c), lexicographic."""
    T = real_cg(l1, l2, l3)
    idx = np.argwhere(T != 0.0)
    return [(int(a), int(b), int(c), float(T[a, b, c])) for a, b, c in idx]
