"""Real spherical harmonics and real Wigner-D matrices (oracle; test infrastructure).

Sobek §2.4: edges carry r_ij = r_j - r_i and the angular features Y(r_hat_ij).
The pages fix neither the basis nor the normalisation; the reading taken is the
real basis of ``oracle.cg.real_basis_U`` (m = -l..l, l=1 ordered (y, z, x)) with
component normalisation sum_m Y_lm(r_hat)^2 = 2l+1 (Y_0 = 1).

Y is an input of the operator, so this module only serves the equivariance checks
(rotated inputs must give rotated outputs) and the pins of the input generator.

Two independent constructions of the real Wigner-D are provided so that each can
pin the other: a least-squares fit of Y(R r) = D Y(r) on sample directions, and
U conj(D_complex) U^dagger from Wigner's small-d formula with z-y-z Euler angles.
"""
from __future__ import annotations

from math import factorial

import numpy as np

from .cg import real_basis_U


def _assoc_legendre(lmax: int, z: np.ndarray) -> dict:
    """P_l^m(z) with the Condon-Shortley phase, for 0 <= m <= l <= lmax."""
    P = {}
    s = np.sqrt(np.clip(1.0 - z * z, 0.0, None))
    for m in range(lmax + 1):
        dfact = 1.0
        for k in range(1, 2 * m, 2):
            dfact *= k
        pmm = (-1) ** m * dfact * s ** m
        P[(m, m)] = pmm
        if m + 1 <= lmax:
            P[(m + 1, m)] = z * (2 * m + 1) * pmm
        for l in range(m + 2, lmax + 1):
            P[(l, m)] = ((2 * l - 1) * z * P[(l - 1, m)] - (l + m - 1) * P[(l - 2, m)]) / (l - m)
    return P


def complex_sh(l: int, vec: np.ndarray) -> np.ndarray:
    """Complex Y_l^m(r_hat), m=-l..l, component-normalised, shape [n, 2l+1]."""
    v = np.asarray(vec, dtype=np.float64)
    r = np.linalg.norm(v, axis=-1)
    x, y, z = v[..., 0] / r, v[..., 1] / r, v[..., 2] / r
    phi = np.arctan2(y, x)
    P = _assoc_legendre(l, z)
    out = np.zeros(v.shape[:-1] + (2 * l + 1,), dtype=np.complex128)
    for m in range(0, l + 1):
        norm = np.sqrt((2 * l + 1) * factorial(l - m) / factorial(l + m))
        ym = norm * P[(l, m)] * np.exp(1j * m * phi)
        out[..., l + m] = ym
        if m > 0:
            out[..., l - m] = (-1) ** m * np.conj(ym)
    return out


def real_sh(l: int, vec: np.ndarray) -> np.ndarray:
    """Real Y_l(r_hat) in the basis of real_basis_U, component-normalised."""
    yc = complex_sh(l, vec)
    yr = yc @ real_basis_U(l).T
    assert np.abs(yr.imag).max() < 1e-10
    return yr.real


def real_sh_all(lmax: int, vec: np.ndarray) -> np.ndarray:
    """Concatenated blocks l = 0..lmax, shape [n, (lmax+1)^2]."""
    return np.concatenate([real_sh(l, vec) for l in range(lmax + 1)], axis=-1)


# ----------------------------------------------------------------------------- Wigner-D

def wigner_D_lstsq(l: int, R: np.ndarray, n_samples: int = 64, seed: int = 0) -> np.ndarray:
    """Real D_l(R) with Y_l(R r) = D_l(R) Y_l(r), fitted on random directions."""
    rng = np.random.default_rng(seed)
    pts = rng.normal(size=(max(n_samples, 4 * (2 * l + 1)), 3))
    A = real_sh(l, pts)
    B = real_sh(l, pts @ R.T)
    D, *_ = np.linalg.lstsq(A, B, rcond=None)
    return D.T


def _small_d(l: int, beta: float) -> np.ndarray:
    """Wigner small-d d^l_{m'm}(beta), rows m', columns m."""
    n = 2 * l + 1
    d = np.zeros((n, n))
    c, s = np.cos(beta / 2), np.sin(beta / 2)
    for mp in range(-l, l + 1):
        for m in range(-l, l + 1):
            pre = np.sqrt(factorial(l + mp) * factorial(l - mp) * factorial(l + m) * factorial(l - m))
            tot = 0.0
            for k in range(0, 2 * l + 1):
                a1, a2, a3, a4 = l + m - k, k, l - k - mp, k - m + mp
                if min(a1, a2, a3, a4) < 0:
                    continue
                tot += ((-1) ** (k - m + mp) / (factorial(a1) * factorial(a2) * factorial(a3) * factorial(a4))
                        * c ** (2 * l - 2 * k + m - mp) * s ** (2 * k - m + mp))
            d[mp + l, m + l] = pre * tot
    return d


def euler_zyz(R: np.ndarray):
    """(alpha, beta, gamma) with R = Rz(alpha) Ry(beta) Rz(gamma) (generic R)."""
    beta = np.arccos(np.clip(R[2, 2], -1.0, 1.0))
    alpha = np.arctan2(R[1, 2], R[0, 2])
    gamma = np.arctan2(R[2, 1], -R[2, 0])
    return alpha, beta, gamma


def wigner_D_euler(l: int, R: np.ndarray) -> np.ndarray:
    """Real D_l(R) = U conj(D_complex(R)) U^dagger, D_complex from small-d."""
    a, b, g = euler_zyz(R)
    ms = np.arange(-l, l + 1)
    Dc = np.exp(-1j * ms[:, None] * a) * _small_d(l, b) * np.exp(-1j * ms[None, :] * g)
    U = real_basis_U(l)
    D = U @ np.conj(Dc) @ U.conj().T
    assert np.abs(D.imag).max() < 1e-10
    return D.real


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    """Haar-random proper rotation (QR of a Gaussian with sign fix)."""
    q, r = np.linalg.qr(rng.normal(size=(3, 3)))
    q = q * np.sign(np.diag(r))[None, :]
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q
