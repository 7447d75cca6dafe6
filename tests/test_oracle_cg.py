"""Pins of the oracle's Clebsch-Gordan tables against things other than itself.

* complex CG: sympy's independent implementation (exact);
* real CG: orthonormality and completeness of the coupling;
* closed forms for small degrees (delta couplings, the dot and cross products in
  (y, z, x) order, the symmetric traceless l=2 product);
* equivariance of every real coupling under random rotations with real
  Wigner-D matrices fitted from spherical harmonics (pins the real basis
  against the SH convention; LunaTP §2.1 requires every path to keep the
  product equivariant).
"""
import itertools

import numpy as np
from oracle import cg, sh

LMAX = 4


def _triples(lmax):
    for l1 in range(lmax + 1):
        for l2 in range(lmax + 1):
            for l3 in range(abs(l1 - l2), min(l1 + l2, lmax) + 1):
                yield l1, l2, l3


def test_complex_cg_matches_sympy():
    from sympy.physics.quantum.cg import CG
    for l1, l2, l3 in _triples(3):
        C = cg.complex_cg(l1, l2, l3)
        for m1 in range(-l1, l1 + 1):
            for m2 in range(-l2, l2 + 1):
                m3 = m1 + m2
                if abs(m3) > l3:
                    continue
                ref = float(CG(l1, m1, l2, m2, l3, m3).doit())
                assert abs(C[m1 + l1, m2 + l2, m3 + l3] - ref) < 1e-15, (l1, m1, l2, m2, l3)


def test_real_cg_orthonormal_and_complete():
    for l1 in range(LMAX + 1):
        for l2 in range(LMAX + 1):
            n = (2 * l1 + 1) * (2 * l2 + 1)
            blocks = []
            for l3 in range(abs(l1 - l2), l1 + l2 + 1):
                R = cg.real_cg(l1, l2, l3)
                G = np.einsum("abc,abd->cd", R, R)
                assert np.abs(G - np.eye(2 * l3 + 1)).max() < 1e-14
                blocks.append(R.reshape(n, -1))
            Q = np.concatenate(blocks, axis=1)          # square, orthogonal
            assert Q.shape == (n, n)
            assert np.abs(Q @ Q.T - np.eye(n)).max() < 1e-14


def test_real_cg_closed_forms():
    for l in range(LMAX + 1):
        I = np.eye(2 * l + 1)
        assert np.abs(cg.real_cg(0, l, l)[0] - I).max() < 1e-15
        assert np.abs(cg.real_cg(l, 0, l)[:, 0, :] - I).max() < 1e-15
    # 1 x 1 -> 0: the dot product / sqrt(3)
    assert np.abs(cg.real_cg(1, 1, 0)[:, :, 0] - np.eye(3) / np.sqrt(3)).max() < 1e-15
    # 1 x 1 -> 1: the cross product / sqrt(2); (y, z, x) is a cyclic relabelling of
    # (x, y, z), so the Levi-Civita symbol keeps its form
    eps = np.zeros((3, 3, 3))
    for a, b, c in itertools.permutations(range(3)):
        eps[a, b, c] = np.linalg.det(np.eye(3)[[a, b, c]])
    R = cg.real_cg(1, 1, 1)
    assert np.abs(R - eps / np.sqrt(2)).max() < 1e-15 or np.abs(R + eps / np.sqrt(2)).max() < 1e-15
    # 1 x 1 -> 2: symmetric and traceless in (m1, m2)
    R2 = cg.real_cg(1, 1, 2)
    for c in range(5):
        assert np.abs(R2[:, :, c] - R2[:, :, c].T).max() < 1e-15
        assert abs(np.trace(R2[:, :, c])) < 1e-15
    # m=0 component of 1x1->2 is +-(2 zz - xx - yy)/sqrt(6) in (y, z, x) order; the
    # first non-zero entry (m1, m2, m3) = (y, y, 0) is positive by convention
    assert np.abs(R2[:, :, 2] - np.diag([1.0, -2.0, 1.0]) / np.sqrt(6)).max() < 1e-15
    # m=2 component is (xx - yy)/sqrt(2), same global sign
    assert np.abs(R2[:, :, 4] - np.diag([-1.0, 0.0, 1.0]) / np.sqrt(2) * -1).max() < 1e-15


def test_real_cg_sign_convention():
    for t in _triples(LMAX):
        flat = cg.real_cg(*t).reshape(-1)
        assert flat[np.nonzero(flat)[0][0]] > 0
        assert not np.any(np.signbit(flat) & (flat == 0))


def test_real_cg_equivariant():
    """R(D1 x, D2 y) = D3 R(x, y) for proper rotations; parity is checked on the
    whole operator, where the path rule p3 = p1 p2 decides it."""
    rng = np.random.default_rng(7)
    for _ in range(3):
        Rm = sh.random_rotation(rng)
        D = {l: sh.wigner_D_lstsq(l, Rm) for l in range(LMAX + 1)}
        for l1, l2, l3 in _triples(LMAX):
            T = cg.real_cg(l1, l2, l3)
            x = rng.normal(size=2 * l1 + 1)
            y = rng.normal(size=2 * l2 + 1)
            lhs = np.einsum("abc,a,b->c", T, D[l1] @ x, D[l2] @ y)
            rhs = D[l3] @ np.einsum("abc,a,b->c", T, x, y)
            assert np.abs(lhs - rhs).max() < 1e-12, (l1, l2, l3)
