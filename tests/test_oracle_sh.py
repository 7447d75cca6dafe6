"""Pins of the oracle's spherical harmonics and Wigner-D, and of the input
generator's SH against the oracle's (two independent constructions)."""
import numpy as np

from inputs.workloads import spherical_harmonics
from oracle import sh


def test_real_sh_closed_forms():
    rng = np.random.default_rng(0)
    v = rng.normal(size=(50, 3))
    u = v / np.linalg.norm(v, axis=1, keepdims=True)
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    assert np.abs(sh.real_sh(0, v) - 1.0).max() < 1e-14
    assert np.abs(sh.real_sh(1, v) - np.sqrt(3) * np.stack([y, z, x], 1)).max() < 1e-14
    Y2 = np.stack([np.sqrt(15) * x * y, np.sqrt(15) * y * z, np.sqrt(5) / 2 * (3 * z * z - 1),
                   np.sqrt(15) * x * z, np.sqrt(15) / 2 * (x * x - y * y)], 1)
    assert np.abs(sh.real_sh(2, v) - Y2).max() < 1e-13


def test_component_normalisation():
    v = np.random.default_rng(1).normal(size=(40, 3))
    for l in range(7):
        Y = sh.real_sh(l, v)
        assert np.abs((Y * Y).sum(1) - (2 * l + 1)).max() < 1e-11


def test_wigner_D_two_constructions_agree_and_compose():
    rng = np.random.default_rng(2)
    R1, R2 = sh.random_rotation(rng), sh.random_rotation(rng)
    for l in range(6):
        Da = sh.wigner_D_lstsq(l, R1)
        Db = sh.wigner_D_euler(l, R1)
        assert np.abs(Da - Db).max() < 1e-11
        assert np.abs(Da @ Da.T - np.eye(2 * l + 1)).max() < 1e-11
        D12 = sh.wigner_D_euler(l, R1 @ R2)
        assert np.abs(D12 - sh.wigner_D_euler(l, R1) @ sh.wigner_D_euler(l, R2)).max() < 1e-11


def test_input_generator_sh_matches_oracle():
    v = np.random.default_rng(3).normal(size=(200, 3))
    for L in range(5):
        assert np.abs(spherical_harmonics(L, v) - sh.real_sh_all(L, v)).max() < 1e-12
