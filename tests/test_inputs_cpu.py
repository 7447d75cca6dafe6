"""The seeded synthetic workloads (inputs/workloads.py) are reproducible and
have the sizes the measurements quote: node and edge counts, mean degree, no
self edges, and component-normalised spherical harmonics."""
import numpy as np
import pytest

from inputs import CONFIGS, make_workload

# (workload, nodes, realised edges) as quoted with the measurements
SIZES = [(1, 64, 1120), (2, 4096, 131308), (3, 64, 1120), (5, 16384, 523786)]


@pytest.mark.parametrize("cid,n,e", SIZES)
def test_workload_sizes(cid, n, e):
    wl = make_workload(cid, 8)
    assert wl.n_nodes == n and len(wl.src) == e and len(wl.dst) == e
    assert not np.any(wl.src == wl.dst)
    assert wl.src.min() >= 0 and wl.src.max() < n and wl.dst.min() >= 0 and wl.dst.max() < n


def test_workload_is_seeded():
    a, b = make_workload(2, 8), make_workload(2, 8)
    assert np.array_equal(a.src, b.src) and np.array_equal(a.dst, b.dst)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.Y, b.Y) and np.array_equal(a.phi, b.phi)


def test_sh_component_normalised():
    wl = make_workload(1, 8)
    c = CONFIGS[1]
    for l in range(c.sh_lmax + 1):
        blk = wl.Y[:, l * l:(l + 1) * (l + 1)].astype(np.float64)
        assert np.allclose((blk ** 2).sum(axis=1), 2 * l + 1, rtol=1e-5)
