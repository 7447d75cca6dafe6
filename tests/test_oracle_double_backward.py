"""Pins of the oracle's second-order program (Sobek §3.3; LunaTP Algorithm 3).

The double backward returns the directional derivative, along v = (x_dot,
Y_dot, phi_dot, A_dot), of the forward output (m_dot = J v) and of the four
first-order adjoints (H v, H the Hessian of <m_bar, m(x, Y, phi, A)>). Pinned by:

* central finite differences of the oracle's forward and first backward, which
  are pinned themselves (test_oracle_conv);
* symmetry of the Hessian, <u, H v> = <H u, v>, which a missing, doubled or
  transposed cross term breaks;
* the exact multilinear split: the operator is linear in each of x, Y, phi and
  A, so J v is the sum of four forwards with one argument replaced by its
  direction, and each block of H v is the sum of first backwards with one other
  argument replaced;
* <m_bar, J v> = <J^T m_bar, v> against the first backward.
"""
import numpy as np
import pytest

from oracle.conv import Problem, backward, double_backward, forward
from test_oracle_conv import PROBLEMS, _graph, _inputs


def _setup(spec, seed, N=7, E=30):
    pr = Problem(*spec)
    rng = np.random.default_rng(seed)
    src, dst = _graph(rng, N, E)
    _, Y, phi, x, A = _inputs(pr, rng, N, src, dst)
    g = rng.normal(size=(N, pr.c_out))
    v = [rng.normal(size=a.shape) for a in (x, Y, phi, A)]
    return pr, rng, N, src, dst, [x, Y, phi, A], g, v


def _dot(a, b):
    return float(sum((u * w).sum() for u, w in zip(a, b)))


@pytest.mark.parametrize("spec", PROBLEMS)
def test_double_backward_finite_differences(spec):
    pr, rng, N, src, dst, args, g, v = _setup(spec, 31)
    mdot, *hv = double_backward(pr, *args, src, dst, g, *v, N, chunk=6)
    h = 1e-6
    ap = [a + h * d for a, d in zip(args, v)]
    am = [a - h * d for a, d in zip(args, v)]
    fd_m = (forward(pr, *ap, src, dst, N) - forward(pr, *am, src, dst, N)) / (2 * h)
    assert np.abs(fd_m - mdot).max() < 1e-7 * max(1.0, np.abs(mdot).max())
    bp = backward(pr, *ap, src, dst, g, N)
    bm = backward(pr, *am, src, dst, g, N)
    for k in range(4):
        fd = (bp[k] - bm[k]) / (2 * h)
        assert np.abs(fd - hv[k]).max() < 1e-7 * max(1.0, np.abs(hv[k]).max()), k


@pytest.mark.parametrize("spec", PROBLEMS)
def test_hessian_is_symmetric(spec):
    pr, rng, N, src, dst, args, g, v = _setup(spec, 37)
    u = [rng.normal(size=a.shape) for a in args]
    _, *hv = double_backward(pr, *args, src, dst, g, *v, N)
    _, *hu = double_backward(pr, *args, src, dst, g, *u, N)
    lhs, rhs = _dot(u, hv), _dot(hu, v)
    assert abs(lhs - rhs) < 1e-11 * max(1.0, abs(lhs))


@pytest.mark.parametrize("spec", PROBLEMS)
def test_multilinear_split(spec):
    pr, rng, N, src, dst, args, g, v = _setup(spec, 41)
    mdot, hx, hY, hphi, hA = double_backward(pr, *args, src, dst, g, *v, N, chunk=4)

    def sub(k):
        a = list(args)
        a[k] = v[k]
        return a
    want_m = sum(forward(pr, *sub(k), src, dst, N) for k in range(4))
    assert np.abs(want_m - mdot).max() < 1e-12 * np.abs(mdot).max()
    b = [backward(pr, *sub(k), src, dst, g, N) for k in range(4)]
    # the adjoint of an argument does not depend on that argument
    want = [b[1][0] + b[2][0] + b[3][0], b[0][1] + b[2][1] + b[3][1],
            b[0][2] + b[1][2] + b[3][2], b[0][3] + b[1][3] + b[2][3]]
    for k, got in enumerate((hx, hY, hphi, hA)):
        assert np.abs(want[k] - got).max() < 1e-12 * max(1.0, np.abs(got).max()), k


@pytest.mark.parametrize("spec", PROBLEMS[:1] + PROBLEMS[2:3])
def test_directional_output_against_first_backward(spec):
    pr, rng, N, src, dst, args, g, v = _setup(spec, 43)
    mdot, *_ = double_backward(pr, *args, src, dst, g, *v, N)
    grads = backward(pr, *args, src, dst, g, N)
    assert abs(float((g * mdot).sum()) - _dot(grads, v)) < 1e-11 * max(1.0, abs(float((g * mdot).sum())))


def test_double_backward_empty_graph():
    pr = Problem(*PROBLEMS[0])
    rng = np.random.default_rng(2)
    N = 4
    e = np.zeros(0, np.int64)
    x, A = rng.normal(size=(N, pr.c_in)), rng.normal(size=(pr.K, pr.n_w))
    z = np.zeros((0, pr.dim_y)), np.zeros((0, pr.K))
    out = double_backward(pr, x, z[0], z[1], A, e, e, rng.normal(size=(N, pr.c_out)),
                          x, z[0], z[1], A, N)
    assert all(not o.any() for o in out)
    assert out[2].shape == (0, pr.dim_y) and out[3].shape == (0, pr.K)
