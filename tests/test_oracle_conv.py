"""Pins of the oracle's convolution and first backward.

* Sobek §3.1: the materialised and the streamed orders are "identical in exact
  arithmetic"; §4.2: Eqs. 33-35 are "an exact reassociation of Eq. 16". Checked by
  brute force on tiny graphs, uvu and uvw.
* Equivariance: rotated (and inverted) inputs give rotated (inverted) outputs,
  with Y recomputed from the rotated edge vectors (Sobek §2.1).
* Scalar special case: x = C x 0e, L_sh = 0, out C x 0e reduces to one sparse
  matrix product per channel, checked against scipy.sparse.
* Backward (Sobek §3.2, LunaTP Algorithm 2): the operator is linear in each of
  x, Y, phi and A separately, so <m_bar, m(v)> = <grad, v> for a direction v in
  one argument; plus central finite differences.
* CSR (LunaTP §4.1): brute-force per-receiver scan on small random graphs.
"""
import numpy as np
import pytest
import scipy.sparse as sp

from oracle import csr, sh
from oracle.conv import (Problem, backward, forward, forward_receiver_factorised,
                         forward_streamed)
from oracle import irreps as ir


def _graph(rng, N, E):
    src = rng.integers(0, N, E)
    dst = rng.integers(0, N, E)
    keep = src != dst
    return src[keep], dst[keep]


def _inputs(pr, rng, N, src, dst):
    vec = rng.normal(size=(len(src), 3))
    Y = sh.real_sh_all(pr.sh_lmax, vec)
    phi = rng.normal(size=(len(src), pr.K))
    x = rng.normal(size=(N, pr.c_in))
    A = rng.normal(size=(pr.K, pr.n_w))
    return vec, Y, phi, x, A


PROBLEMS = [
    ("3x0e+3x1o+3x2e", 2, "3x0e+3x1o+3x1e+3x2e+3x2o", 3, "uvu"),
    ("2x0e+2x1o+2x2e+2x3o", 3, "2x0e+2x1o+2x1e+2x2e+2x2o+2x3o+2x3e", 2, "uvu"),
    ("2x0e+3x1o", 2, "3x0e+2x1o+2x2e", 3, "uvw"),
    ("2x0e+1x1o+2x2e", 2, "2x0e+1x1o+2x1e+1x2e", 2, "uvw"),
]


@pytest.mark.parametrize("spec", PROBLEMS)
def test_schedules_agree(spec):
    pr = Problem(*spec)
    rng = np.random.default_rng(11)
    N = 7
    src, dst = _graph(rng, N, 30)
    _, Y, phi, x, A = _inputs(pr, rng, N, src, dst)
    naive = forward(pr, x, Y, phi, A, src, dst, N, chunk=5)
    rowptr, senders, perm = csr.build(N, src, dst)
    st = forward_streamed(pr, x, Y, phi, A, rowptr, senders, perm)
    rf = forward_receiver_factorised(pr, x, Y, phi, A, rowptr, senders, perm)
    scale = np.abs(naive).max()
    assert np.abs(naive - st).max() < 1e-13 * scale
    assert np.abs(naive - rf).max() < 1e-13 * scale


def _rotate_features(pr_blocks, Dmap, v, improper):
    out = v.copy()
    for b in pr_blocks:
        seg = ir.block_view(v, b)                         # [n, 2l+1, mul]
        rot = np.einsum("ab,nbu->nau", Dmap[b.l], seg)
        if improper:
            rot = rot * b.p
        ir.block_view(out, b)[...] = rot
    return out


@pytest.mark.parametrize("spec", PROBLEMS)
@pytest.mark.parametrize("improper", [False, True])
def test_operator_equivariant(spec, improper):
    pr = Problem(*spec)
    rng = np.random.default_rng(5)
    N = 9
    src, dst = _graph(rng, N, 40)
    vec, Y, phi, x, A = _inputs(pr, rng, N, src, dst)
    R = sh.random_rotation(rng)
    Rfull = -R if improper else R
    lmax = max(max(b.l for b in pr.bin), max(b.l for b in pr.bout))
    D = {l: sh.wigner_D_euler(l, R) for l in range(lmax + 1)}
    out = forward(pr, x, Y, phi, A, src, dst, N)
    Yr = sh.real_sh_all(pr.sh_lmax, vec @ Rfull.T)       # Y of rotated edge vectors
    xr = _rotate_features(pr.bin, D, x, improper)
    out_r = forward(pr, xr, Yr, phi, A, src, dst, N)
    want = _rotate_features(pr.bout, D, out, improper)
    assert np.abs(out_r - want).max() < 1e-12 * max(1.0, np.abs(out).max())


def test_scalar_case_is_spmm():
    C, K, N = 5, 4, 12
    pr = Problem(f"{C}x0e", 0, f"{C}x0e", K, "uvu")
    rng = np.random.default_rng(3)
    src, dst = _graph(rng, N, 60)
    vec, Y, phi, x, A = _inputs(pr, rng, N, src, dst)
    out = forward(pr, x, Y, phi, A, src, dst, N)
    for u in range(C):
        w = (phi @ A[:, u]) * Y[:, 0]
        M = sp.coo_matrix((w, (dst, src)), shape=(N, N)).tocsr()
        assert np.abs(out[:, u] - M @ x[:, u]).max() < 1e-13 * np.abs(out).max()


@pytest.mark.parametrize("spec", PROBLEMS)
def test_backward_adjoint_identities(spec):
    pr = Problem(*spec)
    rng = np.random.default_rng(17)
    N = 8
    src, dst = _graph(rng, N, 35)
    _, Y, phi, x, A = _inputs(pr, rng, N, src, dst)
    g = rng.normal(size=(N, pr.c_out))
    gx, gY, gphi, gA = backward(pr, x, Y, phi, A, src, dst, g, N, chunk=7)
    vx, vY, vp, vA = (rng.normal(size=a.shape) for a in (x, Y, phi, A))

    def dot(a, b):
        return float((a * b).sum())
    # linear in each argument: J_arg[v] is the forward evaluated at v
    assert abs(dot(g, forward(pr, vx, Y, phi, A, src, dst, N)) - dot(gx, vx)) < 1e-11
    assert abs(dot(g, forward(pr, x, vY, phi, A, src, dst, N)) - dot(gY, vY)) < 1e-11
    assert abs(dot(g, forward(pr, x, Y, vp, A, src, dst, N)) - dot(gphi, vp)) < 1e-11
    assert abs(dot(g, forward(pr, x, Y, phi, vA, src, dst, N)) - dot(gA, vA)) < 1e-11


def test_backward_finite_differences():
    pr = Problem(*PROBLEMS[1])
    rng = np.random.default_rng(23)
    N = 6
    src, dst = _graph(rng, N, 25)
    _, Y, phi, x, A = _inputs(pr, rng, N, src, dst)
    g = rng.normal(size=(N, pr.c_out))
    grads = backward(pr, x, Y, phi, A, src, dst, g, N)
    args = [x, Y, phi, A]
    h = 1e-6
    for k in range(4):
        v = rng.normal(size=args[k].shape)
        ap, am = list(args), list(args)
        ap[k] = args[k] + h * v
        am[k] = args[k] - h * v
        fd = ((forward(pr, *ap, src, dst, N) - forward(pr, *am, src, dst, N)) * g).sum() / (2 * h)
        an = (grads[k] * v).sum()
        assert abs(fd - an) < 1e-7 * max(1.0, abs(an))


def test_edge_cases():
    pr = Problem(*PROBLEMS[0])
    rng = np.random.default_rng(1)
    N = 5
    empty = np.zeros(0, np.int64)
    x = rng.normal(size=(N, pr.c_in))
    A = rng.normal(size=(pr.K, pr.n_w))
    out = forward(pr, x, np.zeros((0, pr.dim_y)), np.zeros((0, pr.K)), A, empty, empty, N)
    assert out.shape == (N, pr.c_out) and not out.any()
    # receivers without incoming edges get zeros
    src, dst = np.array([0, 1, 1]), np.array([2, 2, 3])
    _, Y, phi, _, _ = _inputs(pr, rng, N, src, dst)
    out = forward(pr, x, Y, phi, A, src, dst, N)
    assert not out[[0, 1, 4]].any() and out[2].any() and out[3].any()


def test_csr_brute_force():
    rng = np.random.default_rng(9)
    for N, E in [(1, 0), (5, 17), (13, 80), (40, 41)]:
        src = rng.integers(0, N, E)
        dst = rng.integers(0, N, E)
        rowptr, senders, perm = csr.build(N, src, dst)
        k = 0
        for i in range(N):
            assert rowptr[i] == k
            for e in range(E):                           # input order within receiver
                if dst[e] == i:
                    assert perm[k] == e and senders[k] == src[e]
                    k += 1
        assert rowptr[N] == E
        colptr, srcedge, srcrecv = csr.transpose(N, rowptr, senders)
        k = 0
        for j in range(N):
            assert colptr[j] == k
            for pos in range(E):                         # CSR order within source
                if senders[pos] == j:
                    assert srcedge[k] == pos and dst[perm[pos]] == srcrecv[k]
                    k += 1
