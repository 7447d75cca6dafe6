"""Hand-indexed pins of the oracle's feature layout and of its work model.

Layout (Sobek §4.5, "ir_mul"): inside an irrep block of multiplicity C and
degree l, the scalar of component m (0..2l) and channel u sits at
block_offset + m * C + u (channels contiguous). The tests below place single
non-zero scalars at hand-computed indices and check where the result lands.
Each case is chosen so that a transposed reading ([u][m], offset + u(2l+1) + m)
moves either the output index or the weight column that scales it, so a
transposed or shifted block view fails here even though every other oracle test
reads inputs and outputs through the same view on both sides.

Work model (Sobek §3.1 streamed uvu order; §4.2 Eqs. 32-35 for uvw): counted by
hand for one-path contracts whose CG block is known in closed form:
1o x 1o -> 1e is the cross product in (y, z, x) order, 6 non-zero entries.
"""
import math

import numpy as np
import pytest

from oracle import cg, paths
from oracle.conv import Problem, backward, forward


def _one_edge(pr, Y0, phi0, x, A, n_nodes=2):
    src, dst = np.array([0]), np.array([1])
    return forward(pr, x, Y0[None, :], phi0[None, :], A, src, dst, n_nodes)


def test_ir_mul_index_through_identity_coupling():
    # "2x0e+2x1o": block 0 = 0e (offset 0, 2 scalars), block 1 = 1o (offset 2,
    # [3][2]). With L_sh = 0 the path 1o x 0e -> 1o has CG delta(m1, m3), so the
    # scalar at (m, u) of the sender reaches (m, u) of the receiver scaled by the
    # path weight of channel u.
    pr = Problem("2x0e+2x1o", 0, "2x0e+2x1o", 1, "uvu")
    assert [(p.l1, p.l2, p.l3, p.w_off) for p in pr.paths] == [(0, 0, 0, 0), (1, 0, 1, 2)]
    A = np.array([[7.0, 11.0, 3.0, 5.0]])          # path 1: channel 0 -> 3.0, channel 1 -> 5.0
    x = np.zeros((2, 8))
    x[0, 2 + 2 * 2 + 0] = 1.0                       # component m = 2 (x), channel u = 0: index 6
    out = _one_edge(pr, np.array([1.0]), np.array([1.0]), x, A)
    want = np.zeros((2, 8))
    want[1, 6] = 3.0                                # same (m, u), weight of channel 0
    assert np.allclose(out, want, rtol=0, atol=1e-14)
    # channel 1 of component m = 0: index 2 + 0 * 2 + 1 = 3, weight 5.0
    x[:] = 0.0
    x[0, 3] = 1.0
    out = _one_edge(pr, np.array([1.0]), np.array([1.0]), x, A)
    want[:] = 0.0
    want[1, 3] = 5.0
    assert np.allclose(out, want, rtol=0, atol=1e-14)


def test_ir_mul_index_through_dot_product_coupling():
    # 1o x 1o -> 0e is delta(m1, m2) / sqrt(3) (first non-zero positive). With Y_1
    # the unit vector of component m and x non-zero only at (m, u) of the 1o
    # block, only output channel u of the 0e block receives w_u / sqrt(3).
    pr = Problem("3x1o", 1, "3x0e", 1, "uvu")
    assert [(p.l1, p.l2, p.l3) for p in pr.paths] == [(1, 1, 0)]
    A = np.array([[2.0, 3.0, 4.0]])
    for m in range(3):
        for u in range(3):
            x = np.zeros((2, 9))
            x[0, m * 3 + u] = 1.0
            Y0 = np.zeros(4)
            Y0[0] = 1.0
            Y0[1 + m] = 1.0
            out = _one_edge(pr, Y0, np.array([1.0]), x, A)
            want = np.zeros((2, 3))
            want[1, u] = A[0, u] / math.sqrt(3.0)
            assert np.allclose(out, want, rtol=0, atol=1e-15), (m, u)
            # Y_1 along another component: no coupling
            Y0[1 + m] = 0.0
            Y0[1 + (m + 1) % 3] = 1.0
            assert not _one_edge(pr, Y0, np.array([1.0]), x, A).any()


def test_ir_mul_index_of_backward_source_gradient():
    # grad_x of the identity coupling: a single non-zero grad_out at receiver
    # (m, u) of the 1o block comes back at the sender's (m, u) times w_u.
    pr = Problem("2x0e+2x1o", 0, "2x0e+2x1o", 1, "uvu")
    A = np.array([[7.0, 11.0, 3.0, 5.0]])
    g = np.zeros((2, 8))
    g[1, 2 + 1 * 2 + 1] = 1.0                       # m = 1, u = 1: index 5
    x = np.zeros((2, 8))
    gx, gY, gphi, gA = backward(pr, x, np.array([[1.0]]), np.array([[1.0]]), A, np.array([0]),
                                np.array([1]), g, 2)
    want = np.zeros((2, 8))
    want[0, 5] = 5.0
    assert np.allclose(gx, want, rtol=0, atol=1e-14)


def test_cross_product_block_has_six_entries():
    R = cg.real_cg(1, 1, 1)
    assert len(cg.real_cg_sparse(1, 1, 1)) == 6
    # the six entries of the Levi-Civita symbol in (y, z, x) order, all +-1/sqrt(2)
    assert np.allclose(np.abs(R[R != 0]), 1.0 / math.sqrt(2.0))


@pytest.mark.parametrize("K,N,E", [(4, 5, 10), (8, 3, 7)])
def test_work_model_uvu_hand_count(K, N, E):
    # one path 1o x 1o -> 1e (C = 1). Streamed forward per edge and channel:
    # K FMAs for w = phi . A, 6 for the CG contraction (one per non-zero), 3 for
    # acc[m3] += w T[m3]. Backward per edge and channel: h = <m_bar, T> (6 + 3),
    # phi_bar and A_bar (K each), w recomputed (K), x_bar (6 + 3) and Y_bar (6).
    ps = paths.enumerate_paths("1x1o", 1, "1x1e", "uvu")
    assert len(ps) == 1
    wm = paths.work_model(ps, N, E, K, "uvu")
    assert wm["fwd_flops"] == 2 * E * (K + 6 + 3)
    assert wm["bwd_flops"] == 2 * E * (3 * K + 3 * 6 + 2 * 3)
    # second order per edge and channel: w, w_dot (3K); T, T_dot (3 * 6); m_dot
    # (2 * 3); h, h_dot (2 * 3); A_bar_dot, phi_bar_dot (4K); x_bar_dot (2 * 6 +
    # 2 * 3); Y_bar_dot (2 * 6)
    assert wm["dbl_flops"] == 2 * E * (7 * K + 7 * 6 + 4 * 3 + 2 * 3)


def test_work_model_uvw_hand_count():
    # one path 1o x 1o -> 1e, C_in = 2, C_out = 3, K = 4, N = 5, E = 10, nnz = 6,
    # d1 = d3 = 3. Steps of the receiver-factorised schedule (FMA = 2 flops):
    #   state S (Eqs. 32-33), per edge: 2*2*6 (C) + 2*4*2*3 (phi outer C) = 72 -> 720
    #   mixing m = S A (Eqs. 34-35), per receiver: 2*3*4*2*3 = 144 -> 720
    #   backward: S again 720; A_bar = S^T m_bar 720 and S_bar = m_bar A^T 720
    #   (Eq. 36); edge pass per edge 2*2*6 (C) + 2*4*2*3 (T_bar) + 2*4*2*3
    #   (phi_bar) + 2*2*6 (Y_bar) = 144 -> 1440; source state of x_bar per edge
    #   2*3*6 + 2*4*3*3 = 108 -> 1080; its mixing per source 2*3*4*3*2 = 144 -> 720.
    ps = paths.enumerate_paths("2x1o", 1, "3x1e", "uvw")
    assert len(ps) == 1 and ps[0].n_w == 6
    wm = paths.work_model(ps, 5, 10, 4, "uvw")
    assert wm["fwd_flops"] == 720 + 720
    assert wm["bwd_flops"] == 720 + 720 + 720 + 1440 + 1080 + 720
    # second order: S 720; dS per edge 4*2*6 + 4*4*2*3 = 144 -> 1440; five
    # mixing products 5 * 720; edge pass per edge 10*4*2*3 + 10*2*6 = 360 ->
    # 3600; source states per edge 4*3*6 + 6*4*3*3 = 288 -> 2880; two source
    # mixings 2 * 720
    assert wm["dbl_flops"] == 720 + 1440 + 3600 + 3600 + 2880 + 1440
