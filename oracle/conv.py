"""The convolution, its first backward, and two reassociated schedules (oracle).

Test infrastructure. Definitions followed:

* Sobek §2.4: m_i = sum_{j in N(i)} sum_pi sum_a W_{ij,pi,a} T_{pi,a}(x_j, Y_ij)
  with W_{ij,pi,a} = sum_q phi_{ij,q} A_{q,pi,a} (radial factorisation).
* Sobek §2.5 / LunaTP Algorithm 1: the materialised order -- form W and the
  edge messages M for a chunk of edges, then scatter-add M into the receivers.
* T_{pi,a}: the CG product of LunaTP §2.1 Eq. 1, in the real basis of
  ``oracle.cg.real_cg``; uvu ties output channel to input channel (a = u),
  uvw mixes them (a = (u, w)), Sobek §2.3.
* Sobek §3.2 / LunaTP Algorithm 2: h = <m_bar_i, T>, A_bar = sum phi h,
  phi_bar = sum A h, x_bar and Y_bar through the adjoints of the two partial
  Jacobians of the bilinear T, weighted by w.
* Sobek §3.3 (Eqs. 23-31) / LunaTP Algorithm 3: the second-order program, the
  product rule applied to w, T, m, h and the two operand adjoints along
  directions (x_dot, Y_dot, phi_dot, A_dot).
* Sobek §3.1 (streamed order, w live only until consumed) and §4.2 Eqs. 32-35
  (receiver state S, then m = S A) are written as separate loop nests, used only
  to check by brute force on tiny graphs that all orders agree.

Layouts: x [N, C_x] and out [N, C_out] in ir_mul; Y [E, (L+1)^2] with blocks
l = 0..L; phi [E, K]; A [K, N_w] with path pi in columns [w_off, w_off + n_w),
uvu columns = u, uvw columns = u * C_out + w. Edges are given as COO (src, dst)
in any order; all arithmetic is fp64.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np

from . import irreps as _ir
from .cg import real_cg
from .paths import Path, enumerate_paths, n_weights, per_path_irreps_out, y_offset


@dataclass
class Problem:
    irreps_in: str
    sh_lmax: int
    irreps_out: str
    K: int
    mode: str
    irreps_sh: Optional[str] = None   # explicit parities of Y's degrees ("1x0e+1x1e+...")

    def __post_init__(self):
        self.bin = _ir.parse(self.irreps_in)
        sh = self.sh_lmax
        if self.irreps_sh is not None:
            sh = [(b.l, b.p) for b in _ir.parse(self.irreps_sh)]
            assert [l for l, _ in sh] == list(range(self.sh_lmax + 1))
        self.paths: List[Path] = enumerate_paths(self.irreps_in, sh, self.irreps_out, self.mode)
        if self.mode == "uvu_paths":
            # one output block per path (LunaTP Appendix A.1): irreps_out only
            # selects which (l, p) exist; each path is channelwise on its block
            self.irreps_out = per_path_irreps_out(self.irreps_in, sh, self.irreps_out)
            self.mode = "uvu"
        self.bout = _ir.parse(self.irreps_out)
        self.c_in = _ir.dim(self.bin)
        self.c_out = _ir.dim(self.bout)
        self.dim_y = (self.sh_lmax + 1) ** 2
        self.n_w = n_weights(self.paths)


def _T(p: Path, xj: np.ndarray, Ye: np.ndarray) -> np.ndarray:
    """T[e, m3, u] = sum_{m1,m2} R[m1,m2,m3] x_j[e, m1, u] Y[e, m2] (LunaTP Eq. 1)."""
    R = real_cg(p.l1, p.l2, p.l3)
    return np.einsum("abc,eau,eb->ecu", R, xj, Ye, optimize=True)


def _blocks(pr: Problem, p: Path, x, Y, src):
    b1 = pr.bin[p.i_in]
    xj = _ir.block_view(x[src], b1)                       # [e, 2l1+1, mul_in]
    Ye = Y[:, y_offset(p.l2):y_offset(p.l2) + 2 * p.l2 + 1]
    return xj, Ye


def _chunk(pr: Problem, chunk: int) -> int:
    """Edges per materialised chunk, bounded so that W [chunk, N_w] and the edge
    messages [chunk, C_out] (and their adjoints) each stay <= 1 GiB."""
    return max(1, min(chunk, (1 << 27) // max(1, pr.n_w, pr.c_out, pr.c_in)))


def forward(pr: Problem, x, Y, phi, A, src, dst, n_nodes: int, chunk: int = 65536):
    """Materialised forward: per edge chunk W = phi A, messages M, scatter-add."""
    chunk = _chunk(pr, chunk)
    x = np.asarray(x, np.float64)
    out = np.zeros((n_nodes, pr.c_out))
    E = len(src)
    for s in range(0, E, chunk):
        sl = slice(s, min(E, s + chunk))
        sc, dc, Yc, pc = src[sl], dst[sl], np.asarray(Y[sl], np.float64), np.asarray(phi[sl], np.float64)
        W = pc @ np.asarray(A, np.float64)                # [e, N_w] materialised
        M = np.zeros((len(sc), pr.c_out))
        for p in pr.paths:
            xj, Ye = _blocks(pr, p, x, Yc, sc)
            T = _T(p, xj, Ye)                             # [e, 2l3+1, mul_in]
            bo = pr.bout[p.i_out]
            Mo = _ir.block_view(M, bo)                    # view [e, 2l3+1, mul_out]
            Wp = W[:, p.w_off:p.w_off + p.n_w]
            if pr.mode == "uvu":
                Mo += Wp[:, None, :] * T
            else:
                Mo += np.einsum("euw,ecu->ecw", Wp.reshape(-1, p.mul_in, p.mul_out), T)
        np.add.at(out, dc, M)
    return out


def backward(pr: Problem, x, Y, phi, A, src, dst, grad_out, n_nodes: int, chunk: int = 65536):
    """Explicit first-order adjoints (Sobek §3.2, LunaTP Algorithm 2).

    Returns grad_x [N, C_x], grad_Y [E, dimY], grad_phi [E, K], grad_A [K, N_w].
    """
    chunk = _chunk(pr, chunk)
    x = np.asarray(x, np.float64)
    A = np.asarray(A, np.float64)
    g = np.asarray(grad_out, np.float64)
    E = len(src)
    gx = np.zeros((n_nodes, pr.c_in))
    gY = np.zeros((E, pr.dim_y))
    gphi = np.zeros((E, pr.K))
    gA = np.zeros_like(A)
    for s in range(0, E, chunk):
        sl = slice(s, min(E, s + chunk))
        sc, dc = src[sl], dst[sl]
        Yc, pc = np.asarray(Y[sl], np.float64), np.asarray(phi[sl], np.float64)
        W = pc @ A
        Wbar = np.zeros_like(W)                           # materialised per chunk
        gi = g[dc]
        gxc = np.zeros((len(sc), pr.c_in))
        for p in pr.paths:
            xj, Ye = _blocks(pr, p, x, Yc, sc)
            R = real_cg(p.l1, p.l2, p.l3)
            T = _T(p, xj, Ye)
            go = _ir.block_view(gi, pr.bout[p.i_out])     # [e, 2l3+1, mul_out]
            Wp = W[:, p.w_off:p.w_off + p.n_w]
            if pr.mode == "uvu":
                h = np.einsum("ecu,ecu->eu", go, T)
                wg = Wp[:, None, :] * go                  # [e, 2l3+1, mul_in]
            else:
                h = np.einsum("ecw,ecu->euw", go, T).reshape(len(sc), -1)
                wg = np.einsum("euw,ecw->ecu", Wp.reshape(-1, p.mul_in, p.mul_out), go)
            Wbar[:, p.w_off:p.w_off + p.n_w] = h
            # x_bar_j += sum w D_x T^* m_bar ;  Y_bar += sum w D_Y T^* m_bar
            bx = np.einsum("abc,eb,ecu->eau", R, Ye, wg, optimize=True)
            _ir.block_view(gxc, pr.bin[p.i_in])[...] += bx
            gY[sl, y_offset(p.l2):y_offset(p.l2) + 2 * p.l2 + 1] += np.einsum(
                "abc,eau,ecu->eb", R, xj, wg, optimize=True)
        gA += pc.T @ Wbar
        gphi[sl] = Wbar @ A.T
        np.add.at(gx, sc, gxc)
    return gx, gY, gphi, gA


def double_backward(pr: Problem, x, Y, phi, A, src, dst, grad_out, dx, dY, dphi, dA, n_nodes: int,
                    chunk: int = 65536):
    """Second-order program of Sobek §3.3 (Eqs. 23-31), the directional
    derivative of the forward output and of the four first-order adjoints along
    (dx, dY, dphi, dA), with the output adjoint grad_out held fixed:

      w_dot  = phi_dot A + phi A_dot                    T_dot = D_xT[x_dot] + D_YT[Y_dot]
      m_dot  = sum (w_dot T + w T_dot)                  h_dot = <m_bar, T_dot>
      A_bar_dot   = sum phi_dot h + phi h_dot           phi_bar_dot = A_dot h + A h_dot
      x_bar_dot_j = sum w_dot B^x + w B^x_dot           Y_bar_dot   = sum w_dot B^Y + w B^Y_dot
      with B^x = D_xT^* m_bar, B^Y = D_YT^* m_bar and their directional derivatives
      (bilinearity: B^x_dot uses Y_dot, B^Y_dot uses x_dot).

    This is also the product of the Hessian of <m_bar, m> with the direction and
    the forward Jacobian applied to it, i.e. what LunaTP Algorithm 3 returns for
    cotangents (dx, dY, dphi, dA) of the first-order outputs. Edge-chunked and
    materialised like ``backward``. Returns (m_dot [N, C_out], x_bar_dot [N, C_x],
    Y_bar_dot [E, dimY], phi_bar_dot [E, K], A_bar_dot [K, N_w]).
    """
    chunk = _chunk(pr, chunk)
    f = lambda a: np.asarray(a, np.float64)
    x, A, g, dx, dA = f(x), f(A), f(grad_out), f(dx), f(dA)
    E = len(src)
    mdot = np.zeros((n_nodes, pr.c_out))
    gx = np.zeros((n_nodes, pr.c_in))
    gY = np.zeros((E, pr.dim_y))
    gphi = np.zeros((E, pr.K))
    gA = np.zeros_like(A)
    for s in range(0, E, chunk):
        sl = slice(s, min(E, s + chunk))
        sc, dc = src[sl], dst[sl]
        Yc, pc, dYc, dpc = f(Y[sl]), f(phi[sl]), f(dY[sl]), f(dphi[sl])
        W = pc @ A                                        # w
        Wd = dpc @ A + pc @ dA                            # w_dot
        Wbar = np.zeros_like(W)                           # h
        Wbard = np.zeros_like(W)                          # h_dot
        gi = g[dc]
        Mc = np.zeros((len(sc), pr.c_out))
        gxc = np.zeros((len(sc), pr.c_in))
        for p in pr.paths:
            b1, bo = pr.bin[p.i_in], pr.bout[p.i_out]
            xj = _ir.block_view(x[sc], b1)
            dxj = _ir.block_view(dx[sc], b1)
            y0 = y_offset(p.l2)
            Ye, dYe = Yc[:, y0:y0 + 2 * p.l2 + 1], dYc[:, y0:y0 + 2 * p.l2 + 1]
            R = real_cg(p.l1, p.l2, p.l3)
            T = _T(p, xj, Ye)
            Td = _T(p, dxj, Ye) + _T(p, xj, dYe)           # T_dot
            go = _ir.block_view(gi, bo)
            Mo = _ir.block_view(Mc, bo)
            Wp = W[:, p.w_off:p.w_off + p.n_w]
            Wdp = Wd[:, p.w_off:p.w_off + p.n_w]
            if pr.mode == "uvu":
                Mo += Wdp[:, None, :] * T + Wp[:, None, :] * Td          # m_dot
                h = np.einsum("ecu,ecu->eu", go, T)
                hd = np.einsum("ecu,ecu->eu", go, Td)
                wg = Wp[:, None, :] * go
                wgd = Wdp[:, None, :] * go
            else:
                W3 = Wp.reshape(-1, p.mul_in, p.mul_out)
                Wd3 = Wdp.reshape(-1, p.mul_in, p.mul_out)
                Mo += np.einsum("euw,ecu->ecw", Wd3, T) + np.einsum("euw,ecu->ecw", W3, Td)
                h = np.einsum("ecw,ecu->euw", go, T).reshape(len(sc), -1)
                hd = np.einsum("ecw,ecu->euw", go, Td).reshape(len(sc), -1)
                wg = np.einsum("euw,ecw->ecu", W3, go)
                wgd = np.einsum("euw,ecw->ecu", Wd3, go)
            Wbar[:, p.w_off:p.w_off + p.n_w] = h
            Wbard[:, p.w_off:p.w_off + p.n_w] = hd
            # x_bar_dot: w_dot D_xT^*(Y) m_bar + w D_xT^*(Y_dot) m_bar
            bx = (np.einsum("abc,eb,ecu->eau", R, Ye, wgd, optimize=True)
                  + np.einsum("abc,eb,ecu->eau", R, dYe, wg, optimize=True))
            _ir.block_view(gxc, b1)[...] += bx
            # Y_bar_dot: w_dot D_YT^*(x) m_bar + w D_YT^*(x_dot) m_bar
            gY[sl, y0:y0 + 2 * p.l2 + 1] += (np.einsum("abc,eau,ecu->eb", R, xj, wgd, optimize=True)
                                             + np.einsum("abc,eau,ecu->eb", R, dxj, wg, optimize=True))
        gA += dpc.T @ Wbar + pc.T @ Wbard                 # A_bar_dot
        gphi[sl] = Wbar @ dA.T + Wbard @ A.T              # phi_bar_dot
        np.add.at(mdot, dc, Mc)
        np.add.at(gx, sc, gxc)
    return mdot, gx, gY, gphi, gA


# ------------------------------------------------------------------ reassociated orders

def forward_streamed(pr: Problem, x, Y, phi, A, rowptr, senders, perm):
    """Sobek §3.1 order: per receiver, per edge, per path and channel, the scalar
    w = sum_q phi_q A_q is formed, consumed at once, and dropped (no W, no M).
    Plain loops; for tiny graphs only. Y, phi are in COO order, indexed via perm.
    """
    N = len(rowptr) - 1
    out = np.zeros((N, pr.c_out))
    for i in range(N):
        for k in range(rowptr[i], rowptr[i + 1]):
            j, e = senders[k], perm[k]
            for p in pr.paths:
                b1, bo = pr.bin[p.i_in], pr.bout[p.i_out]
                R = real_cg(p.l1, p.l2, p.l3)
                xj = _ir.block_view(x[j], b1)
                Ye = Y[e, y_offset(p.l2):y_offset(p.l2) + 2 * p.l2 + 1]
                o = _ir.block_view(out[i], bo)
                for u in range(p.mul_in):
                    t = np.einsum("abc,a,b->c", R, xj[:, u], Ye)
                    if pr.mode == "uvu":
                        w = float(phi[e] @ A[:, p.w_off + u])
                        o[:, u] += w * t
                    else:
                        for wo in range(p.mul_out):
                            w = float(phi[e] @ A[:, p.w_off + u * p.mul_out + wo])
                            o[:, wo] += w * t
    return out


def forward_receiver_factorised(pr: Problem, x, Y, phi, A, rowptr, senders, perm):
    """Sobek §4.2: C (Eq. 32), receiver state S (Eq. 33) with no output-channel
    axis, then one mixing per receiver m = S A (Eqs. 34-35)."""
    N = len(rowptr) - 1
    out = np.zeros((N, pr.c_out))
    for i in range(N):
        for p in pr.paths:
            b1, bo = pr.bin[p.i_in], pr.bout[p.i_out]
            R = real_cg(p.l1, p.l2, p.l3)
            S = np.zeros((pr.K, p.mul_in, 2 * p.l3 + 1))            # S_{i,pi,q,u,mo}
            for k in range(rowptr[i], rowptr[i + 1]):
                j, e = senders[k], perm[k]
                xj = _ir.block_view(x[j], b1)
                Ye = Y[e, y_offset(p.l2):y_offset(p.l2) + 2 * p.l2 + 1]
                Cm = np.einsum("abc,au,b->uc", R, xj, Ye)           # C_{pi,u,mo}
                S += phi[e][:, None, None] * Cm[None]
            o = _ir.block_view(out[i], bo)
            Ap = A[:, p.w_off:p.w_off + p.n_w]
            if pr.mode == "uvu":
                o += np.einsum("quc,qu->cu", S, Ap)
            else:
                o += np.einsum("quc,quw->cw", S, Ap.reshape(pr.K, p.mul_in, p.mul_out))
    return out
