"""Path enumeration and weight layout (oracle; test infrastructure).

Sobek §2.2: an input irrep (l_in, s_in) couples with a spherical-harmonic irrep
(l_sh, s_sh) into l_out in |l_in - l_sh| .. l_in + l_sh with parity s_in * s_sh.
LunaTP §2.1 calls each coupling (l1, l2) -> l a path. Sobek §2.4: path pi carries
n_pi = C_in C_out weights for fully connected (uvw) mixing and n_pi = C for
channelwise (uvu) mixing; N_w = sum_pi n_pi.

Reading of the enumeration order (the pages are silent; it fixes the layout of A
and of the output sums): for each input block in the order written, for l2 =
0..L_sh ascending, for l3 = |l1-l2|..l1+l2 ascending, one path to every output
block of degree l3 and parity p1*p2 (in output order). Output blocks receive the
sum over all their paths. Spherical harmonics carry their natural parity
(-1)^l2 unless an explicit list of (l2, p2) is given.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence, Tuple, Union

from . import irreps as _ir
from .cg import real_cg_sparse


@dataclass(frozen=True)
class Path:
    index: int
    i_in: int       # input block
    l1: int
    p1: int
    l2: int
    p2: int
    l3: int
    p3: int
    i_out: int      # output block
    mul_in: int
    mul_out: int
    w_off: int      # first column of this path in A [K, N_w]
    n_w: int        # columns of this path


def sh_irreps(sh: Union[int, Sequence[Tuple[int, int]]]) -> List[Tuple[int, int]]:
    if isinstance(sh, int):
        return [(l, (-1) ** l) for l in range(sh + 1)]
    return [(int(l), int(p)) for l, p in sh]


def y_offset(l2: int) -> int:
    """Blocks of Y are l = 0..L in order, so block l starts at l^2."""
    return l2 * l2


def per_path_irreps_out(irreps_in: str, sh, irreps_out: str) -> str:
    """Output irreps of the channelwise convolution with one output block per path
    (LunaTP Appendix A.1, Table 1: the outputs of the uvu paths are concatenated).

    Paths are enumerated in the same order as ``enumerate_paths``; a path exists
    when its (l3, p3) appears in ``irreps_out`` (multiplicities there are
    ignored), and it owns a block of its input multiplicity.
    """
    bin_ = _ir.parse(irreps_in)
    allowed = {(b.l, b.p) for b in _ir.parse(irreps_out)}
    terms = []
    for b1 in bin_:
        for (l2, p2) in sh_irreps(sh):
            for l3 in range(abs(b1.l - l2), b1.l + l2 + 1):
                p3 = b1.p * p2
                if (l3, p3) in allowed:
                    terms.append(f"{b1.mul}x{l3}{'e' if p3 == 1 else 'o'}")
    return "+".join(terms)


def enumerate_paths(irreps_in: str, sh, irreps_out: str, mode: str) -> List[Path]:
    """Paths in enumeration order. mode "uvu" / "uvw": every output block of the
    right (l3, p3) receives a path and sums its paths; mode "uvu_paths": one
    output block per path, in path order (``irreps_out`` only selects which
    (l3, p3) exist; the blocks are those of ``per_path_irreps_out``)."""
    if mode == "uvu_paths":
        bin_ = _ir.parse(irreps_in)
        allowed = {(b.l, b.p) for b in _ir.parse(irreps_out)}
        paths = []
        w = 0
        for i1, b1 in enumerate(bin_):
            for (l2, p2) in sh_irreps(sh):
                for l3 in range(abs(b1.l - l2), b1.l + l2 + 1):
                    p3 = b1.p * p2
                    if (l3, p3) in allowed:
                        k = len(paths)
                        paths.append(Path(k, i1, b1.l, b1.p, l2, p2, l3, p3, k, b1.mul, b1.mul, w, b1.mul))
                        w += b1.mul
        return paths
    bin_ = _ir.parse(irreps_in)
    bout = _ir.parse(irreps_out)
    shl = sh_irreps(sh)
    paths: List[Path] = []
    w = 0
    for i1, b1 in enumerate(bin_):
        for (l2, p2) in shl:
            for l3 in range(abs(b1.l - l2), b1.l + l2 + 1):
                p3 = b1.p * p2
                for io, bo in enumerate(bout):
                    if bo.l != l3 or bo.p != p3:
                        continue
                    if mode == "uvu":
                        if bo.mul != b1.mul:
                            raise ValueError("uvu needs equal input and output multiplicity "
                                             f"on every path, got {b1.mul} -> {bo.mul}")
                        nw = b1.mul
                    elif mode == "uvw":
                        nw = b1.mul * bo.mul
                    else:
                        raise ValueError(mode)
                    paths.append(Path(len(paths), i1, b1.l, b1.p, l2, p2, l3, p3, io,
                                      b1.mul, bo.mul, w, nw))
                    w += nw
    return paths


def n_weights(paths: List[Path]) -> int:
    return sum(p.n_w for p in paths)


def concatenated_out_mul(irreps_in: str, sh, out_lp: Sequence[Tuple[int, int]]):
    """Per-path concatenated uvu output multiplicity per output (l, p).

    LunaTP Table 1 lists, for each case, output irreps whose multiplicity is the
    sum over paths into (l, p) of the path's input multiplicity (uvu, one output
    slot per path). Used as a pin of the enumeration rule.
    """
    bin_ = _ir.parse(irreps_in)
    shl = sh_irreps(sh)
    want = set((int(l), int(p)) for l, p in out_lp)
    tot = {lp: 0 for lp in want}
    for b1 in bin_:
        for (l2, p2) in shl:
            for l3 in range(abs(b1.l - l2), b1.l + l2 + 1):
                key = (l3, b1.p * p2)
                if key in want:
                    tot[key] += b1.mul
    return tot


def work_model(paths: List[Path], n_nodes: int, n_edges: int, K: int, mode: str) -> dict:
    """Algorithmic flop counts (FMA = 2 flops) of the streamed schedules.

    uvu (Sobek §3.1 order, w live only until consumed), per edge, channel, path:
      forward  K (w = phi . A) + nnz (CG contraction) + (2 l3 + 1) (weighted
               accumulate);
      backward 3 K (w, phi_bar, A_bar) + 3 nnz (h, x_bar, Y_bar contractions)
               + 2 (2 l3 + 1).
    uvw (Sobek §4.2 Eqs. 32-35 forward, §4.3 backward), per path with
    d1 = 2 l1 + 1, d3 = 2 l3 + 1:
      state  e  = E (2 C_in nnz + 2 K C_in d3)        (Eqs. 32-33)
      mixing r  = N 2 d3 K C_in C_out                 (Eqs. 34-35)
      forward  = e + r;
      backward = e (state recomputed) + 2 r (A_bar = S^T m_bar and
               S_bar = m_bar A^T, Eq. 36) + E (4 K C_in d3 + 4 C_in nnz) (edge
               pass: C, T_bar, phi_bar, Y_bar) + E (2 C_out nnz + 2 K C_out d1)
               (source state of x_bar) + N 2 d1 K C_out C_in (its mixing).
    Second order (Sobek §3.3 / §4.4), along (x_dot, Y_dot, phi_dot, A_dot):
      uvu per edge, channel, path: w, w_dot (3 K); T, T_dot (3 nnz); m_dot
          (2 d3); h, h_dot (2 d3); A_bar_dot, phi_bar_dot (4 K); x_bar_dot
          (2 nnz + 2 d1); Y_bar_dot (2 nnz);
      uvw: e + E (4 C_in nnz + 4 K C_in d3) (directional state dS) + 5 r (dm =
          dS A + S dA, dA_bar = dS^T m_bar, S_bar, dS_bar = m_bar dA^T) +
          E (10 K C_in d3 + 10 C_in nnz) (edge pass on S_bar, dS_bar, C, C_dot) +
          E (4 C_out nnz + 6 K C_out d1) (source states S', dS') + 2 N 2 d1 K
          C_out C_in (x_bar_dot = dS' A' + S' dA').
    """
    fwd = 0
    bwd = 0
    dbl = 0
    for p in paths:
        nnz = len(real_cg_sparse(p.l1, p.l2, p.l3))
        d1 = 2 * p.l1 + 1
        d3 = 2 * p.l3 + 1
        if mode in ("uvu", "uvu_paths"):
            C = p.mul_in
            fwd += 2 * n_edges * C * (K + nnz + d3)
            bwd += 2 * n_edges * C * (3 * K + 3 * nnz + 2 * d3)
            dbl += 2 * n_edges * C * (7 * K + 7 * nnz + 4 * d3 + 2 * d1)
        else:
            ci, co = p.mul_in, p.mul_out
            e = n_edges * (2 * ci * nnz + 2 * K * ci * d3)
            r = n_nodes * 2 * d3 * K * ci * co
            fwd += e + r
            bwd += (e + 2 * r + n_edges * (4 * K * ci * d3 + 4 * ci * nnz)
                    + n_edges * (2 * co * nnz + 2 * K * co * d1) + n_nodes * 2 * d1 * K * co * ci)
            dbl += (e + n_edges * (4 * ci * nnz + 4 * K * ci * d3) + 5 * r
                    + n_edges * (10 * K * ci * d3 + 10 * ci * nnz)
                    + n_edges * (4 * co * nnz + 6 * K * co * d1) + 2 * n_nodes * 2 * d1 * K * co * ci)
    return {"fwd_flops": fwd, "bwd_flops": bwd, "dbl_flops": dbl}
