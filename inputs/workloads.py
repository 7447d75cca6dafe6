"""The five synthetic workloads of the tensor-product convolution.

They stand in for the pages' datasets (LunaTP §5 / App. A sample OMat24 and
MPTrj structures with periodic neighbour lists; Sobek §5.1 builds radius graphs
on synthetic positions), none of which is available here.

Recipe (seed = workload id; draw order positions, x, A, grad_out):
* positions uniform in a cube; workload 1 is an open 6 A box with a 3 A cutoff;
  workloads 2, 4, 5 are periodic cubes of side (N / rho)^(1/3) with
  rho = d / (4/3 pi r_c^3), r_c = 5 A, d the target mean degree; workload 3
  reuses workload 1's positions;
* edges: every ordered pair i != j closer than r_c (minimum image when periodic),
  emitted in (src, dst) lexicographic order, so the receiver CSR is a real
  reordering;
* Y: component-normalised real spherical harmonics of r_hat_ij, r_ij = r_j - r_i
  (j sender, i receiver), blocks l = 0..L, m = -l..l, l = 1 ordered (y, z, x);
* phi: K Bessel functions sqrt(2/r_c) sin(n pi r / r_c) / r times the cosine
  cutoff (cos(pi r / r_c) + 1) / 2;
* x, grad_out ~ N(0, 1); A ~ N(0, s) with s the standard deviation
  1/sqrt(8) (workload 1), 1/sqrt(K) (2-4), 1/sqrt(16*32) (5);
* floating inputs are drawn in fp64 and rounded once to the workload dtype.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
from scipy.spatial import cKDTree
from scipy.special import sph_harm_y


@dataclass(frozen=True)
class Config:
    id: int
    name: str
    irreps_in: str
    sh_lmax: int
    irreps_out: str
    K: int
    mode: str
    dtype: str          # "f32" | "f64"
    n_nodes: int
    box: float          # cube side (A)
    periodic: bool
    r_cut: float
    a_std: float
    backward: bool
    positions_from: int = 0   # reuse another workload's positions
    irreps_sh: Optional[str] = None   # parities of Y's degrees where not (-1)^l


def _lp(mul: int, lmax: int, all_parities: bool, skip=()) -> str:
    terms = []
    for l in range(lmax + 1):
        nat = "e" if l % 2 == 0 else "o"
        terms.append(f"{mul}x{l}{nat}")
        if all_parities and l > 0:
            terms.append(f"{mul}x{l}{'o' if nat == 'e' else 'e'}")
    return "+".join(t for t in terms if t not in skip)


def _box(n: int, degree: float, r_cut: float) -> float:
    rho = degree / (4.0 / 3.0 * np.pi * r_cut ** 3)
    return float((n / rho) ** (1.0 / 3.0))


CONFIGS = {
    1: Config(1, "tiny check f64 uvu (64 nodes, 6 A open box, r_c 3 A)",
              "8x0e+8x1o+8x2e", 2, _lp(8, 2, True), 8, "uvu", "f64",
              64, 6.0, False, 3.0, 1.0 / np.sqrt(8.0), True),
    2: Config(2, "MACE-like channelwise f32 uvu (4096 atoms, ~32 nbrs, 128 ch, L_sh 3)",
              "128x0e+128x1o", 3, "128x0e+128x1o+128x2e+128x3o", 8, "uvu", "f32",
              4096, _box(4096, 32.0, 5.0), True, 5.0, 1.0 / np.sqrt(8.0), False),
    3: Config(3, "tiny geometry f64 uvu, 64 channels, l <= 3",
              "64x0e+64x1o+64x2e+64x3o", 3, _lp(64, 3, True), 8, "uvu", "f64",
              64, 6.0, False, 3.0, 1.0 / np.sqrt(8.0), True, positions_from=1),
    4: Config(4, "large graph f32 uvu (100k atoms, ~40 nbrs, 64 ch, l <= 2)",
              "64x0e+64x1o+64x2e", 2, _lp(64, 2, True), 8, "uvu", "f32",
              100_000, _box(100_000, 40.0, 5.0), True, 5.0, 1.0 / np.sqrt(8.0), True),
    5: Config(5, "fully connected f32 uvw (16384 atoms, ~32 nbrs, 32 ch, l <= 4, K 16)",
              "32x0e+32x1o+32x2e+32x3o+32x4e", 4, _lp(32, 4, True), 16, "uvw", "f32",
              16_384, _box(16_384, 32.0, 5.0), True, 5.0, 1.0 / np.sqrt(16.0 * 32.0), True),
}


# The ten irrep cases of LunaTP's kernel microbenchmarks (Appendix A.1, Table 1:
# hidden, edge and output irreps), on their workload's shape: 768 atoms,
# periodic, r_c 6 A, 48.6 neighbours on average (OMat24 structures there;
# uniform positions here). Outputs are per path (mode "uvu_paths"): the output
# irreps listed select which (l, p) the paths may produce. K = 8 Bessel
# functions give the per-edge path weights through W = phi A.
_LUNATP = [
    ("C1", "128x0e+64x1e+32x2e", "1x0e+1x1e+1x2e", "224x0e+384x1e+352x2e"),
    ("C2", "128x0e+128x1o+128x2e", "1x0e+1x1o+1x2e+1x3o", "384x0e+640x1o+640x2e+512x3o"),
    ("C3", "128x0e+64x1o+32x2e+32x3o", "1x0e+1x1o+1x2e+1x3o", "256x0e+352x1o+384x2e+320x3o"),
    ("C4", "256x0e+256x1o+256x2e+256x3o", "1x0e+1x1o+1x2e+1x3o", "1024x0e+1536x1o+1792x2e+1536x3o"),
    ("C5", "320x0e+96x1o+64x2e+32x3o+32x4e", "1x0e+1x1o+1x2e+1x3o+1x4e",
     "544x0e+736x1o+832x2e+800x3o+704x4e"),
    ("C6", "128x0e+128x1o+128x2e+128x3o+128x4e", "1x0e+1x1o+1x2e+1x3o+1x4e",
     "640x0e+1024x1o+1280x2e+1280x3o+1152x4e"),
    ("C7", "128x0e+64x1o+32x2e+32x3o+32x4e+32x5o", "1x0e+1x1o+1x2e+1x3o+1x4e+1x5o",
     "320x0e+480x1o+576x2e+608x3o+608x4e+512x5o"),
    ("C8", "96x0e+96x1o+96x2e+96x3o+96x4e+96x5o", "1x0e+1x1o+1x2e+1x3o+1x4e+1x5o",
     "576x0e+960x1o+1248x2e+1344x3o+1344x4e+1152x5o"),
    ("C9", "128x0e+64x1o+32x2e+32x3o+32x4e+32x5o+32x6e", "1x0e+1x1o+1x2e+1x3o+1x4e+1x5o+1x6e",
     "352x0e+544x1o+672x2e+736x3o+768x4e+736x5o+640x6e"),
    ("C10", "64x0e+64x1o+64x2e+64x3o+64x4e+64x5o+64x6e", "1x0e+1x1o+1x2e+1x3o+1x4e+1x5o+1x6e",
     "448x0e+768x1o+1024x2e+1152x3o+1216x4e+1152x5o+1024x6e"),
]
for _k, (_name, _hid, _sh, _out) in enumerate(_LUNATP):
    _cid = 11 + _k
    _lsh = len(_sh.split("+")) - 1
    CONFIGS[_cid] = Config(_cid, f"LunaTP {_name} f32 per-path uvu (768 atoms, ~48.6 nbrs, r_c 6 A, L_sh {_lsh})",
                           _hid, _lsh, _out, 8, "uvu_paths", "f32", 768, _box(768, 48.6, 6.0), True, 6.0,
                           1.0 / np.sqrt(8.0), True, irreps_sh=_sh)
LUNATP_CASES = {name: 11 + k for k, (name, *_r) in enumerate(_LUNATP)}


def _positions(cfg: Config, rng: np.random.Generator) -> np.ndarray:
    return rng.uniform(0.0, cfg.box, size=(cfg.n_nodes, 3))


def morton_order(pos: np.ndarray, box: float, bits: int = 10) -> np.ndarray:
    """Permutation that sorts points along a Z-order (Morton) curve of the box:
    each coordinate quantised to `bits` bits, the bits interleaved x, y, z."""
    q = np.clip((pos / box * (1 << bits)).astype(np.int64), 0, (1 << bits) - 1)
    code = np.zeros(len(pos), np.int64)
    for b in range(bits):
        for d in range(3):
            code |= ((q[:, d] >> b) & 1) << (3 * b + d)
    return np.argsort(code, kind="stable")


def radius_graph(pos: np.ndarray, box: float, periodic: bool, r_cut: float):
    """All ordered pairs (src, dst), src != dst, |r_dst - r_src| < r_cut (min. image)."""
    if periodic:
        tree = cKDTree(np.mod(pos, box), boxsize=box)
    else:
        tree = cKDTree(pos)
    pairs = tree.query_pairs(r_cut, output_type="ndarray")
    if len(pairs) == 0:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    a = np.concatenate([pairs[:, 0], pairs[:, 1]]).astype(np.int64)
    b = np.concatenate([pairs[:, 1], pairs[:, 0]]).astype(np.int64)
    order = np.lexsort((b, a))
    return a[order], b[order]


def edge_vectors(pos, src, dst, box, periodic):
    """r_ij = r_j - r_i for edge j -> i, i.e. sender minus receiver (minimum image)."""
    d = pos[src] - pos[dst]
    if periodic:
        d = d - box * np.round(d / box)
    return d


def spherical_harmonics(lmax: int, vec: np.ndarray) -> np.ndarray:
    """Component-normalised real SH, blocks l = 0..lmax, from scipy's complex Y."""
    v = np.asarray(vec, np.float64)
    r = np.linalg.norm(v, axis=1)
    theta = np.arccos(np.clip(v[:, 2] / r, -1.0, 1.0))
    azim = np.arctan2(v[:, 1], v[:, 0])
    cols = []
    for l in range(lmax + 1):
        s = np.sqrt(4.0 * np.pi)
        blk = np.zeros((len(v), 2 * l + 1))
        for m in range(-l, l + 1):
            if m == 0:
                blk[:, l] = s * sph_harm_y(l, 0, theta, azim).real
            elif m > 0:
                blk[:, l + m] = s * np.sqrt(2.0) * (-1) ** m * sph_harm_y(l, m, theta, azim).real
            else:
                blk[:, l + m] = s * np.sqrt(2.0) * (-1) ** (-m) * sph_harm_y(l, -m, theta, azim).imag
        cols.append(blk)
    return np.concatenate(cols, axis=1)


def bessel_cutoff(r: np.ndarray, K: int, r_cut: float) -> np.ndarray:
    n = np.arange(1, K + 1, dtype=np.float64)
    rr = r[:, None]
    b = np.sqrt(2.0 / r_cut) * np.sin(n[None, :] * np.pi * rr / r_cut) / rr
    env = 0.5 * (np.cos(np.pi * r / r_cut) + 1.0)
    return b * env[:, None]


def _irreps_dim(s: str) -> int:
    tot = 0
    for t in s.split("+"):
        mul, ir = t.split("x")
        tot += int(mul) * (2 * int(ir[:-1]) + 1)
    return tot


@dataclass
class Workload:
    cfg: Config
    pos: np.ndarray
    src: np.ndarray      # COO, int64
    dst: np.ndarray
    Y: np.ndarray        # [E, (L+1)^2] in COO order, workload dtype
    phi: np.ndarray      # [E, K] in COO order, workload dtype
    x: np.ndarray        # [N, C_x] ir_mul, workload dtype
    A: np.ndarray        # [K, N_w], workload dtype
    grad_out: np.ndarray  # [N, C_out], workload dtype
    n_w: int = field(default=0)

    @property
    def n_nodes(self) -> int:
        return self.cfg.n_nodes

    @property
    def n_edges(self) -> int:
        return len(self.src)

    @property
    def np_dtype(self):
        return np.float32 if self.cfg.dtype == "f32" else np.float64


def make_workload(cfg_id: int, n_w: int, n_nodes: Optional[int] = None,
                  edge_keep: Optional[float] = None, c_out: Optional[int] = None,
                  node_order: Optional[str] = None) -> Workload:
    """Build workload ``cfg_id``.

    n_w (the weight count of the operator's path layout) and c_out (the output
    width, needed where the paths define the output blocks) are arguments so that
    this module stays free of the operator's path rules. ``n_nodes`` shrinks a
    periodic workload at fixed density (for fast tests); ``edge_keep`` keeps a
    seeded fraction of the edges (for workspace-versus-edge-count checks).
    ``node_order="morton"`` numbers the nodes along a Z-order curve of their
    positions (a spatially sorted variant; the default keeps generation order,
    which is spatially random).
    """
    cfg = CONFIGS[cfg_id]
    if n_nodes is not None and n_nodes != cfg.n_nodes:
        if not cfg.periodic:
            raise ValueError("only periodic workloads can be resized")
        deg = cfg.n_nodes / cfg.box ** 3
        cfg = Config(**{**cfg.__dict__, "n_nodes": n_nodes,
                        "box": float((n_nodes / deg) ** (1.0 / 3.0))})
    rng = np.random.default_rng(cfg.id)
    if cfg.positions_from:
        pos = _positions(CONFIGS[cfg.positions_from], np.random.default_rng(cfg.positions_from))
    else:
        pos = _positions(cfg, rng)
    if node_order == "morton":
        pos = pos[morton_order(pos, cfg.box)]
    elif node_order is not None:
        raise ValueError(f"unknown node order {node_order!r}")
    src, dst = radius_graph(pos, cfg.box, cfg.periodic, cfg.r_cut)
    if edge_keep is not None:
        keep = np.random.default_rng(1000 + cfg.id).random(len(src)) < edge_keep
        src, dst = src[keep], dst[keep]
    vec = edge_vectors(pos, src, dst, cfg.box, cfg.periodic)
    r = np.linalg.norm(vec, axis=1)
    dt = np.float32 if cfg.dtype == "f32" else np.float64
    Y = spherical_harmonics(cfg.sh_lmax, vec).astype(dt)
    phi = bessel_cutoff(r, cfg.K, cfg.r_cut).astype(dt)
    x = rng.normal(size=(cfg.n_nodes, _irreps_dim(cfg.irreps_in))).astype(dt)
    A = (rng.normal(size=(cfg.K, n_w)) * cfg.a_std).astype(dt)
    g = rng.normal(size=(cfg.n_nodes, c_out if c_out is not None else _irreps_dim(cfg.irreps_out))).astype(dt)
    return Workload(cfg, pos, src, dst, Y, phi, x, A, g, n_w)


# ----------------------------------------------------------------------------- scaling graphs
#
# Sobek §5.1's scaling axes, on synthetic periodic positions at the density of
# the fully connected workload (mean degree 32 at r_c = 5 A): a degree axis
# (one set of 2048 positions, the cutoff set for the wanted mean degree) and a
# graph-count axis (B copies of one 128-node, degree-32 graph). The pages do
# not print the exact grids; the degrees and counts are chosen to span their
# 8.2e3 - 2.1e6 edge range.

SOBEK_RHO = 32.0 / (4.0 / 3.0 * np.pi * 5.0 ** 3)     # atoms per A^3
SOBEK_DEGREES = (4, 8, 16, 32, 64, 128, 256, 512, 1023)
SOBEK_COUNTS = (2, 8, 32, 128, 511)


def _graph_features(pos, src, dst, box, r_cut, irreps_in, sh_lmax, K, n_w, c_out, a_std, seed):
    rng = np.random.default_rng(seed)
    vec = edge_vectors(pos, src, dst, box, True)
    r = np.linalg.norm(vec, axis=1)
    Y = spherical_harmonics(sh_lmax, vec).astype(np.float32)
    phi = bessel_cutoff(r, K, r_cut).astype(np.float32)
    n = len(pos)
    x = rng.normal(size=(n, _irreps_dim(irreps_in))).astype(np.float32)
    A = (rng.normal(size=(K, n_w)) * a_std).astype(np.float32)
    g = rng.normal(size=(n, c_out)).astype(np.float32)
    return Y, phi, x, A, g


def sobek_degree_graph(degree: int, n_nodes: int = 2048, seed: int = 0):
    """(positions, src, dst, box, r_cut): radius graph on fixed periodic
    positions with the cutoff set for a mean receiver degree of `degree`."""
    box = float((n_nodes / SOBEK_RHO) ** (1.0 / 3.0))
    pos = np.random.default_rng(seed).uniform(0.0, box, size=(n_nodes, 3))
    r_cut = float((3.0 * degree / (4.0 * np.pi * SOBEK_RHO)) ** (1.0 / 3.0))
    r_cut = min(r_cut, 0.4999 * box)
    src, dst = radius_graph(pos, box, True, r_cut)
    return pos, src, dst, box, r_cut


def sobek_count_graph(copies: int, n_nodes: int = 128, seed: int = 0):
    """(positions, src, dst, box, r_cut) of `copies` disjoint copies of one
    128-node, mean-degree-32 periodic graph (node ids offset per copy; the
    positions of every copy are the same, each copy in its own periodic box)."""
    box = float((n_nodes / SOBEK_RHO) ** (1.0 / 3.0))
    pos = np.random.default_rng(seed).uniform(0.0, box, size=(n_nodes, 3))
    src, dst = radius_graph(pos, box, True, 5.0)
    off = np.repeat(np.arange(copies, dtype=np.int64) * n_nodes, len(src))
    return (np.tile(pos, (copies, 1)), np.tile(src, copies) + off, np.tile(dst, copies) + off, box, 5.0)


def sobek_workload(graph, irreps: str, sh_lmax: int, K: int, n_w: int, c_out: int, seed: int = 1):
    """Inputs of a fully connected profile (in = out irreps) on a scaling
    graph: Y, phi (K Bessel functions x cosine cutoff), x, A ~ N(0, 1/sqrt(K C)),
    grad_out; float32, COO edge order."""
    pos, src, dst, box, r_cut = graph
    mul0 = int(irreps.split("x")[0])
    Y, phi, x, A, g = _graph_features(pos, src, dst, box, r_cut, irreps, sh_lmax, K, n_w, c_out,
                                      1.0 / np.sqrt(K * mul0), seed)
    return dict(src=src, dst=dst, Y=Y, phi=phi, x=x, A=A, grad_out=g, n_nodes=len(pos))
