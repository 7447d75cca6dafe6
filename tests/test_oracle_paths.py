"""Pins of the oracle's path enumeration against numbers the pages print."""
import os

import pytest

from oracle import paths

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _profile_irreps(profile: str) -> str:
    muls = [int(v) for v in profile.split("/")]
    return "+".join(f"{m}x{l}{'e' if l % 2 == 0 else 'o'}" for l, m in enumerate(muls))


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


@pytest.mark.parametrize("row", list(_rows("sobek_nw.txt")))
def test_sobek_nw(row):
    profile, nw, mw = row.split()
    ir = _profile_irreps(profile)
    lmax = len(profile.split("/")) - 1
    ps = paths.enumerate_paths(ir, lmax, ir, "uvw")
    assert paths.n_weights(ps) == int(nw)
    if mw != "-":
        assert round(4 * 1.0e6 * paths.n_weights(ps) / 2 ** 30, 1) == float(mw)


@pytest.mark.parametrize("row", list(_rows("lunatp_table1_out_mul.txt")))
def test_lunatp_output_multiplicities(row):
    case, hid, edge, out = [c.strip() for c in row.split("|")]
    sh_ir = []
    for t in edge.split("+"):
        ir = t.split("x")[1]
        sh_ir.append((int(ir[:-1]), 1 if ir[-1] == "e" else -1))
    want = {}
    for t in out.split("+"):
        mul, ir = t.split("x")
        want[(int(ir[:-1]), 1 if ir[-1] == "e" else -1)] = int(mul)
    got = paths.concatenated_out_mul(hid, sh_ir, list(want))
    assert got == want, case


def test_uvu_rejects_unequal_multiplicity():
    with pytest.raises(ValueError):
        paths.enumerate_paths("8x0e", 1, "4x1o", "uvu")


def test_layout_offsets_are_contiguous():
    ps = paths.enumerate_paths("4x0e+3x1o", 2, "4x0e+3x1o+2x2e", "uvw")
    off = 0
    for p in ps:
        assert p.w_off == off and p.n_w == p.mul_in * p.mul_out
        assert p.p3 == p.p1 * p.p2 and abs(p.l1 - p.l2) <= p.l3 <= p.l1 + p.l2
        off += p.n_w
