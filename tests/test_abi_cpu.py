"""CPU checks of the C-ABI library: it loads, exports every symbol that
include/tpconv.h declares, and its host planner agrees with the oracle (paths,
weight layout, real CG coefficients, work model). No CUDA call is made."""
import ctypes
import os
import re

import numpy as np
import pytest

import clebsch_gordan_tensor_node_b200 as tpc
from clebsch_gordan_tensor_node_b200 import _lib
from inputs import CONFIGS
from oracle import cg as ocg
from oracle import paths as opaths

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _sh(c):
    """Y's degrees and parities of a workload (natural parity unless given)."""
    if c.irreps_sh is None:
        return c.sh_lmax
    return [(int(t.split("x")[1][:-1]), 1 if t[-1] == "e" else -1) for t in c.irreps_sh.split("+")]


def _declared():
    txt = open(os.path.join(ROOT, "include", "tpconv.h")).read()
    return sorted(set(re.findall(r"^\s*(?:int|const char\*)\s+(tp_\w+)\s*\(", txt, re.M)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 14
    L = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_lib.SIGNATURES)


@pytest.mark.parametrize("cid", sorted(CONFIGS))
def test_planner_matches_oracle_paths(cid):
    c = CONFIGS[cid]
    plan = tpc.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.dtype, irreps_sh=c.irreps_sh)
    ps = opaths.enumerate_paths(c.irreps_in, _sh(c), c.irreps_out, c.mode)
    assert plan.n_paths == len(ps)
    assert plan.n_w == opaths.n_weights(ps)
    for k, p in enumerate(ps):
        q = plan.path(k)
        assert (q.l1, q.p1, q.l2, q.p2, q.l3, q.p3) == (p.l1, p.p1, p.l2, p.p2, p.l3, p.p3)
        assert (q.block_in, q.block_out, q.w_off, q.n_w) == (p.i_in, p.i_out, p.w_off, p.n_w)
        assert q.nnz == len(ocg.real_cg_sparse(p.l1, p.l2, p.l3))


def test_planner_cg_matches_oracle():
    plan = tpc.Plan("1x0e+1x1o+1x2e+1x3o+1x4e", 4,
                    "1x0e+1x1o+1x1e+1x2e+1x2o+1x3o+1x3e+1x4e+1x4o", 4, "uvw", "f64")
    for k in range(plan.n_paths):
        p = plan.path(k)
        R = ocg.real_cg(p.l1, p.l2, p.l3)
        got = plan.cg(k)
        assert len(got) == int((R != 0).sum())
        for m1, m2, m3, c in got:
            assert abs(c - R[m1, m2, m3]) <= 1e-15 * abs(R[m1, m2, m3])  # a few ulp


@pytest.mark.parametrize("cid", sorted(CONFIGS))
def test_work_model_matches_oracle(cid):
    c = CONFIGS[cid]
    plan = tpc.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.dtype, irreps_sh=c.irreps_sh)
    ps = opaths.enumerate_paths(c.irreps_in, _sh(c), c.irreps_out, c.mode)
    N, E = 1000, 31000
    want = opaths.work_model(ps, N, E, c.K, c.mode)
    assert plan.work_model(N, E, 0)[0] == pytest.approx(want["fwd_flops"], rel=1e-12)
    assert plan.work_model(N, E, 1)[0] == pytest.approx(want["bwd_flops"], rel=1e-12)
    assert plan.work_model(N, E, 2)[0] == pytest.approx(want["dbl_flops"], rel=1e-12)


def test_workspace_does_not_depend_on_edges():
    c = CONFIGS[4]
    plan = tpc.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.dtype)
    # the C signature takes no edge count at all; check it is finite and fixed in N
    a = plan.workspace_size(100_000, 1)
    b = plan.workspace_size(1_000_000, 1)
    assert a == b and 0 < a < 256 << 20
    assert plan.workspace_size(100_000, 0) == 0


@pytest.mark.parametrize("args,status", [
    (("8x0e+", 1, "8x0e", 8, "uvu", "f32"), -1),
    (("8x0e", 1, "8x0q", 8, "uvu", "f32"), -1),
    (("8x0e", 1, "4x1o", 8, "uvu", "f32"), -2),     # uvu with unequal multiplicity
    (("8x7e", 1, "8x7e", 8, "uvu", "f32"), -2),     # degree above the compiled limit (6)
    (("8x5e", 1, "8x5e", 8, "uvw", "f32"), -2),     # fully connected: limit 4
    (("8x5e", 1, "8x5e", 8, "uvu", "f64"), -2),     # fp64: limit 4
    (("8x5e", 1, "8x5e", 16, "uvu", "f32"), -2),    # K above 8: limit 4
    (("8x0e", 1, "8x3o", 8, "uvu_paths", "f32"), -1),   # no path reaches the outputs
    (("8x0e", 1, "8x0e", 33, "uvu", "f32"), -2),    # K above 16
])
def test_plan_errors(args, status):
    with pytest.raises(tpc.TpConvError) as ei:
        tpc.Plan(*args)
    assert ei.value.status == status


def test_launch_count_matches_the_schedule():
    """Kernels one call enqueues: uvu forward 1, backward 3 (edge, source, slot
    sum); uvw per receiver chunk 2 forward (state, mixing) and 5 backward."""
    import clebsch_gordan_tensor_node_b200 as tpc
    uvu = tpc.Plan("8x0e+8x1o", 1, "8x0e+8x1o", 8, "uvu", "f32")
    assert uvu.launch_count(1000, 0) == 1 and uvu.launch_count(1000, 1) == 3
    assert uvu.launch_count(0, 0) == 0
    uvw = tpc.Plan("8x0e+8x1o", 1, "8x0e+8x1o", 8, "uvw", "f32")
    # a graph small enough for one state chunk in each direction, one GEMM batch
    assert uvw.launch_count(100, 0) == 1 + 2
    assert uvw.launch_count(100, 1) == 1 + 5 + 2 + 1
    # second order: pack A and dA; per receiver chunk 8 + 5 GEMM batches, per
    # source chunk 3 + 2, unpack
    assert uvw.launch_count(100, 2) == 2 + 13 + 5 + 1
    assert uvu.launch_count(1000, 2) == 4


def test_state_budget_sets_chunks_and_workspace():
    """A smaller uvw state budget gives more receiver chunks (more launches) and a
    smaller workspace; a budget below one node's state is rejected."""
    c = CONFIGS[5]
    plan = tpc.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.dtype)
    N = 4000
    big_ws, big_n = plan.workspace_size(N, 1), plan.launch_count(N, 1)
    plan.set_state_budget(64 << 20)
    assert plan.workspace_size(N, 1) < big_ws
    assert plan.launch_count(N, 1) > big_n
    assert plan.launch_count(N, 0) > 3
    with pytest.raises(tpc.TpConvError) as ei:
        plan.set_state_budget(1024)
    assert ei.value.status == -1 and "one node" in str(ei.value)
    uvu = tpc.Plan("8x0e", 0, "8x0e", 4, "uvu", "f32")
    uvu.set_state_budget(1)            # no state chunks: accepted, no effect
    assert uvu.workspace_size(10, 0) == 0


def test_per_path_outputs_match_lunatp_table1():
    """Per-path (concatenated) channelwise outputs: the planner's output blocks,
    summed per (l, p), give the output multiplicities of LunaTP Appendix A.1,
    Table 1 for all ten cases, and every block belongs to exactly one path."""
    from inputs import LUNATP_CASES
    gold = {}
    for line in open(os.path.join(ROOT, "tests", "golden", "lunatp_table1_out_mul.txt")):
        if line.strip() and not line.startswith("#"):
            case, _, _, out = [c.strip() for c in line.split("|")]
            gold[case] = {}
            for t in out.split("+"):
                mul, ir = t.split("x")
                gold[case][(int(ir[:-1]), 1 if ir[-1] == "e" else -1)] = int(mul)
    for case, cid in LUNATP_CASES.items():
        c = CONFIGS[cid]
        plan = tpc.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.dtype, irreps_sh=c.irreps_sh)
        assert plan.info.mode == 2
        tot = {}
        outs = set()
        for k in range(plan.n_paths):
            p = plan.path(k)
            assert p.block_out == k and p.mul_out == p.mul_in
            outs.add(p.out_off)
            tot[(p.l3, p.p3)] = tot.get((p.l3, p.p3), 0) + p.mul_in
        assert tot == gold[case], case
        assert len(outs) == plan.n_paths


def test_schedule_option():
    """The receiver-state order is accepted for channelwise plans within its
    compiled limits and rejected outside them."""
    uvu = tpc.Plan("8x0e+8x1o", 1, "8x0e+8x1o", 8, "uvu", "f32")
    uvu.set_schedule("receiver_state")
    uvu.set_schedule("streamed")
    wide = tpc.Plan("8x0e", 1, "8x0e+8x1o", 16, "uvu", "f32")
    with pytest.raises(tpc.TpConvError) as ei:
        wide.set_schedule("receiver_state")
    assert ei.value.status == -2
    uvw = tpc.Plan("8x0e", 1, "8x0e+8x1o", 8, "uvw", "f32")
    uvw.set_schedule("receiver_state")
    with pytest.raises(tpc.TpConvError):
        uvw.set_schedule("streamed")
