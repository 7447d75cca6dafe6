"""GPU parity on the ten irrep cases of LunaTP's kernel microbenchmarks
(Appendix A.1, Table 1): channelwise products with one output block per path,
degrees up to 6, the spherical harmonics all even in case C1.

Each case runs on its workload's geometry (r_c 6 A, ~48.6 neighbours) at 112
atoms, small enough for the oracle; forward and first backward for every case,
the second-order program for four of them, all through the C ABI against the
oracle at the fp32 bar (max|gpu - oracle| / max|oracle| <= 1e-4).
"""
import numpy as np
import pytest

import clebsch_gordan_tensor_node_b200 as tpc
from gpu_util import TOL, GpuRun, plan_for, problem, rel_err, workload
from inputs import LUNATP_CASES
from oracle import conv as oconv

pytestmark = pytest.mark.gpu

N_SMALL = 112


@pytest.mark.parametrize("case", sorted(LUNATP_CASES, key=lambda c: int(c[1:])))
def test_lunatp_case_forward_backward(case):
    cid = LUNATP_CASES[case]
    wl = workload(cid, n_nodes=N_SMALL)
    run = GpuRun(plan_for(cid), wl)
    pr = problem(cid)
    assert run.plan.c_out == pr.c_out and run.plan.n_w == pr.n_w
    out = run.forward()
    want = oconv.forward(pr, wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.n_nodes)
    assert rel_err(out.cpu().numpy(), want) <= TOL["f32"], "out"
    gx, gY, gphi, gA = run.backward()
    ox, oY, ophi, oA = oconv.backward(pr, wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.grad_out, wl.n_nodes)
    assert rel_err(gx.cpu().numpy(), ox) <= TOL["f32"], "grad_x"
    assert rel_err(run.to_coo(gY), oY) <= TOL["f32"], "grad_Y"
    assert rel_err(run.to_coo(gphi), ophi) <= TOL["f32"], "grad_phi"
    assert rel_err(gA.cpu().numpy(), oA) <= TOL["f32"], "grad_A"
    assert tpc.tp_get_device_error() == 0


@pytest.mark.parametrize("case", ["C1", "C5", "C7", "C10"])
def test_lunatp_case_double_backward(case):
    from test_gpu_double_backward import _dbl, _directions
    cid = LUNATP_CASES[case]
    wl = workload(cid, n_nodes=N_SMALL)
    run = GpuRun(plan_for(cid), wl)
    d = _directions(wl, 50 + cid)
    got = _dbl(run, d)
    want = oconv.double_backward(problem(cid), wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.grad_out, *d,
                                 wl.n_nodes)
    for k, (g, w) in enumerate(zip(got, want)):
        gn = run.to_coo(g) if k in (2, 3) else g.cpu().numpy()
        assert rel_err(gn, w) <= TOL["f32"], k
    assert tpc.tp_get_device_error() == 0
