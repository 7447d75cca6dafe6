"""Fully connected plans whose blocks are wider than 64 channels: the tcgen05
mixing GEMM holds a 128 x N accumulator with N up to 256 and a shallower
shared-memory ring. Sobek's profiles (in = out irreps, alternating parity, K =
16, §5.1) on one copy of its 128-node, degree-32 graph, forward and first
backward against the oracle at the fp32 bar."""
import types

import numpy as np
import pytest

import clebsch_gordan_tensor_node_b200 as tpc
from gpu_util import TOL, GpuRun, rel_err
from inputs import sobek_count_graph, sobek_workload
from oracle import conv as oconv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("irreps,L", [("128x0e+64x1o", 1), ("256x0e+32x1o", 1), ("128x0e+128x1o", 1)])
def test_wide_block_uvw_parity(irreps, L):
    plan = tpc.Plan(irreps, L, irreps, 16, "uvw", "f32")
    pr = oconv.Problem(irreps, L, irreps, 16, "uvw")
    w = sobek_workload(sobek_count_graph(1), irreps, L, 16, plan.n_w, plan.c_out)
    wl = types.SimpleNamespace(n_nodes=w["n_nodes"], **{k: w[k] for k in ("src", "dst", "x", "Y", "phi", "A",
                                                                          "grad_out")})
    run = GpuRun(plan, wl)
    out = run.forward()
    want = oconv.forward(pr, wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.n_nodes)
    assert rel_err(out.cpu().numpy(), want) <= TOL["f32"]
    gx, gY, gphi, gA = run.backward()
    ox, oY, ophi, oA = oconv.backward(pr, wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.grad_out, wl.n_nodes)
    assert rel_err(gx.cpu().numpy(), ox) <= TOL["f32"]
    assert rel_err(run.to_coo(gY), oY) <= TOL["f32"]
    assert rel_err(run.to_coo(gphi), ophi) <= TOL["f32"]
    assert rel_err(gA.cpu().numpy(), oA) <= TOL["f32"]
    assert tpc.tp_get_device_error() == 0
