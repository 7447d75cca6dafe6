"""GPU parity of the second-order program (tp_conv_double_backward) against the
oracle (Sobek §3.3; LunaTP Appendix F, Algorithm 3), through the C ABI.

Directions (dx, dY, dphi, dA) are seeded N(0, 1) draws of the inputs' shapes and
dtype. Bar: per output tensor max|gpu - oracle| / max|oracle| <= 1e-4 (fp32),
1e-10 (fp64); run to run bitwise identical. At full size of the large graph the
receiver-, edge- and source-owned outputs are checked on sampled rows against
the oracle restricted to the edges that feed them, and dgrad_A through the
symmetry of the Hessian: <V, (H v)_A> = sum over x, Y, phi of <(H u)_k, v_k>
for u = (0, 0, 0, V), since the operator is linear in A.
"""
import numpy as np
import pytest
import torch

import clebsch_gordan_tensor_node_b200 as tpc
from gpu_util import TOL, GpuRun, plan_for, problem, rel_err, workload
from inputs import CONFIGS
from oracle import conv as oconv

pytestmark = pytest.mark.gpu


def _directions(wl, seed):
    rng = np.random.default_rng(seed)
    dt = wl.np_dtype
    return [rng.normal(size=a.shape).astype(dt) for a in (wl.x, wl.Y, wl.phi, wl.A)]


def _dbl(run, d):
    p = run.perm.long()
    dev = run.x.device
    dx = torch.from_numpy(d[0]).to(dev)
    dY = torch.from_numpy(d[1]).to(dev)[p].contiguous()
    dphi = torch.from_numpy(d[2]).to(dev)[p].contiguous()
    dA = torch.from_numpy(d[3]).to(dev)
    return tpc.tp_conv_double_backward(run.plan, run.x, run.Y, run.phi, run.A, run.rowptr, run.senders,
                                       run.colptr, run.srcedge, run.srcrecv, run.gout, dx, dY, dphi, dA)


CASES = [(1, None), (3, None), (4, 1500), (2, 384)]


@pytest.mark.parametrize("cid,n", CASES)
def test_double_backward_parity(cid, n):
    c = CONFIGS[cid]
    wl = workload(cid, n_nodes=n)
    run = GpuRun(plan_for(cid), wl)
    d = _directions(wl, 7 + cid)
    got = _dbl(run, d)
    want = oconv.double_backward(problem(cid), wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.grad_out, *d,
                                 wl.n_nodes)
    names = ("d_out", "dgrad_x", "dgrad_Y", "dgrad_phi", "dgrad_A")
    for k, (g, w) in enumerate(zip(got, want)):
        gn = run.to_coo(g) if k in (2, 3) else g.cpu().numpy()
        assert rel_err(gn, w) <= TOL[c.dtype], names[k]
    assert tpc.tp_get_device_error() == 0
    again = _dbl(run, d)
    for a, b in zip(got, again):
        assert torch.equal(a, b)


def test_double_backward_uvw_across_state_chunks():
    """Fully connected workload at 200 nodes under a state budget of 60 nodes,
    so the receiver program (directional state, mixings, three edge passes) and
    the source states run over four chunks each."""
    from test_gpu_parity import _state_row_bytes
    cid = 5
    wl = workload(cid, n_nodes=200)
    plan = plan_for(cid)
    s_row, sa_row = _state_row_bytes(plan)
    plan.set_state_budget(60 * max(s_row, sa_row))
    run = GpuRun(plan, wl)
    d = _directions(wl, 12)
    got = _dbl(run, d)
    want = oconv.double_backward(problem(cid), wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.grad_out, *d,
                                 wl.n_nodes)
    names = ("d_out", "dgrad_x", "dgrad_Y", "dgrad_phi", "dgrad_A")
    for k, (g, w) in enumerate(zip(got, want)):
        gn = run.to_coo(g) if k in (2, 3) else g.cpu().numpy()
        assert rel_err(gn, w) <= TOL["f32"], names[k]
    assert tpc.tp_get_device_error() == 0
    again = _dbl(run, d)
    for a, b in zip(got, again):
        assert torch.equal(a, b)


def test_double_backward_full_size_sampled():
    cid = 4
    wl = workload(cid)
    run = GpuRun(plan_for(cid), wl)
    pr = problem(cid)
    d = _directions(wl, 21)
    mdot, gx, gY, gphi, gA = _dbl(run, d)
    rng = np.random.default_rng(5)
    recv = rng.choice(wl.n_nodes, 24, replace=False)
    sel = np.isin(wl.dst, recv)
    sub = lambda m: (wl.x, wl.Y[m], wl.phi[m], wl.A, wl.src[m], wl.dst[m], wl.grad_out,
                     d[0], d[1][m], d[2][m], d[3], wl.n_nodes)
    w = oconv.double_backward(pr, *sub(sel))
    assert rel_err(mdot.cpu().numpy()[recv], w[0][recv]) <= TOL["f32"]
    assert rel_err(run.to_coo(gY)[sel], w[2]) <= TOL["f32"]
    assert rel_err(run.to_coo(gphi)[sel], w[3]) <= TOL["f32"]
    srcs = rng.choice(wl.n_nodes, 24, replace=False)
    ssel = np.isin(wl.src, srcs)
    w = oconv.double_backward(pr, *sub(ssel))
    assert rel_err(gx.cpu().numpy()[srcs], w[1][srcs]) <= TOL["f32"]
    # dgrad_A through the symmetry of the Hessian
    V = np.random.default_rng(9).normal(size=wl.A.shape).astype(np.float32)
    z = [np.zeros_like(wl.x), np.zeros_like(wl.Y), np.zeros_like(wl.phi), V]
    _, hx, hY, hphi, hA = _dbl(run, z)
    assert float(hA.abs().max()) == 0.0              # linear in A: no A-A block
    dev = run.x.device
    p = run.perm.long()
    terms = [float((hx.double() * torch.from_numpy(d[0]).to(dev).double()).sum()),
             float((hY.double() * torch.from_numpy(d[1]).to(dev)[p].double()).sum()),
             float((hphi.double() * torch.from_numpy(d[2]).to(dev)[p].double()).sum())]
    lhs = float((gA.double() * torch.from_numpy(V).to(dev).double()).sum())
    assert abs(lhs - sum(terms)) <= 1e-4 * max(abs(lhs), max(abs(t) for t in terms))
    assert tpc.tp_get_device_error() == 0


def test_double_backward_without_edges():
    """Nodes but no edges: every output is zero (and is written)."""
    cid = 1
    plan = plan_for(cid)
    c = CONFIGS[cid]
    N = 5
    dev = "cuda"
    dt = plan.torch_dtype
    x = torch.randn(N, plan.c_in, dtype=dt, device=dev)
    A = torch.randn(plan.n_radial, plan.n_w, dtype=dt, device=dev)
    g = torch.randn(N, plan.c_out, dtype=dt, device=dev)
    rowptr = torch.zeros(N + 1, dtype=torch.int32, device=dev)
    e = torch.zeros(0, dtype=torch.int32, device=dev)
    Y = torch.zeros(0, plan.dim_y, dtype=dt, device=dev)
    phi = torch.zeros(0, plan.n_radial, dtype=dt, device=dev)
    out = (torch.full((N, plan.c_out), float("nan"), dtype=dt, device=dev),
           torch.full((N, plan.c_in), float("nan"), dtype=dt, device=dev),
           torch.zeros(0, plan.dim_y, dtype=dt, device=dev), torch.zeros(0, plan.n_radial, dtype=dt, device=dev),
           torch.full((plan.n_radial, plan.n_w), float("nan"), dtype=dt, device=dev))
    res = tpc.tp_conv_double_backward(plan, x, Y, phi, A, rowptr, e, rowptr, e, e, g, x, Y, phi, A, out=out)
    torch.cuda.synchronize()
    for t in (res[0], res[1], res[4]):
        assert torch.count_nonzero(t).item() == 0 and torch.isfinite(t).all()
    assert tpc.tp_get_device_error() == 0
