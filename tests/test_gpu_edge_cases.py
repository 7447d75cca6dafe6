"""GPU edge cases against the oracle: empty graphs, isolated and hub nodes
(rows longer than the shared-memory sort), odd multiplicities, partial channel
tiles, padded radial widths, and bad indices reported through the device error
word instead of a trap."""
import numpy as np
import pytest
import torch

import clebsch_gordan_tensor_node_b200 as tpc
from gpu_util import TOL, rel_err
from inputs.workloads import spherical_harmonics
from oracle import conv as oconv
from oracle import csr as ocsr

pytestmark = pytest.mark.gpu


class _WL:
    def __init__(self, pr, N, src, dst, dtype, seed):
        rng = np.random.default_rng(seed)
        dt = np.float32 if dtype == "f32" else np.float64
        self.n_nodes, self.src, self.dst = N, np.asarray(src, np.int64), np.asarray(dst, np.int64)
        E = len(src)
        vec = rng.normal(size=(E, 3))
        self.Y = spherical_harmonics(pr.sh_lmax, vec).astype(dt) if E else np.zeros((0, pr.dim_y), dt)
        self.phi = rng.normal(size=(E, pr.K)).astype(dt)
        self.x = rng.normal(size=(N, pr.c_in)).astype(dt)
        self.A = rng.normal(size=(pr.K, pr.n_w)).astype(dt)
        self.grad_out = rng.normal(size=(N, pr.c_out)).astype(dt)


def _run_and_compare(spec, dtype, N, src, dst, seed=0):
    from gpu_util import GpuRun
    pr = oconv.Problem(*spec)
    wl = _WL(pr, N, src, dst, dtype, seed)
    plan = tpc.Plan(*spec, dtype)
    run = GpuRun(plan, wl)
    rp, snd, perm = ocsr.build(N, wl.src, wl.dst)
    assert np.array_equal(run.rowptr.cpu().numpy(), rp)
    assert np.array_equal(run.perm.cpu().numpy(), perm)
    cp, se, sr = ocsr.transpose(N, rp, snd)
    assert np.array_equal(run.srcedge.cpu().numpy(), se)
    assert np.array_equal(run.srcrecv.cpu().numpy(), sr)
    out = run.forward()
    want = oconv.forward(pr, wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, N)
    assert rel_err(out.cpu().numpy(), want) <= TOL[dtype]
    gx, gY, gphi, gA = run.backward()
    ox, oY, ophi, oA = oconv.backward(pr, wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.grad_out, N)
    assert rel_err(gx.cpu().numpy(), ox) <= TOL[dtype]
    if len(src):
        assert rel_err(run.to_coo(gY), oY) <= TOL[dtype]
        assert rel_err(run.to_coo(gphi), ophi) <= TOL[dtype]
    assert rel_err(gA.cpu().numpy(), oA) <= TOL[dtype]
    assert tpc.tp_get_device_error() == 0
    return out


SPEC = ("8x0e+8x1o+8x2e", 2, "8x0e+8x1o+8x1e+8x2e+8x2o", 8, "uvu")


def test_empty_graph():
    out = _run_and_compare(SPEC, "f64", 5, [], [])
    assert not out.any()
    out = _run_and_compare(("2x0e+3x1o", 2, "3x0e+2x1o+2x2e", 3, "uvw"), "f32", 5, [], [])
    assert not out.any()


def test_isolated_and_hub_nodes():
    rng = np.random.default_rng(4)
    N = 40
    # node 0 receives 700 edges, node 1 sends 700 edges, nodes 30..39 are isolated
    src = np.concatenate([rng.integers(2, 30, 700), np.full(700, 1), rng.integers(2, 30, 300)])
    dst = np.concatenate([np.zeros(700, int), rng.integers(2, 30, 700), rng.integers(2, 30, 300)])
    keep = src != dst
    _run_and_compare(SPEC, "f64", N, src[keep], dst[keep], seed=1)
    _run_and_compare(("2x0e+3x1o", 2, "3x0e+2x1o+2x2e", 3, "uvw"), "f64", N, src[keep], dst[keep], seed=1)


@pytest.mark.parametrize("spec,dtype", [
    (("3x0e+3x1o", 2, "3x0e+3x1o+3x1e+3x2e", 5, "uvu"), "f32"),        # odd mul, K padded
    (("80x0e+80x1o", 1, "80x0e+80x1o+80x1e", 16, "uvu"), "f64"),       # 3 channel tiles
    (("96x0e+96x1o+96x2e", 2, "96x0e+96x1o+96x2e", 16, "uvu"), "f32"), # K 16, CPL 2, 2 tiles
    (("4x0e+4x1o+4x2e+4x3o+4x4e", 4, "4x0e+4x1o+4x2e+4x3o+4x4e", 3, "uvu"), "f64"),  # l = 4
    (("2x0e+3x1o", 2, "3x0e+2x1o+2x2e", 3, "uvw"), "f64"),               # uvw, unequal muls
    (("40x0e+8x1o+5x2e", 2, "7x0e+40x1o+3x1e+9x2e", 16, "uvw"), "f32"),  # uvw, mul > 32
    (("6x0e+6x1o+6x2e+6x3o+6x4e", 4, "6x0e+6x1o+6x2e+6x3o+6x4e+6x4o", 11, "uvw"), "f64"),
])
def test_shapes(spec, dtype):
    rng = np.random.default_rng(8)
    N = 23
    src, dst = rng.integers(0, N, 260), rng.integers(0, N, 260)
    keep = src != dst
    _run_and_compare(spec, dtype, N, src[keep], dst[keep], seed=2)


def test_bad_sender_sets_device_error():
    plan = tpc.Plan(*SPEC, "f64")
    N = 4
    rowptr = torch.tensor([0, 1, 2, 2, 3], dtype=torch.int32, device="cuda")
    senders = torch.tensor([1, 7, 0], dtype=torch.int32, device="cuda")   # 7 is out of range
    x = torch.randn(N, plan.c_in, dtype=torch.float64, device="cuda")
    Y = torch.randn(3, plan.dim_y, dtype=torch.float64, device="cuda")
    phi = torch.randn(3, plan.n_radial, dtype=torch.float64, device="cuda")
    A = torch.randn(plan.n_radial, plan.n_w, dtype=torch.float64, device="cuda")
    tpc.tp_conv_forward(plan, x, Y, phi, A, rowptr, senders)
    assert tpc.tp_get_device_error() == -5
    assert tpc.tp_get_device_error() == 0          # cleared
    bad_rowptr = torch.tensor([0, 2, 1, 2, 3], dtype=torch.int32, device="cuda")
    tpc.tp_conv_forward(plan, x, Y, phi, A, bad_rowptr, torch.tensor([1, 2, 0], dtype=torch.int32,
                                                                     device="cuda"))
    assert tpc.tp_get_device_error() == -6
    # the context is still usable
    out = tpc.tp_conv_forward(plan, x, Y, phi, A, rowptr, torch.tensor([1, 2, 0], dtype=torch.int32,
                                                                        device="cuda"))
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()


def test_bad_coo_index_sets_device_error():
    src = torch.tensor([0, 1, 9], dtype=torch.int32, device="cuda")
    dst = torch.tensor([1, 2, 0], dtype=torch.int32, device="cuda")
    rowptr, senders, perm = tpc.tp_csr_build(src, dst, 3)
    assert tpc.tp_get_device_error() == -5
    assert rowptr.cpu().tolist() == [0, 0, 1, 2]
    assert perm.cpu().tolist()[2] == -1
