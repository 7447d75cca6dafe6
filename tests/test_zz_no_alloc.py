"""The workspace-free backward (tp_conv_backward_noalloc) against tp_conv_backward.

Callers that cannot allocate device memory where they run the backward (engine
plugins, code inside an open stream capture, fixed memory reservations) use the
entry point that keeps its grad_A partial sums in the library's static device
scratch. It must give what tp_conv_backward gives, within the parity tolerance
(only the order of the grad_A additions may differ), on consecutive calls, since
each call reuses the scratch that the previous one left behind.

Called through the C ABI (ctypes); this file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from clebsch_gordan_tensor_node_b200 import _lib
from gpu_util import TOL, GpuRun, plan_for, rel_err, workload
from inputs import CONFIGS

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr() if t.numel() else 0)


@pytest.mark.parametrize("cid,n", [(4, 1500), (1, None), (3, None)])
def test_noalloc_backward_matches_backward(cid, n):
    c = CONFIGS[cid]
    run = GpuRun(plan_for(cid), workload(cid, n_nodes=n))
    want = [t.clone() for t in run.backward()]
    torch.cuda.synchronize()
    N, E = run.x.shape[0], run.senders.numel()
    L = _lib.lib()
    for call in range(2):
        got = [torch.full_like(t, float("nan")) for t in want]
        st = L.tp_conv_backward_noalloc(
            run.plan.handle, _p(run.x), _p(run.Y), _p(run.phi), _p(run.A), _p(run.rowptr),
            _p(run.senders), _p(run.colptr), _p(run.srcedge), _p(run.srcrecv), _p(run.gout), N, E,
            _p(got[0]), _p(got[1]), _p(got[2]), _p(got[3]),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, L.tp_last_error_message().decode()
        assert L.tp_get_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
        for g, w, name in zip(got, want, ("grad_x", "grad_Y", "grad_phi", "grad_A")):
            assert torch.isfinite(g).all(), (call, name)
            assert rel_err(g.cpu().numpy(), w.cpu().numpy()) <= TOL[c.dtype], (call, name)


def test_noalloc_rejects_uvw_plans():
    from clebsch_gordan_tensor_node_b200 import Plan
    plan = Plan("2x0e+2x1o", 1, "2x0e+2x1o", 4, "uvw", "f32")
    L = _lib.lib()
    z = ctypes.c_void_p(0)
    st = L.tp_conv_backward_noalloc(plan.handle, z, z, z, z, z, z, z, z, z, z, 1, 0, z, z, z, z, z)
    assert st == -2


def test_noalloc_empty_graph_zeroes_grad_A():
    """With no nodes there is nothing to accumulate: grad_A must still come back
    zero (overwritten), whatever the previous calls left in the scratch."""
    cid = 4
    run = GpuRun(plan_for(cid), workload(cid, n_nodes=1500))
    run.backward()                          # leave the scratch and outputs in use
    L = _lib.lib()
    gA = torch.full_like(run.A, float("nan"))
    gx = torch.empty_like(run.x)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    z = ctypes.c_void_p(0)
    st = L.tp_conv_backward_noalloc(run.plan.handle, _p(run.x), z, z, _p(run.A), _p(run.rowptr), z,
                                    _p(run.colptr), z, z, _p(run.gout), 0, 0, _p(gx), z, z, _p(gA), s)
    assert st == 0, L.tp_last_error_message().decode()
    torch.cuda.synchronize()
    assert torch.count_nonzero(gA).item() == 0 and torch.isfinite(gA).all()
