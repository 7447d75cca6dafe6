"""The channelwise forward in the receiver-factorised order (Sobek §4.2, Eqs.
32-35 applied to uvu: the receiver state S_i = sum_e phi_e (outer) C(x_j, Y_e),
mixed once per receiver) against the oracle and against the streamed order
(Sobek §3.1). Both are the same operator up to the order of the additions."""
import pytest
import torch

import clebsch_gordan_tensor_node_b200 as tpc
from gpu_util import TOL, GpuRun, plan_for, problem, rel_err, workload
from inputs import CONFIGS
from oracle import conv as oconv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cid,n", [(1, None), (3, None), (2, 384), (4, 1500)])
def test_receiver_state_forward_parity(cid, n):
    c = CONFIGS[cid]
    wl = workload(cid, n_nodes=n)
    plan = plan_for(cid)
    run = GpuRun(plan, wl)
    streamed = run.forward().clone()
    plan.set_schedule("receiver_state")
    state = run.forward()
    want = oconv.forward(problem(cid), wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.n_nodes)
    assert rel_err(state.cpu().numpy(), want) <= TOL[c.dtype]
    assert rel_err(state.cpu().numpy(), streamed.cpu().numpy()) <= TOL[c.dtype]
    assert torch.equal(state, run.forward())          # run to run bitwise
    assert tpc.tp_get_device_error() == 0
