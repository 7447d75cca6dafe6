"""Receiver-range sharding with the library's kernels, two ranks run one after
the other on one GPU (their local steps only; the collectives are the CPU
test's): forward rows, grad_Y and grad_phi of each rank's edges, and the sums
of the partial grad_x and grad_A equal the unsharded call within the parity
bar."""
import pytest
import torch

import clebsch_gordan_tensor_node_b200 as tpc
from clebsch_gordan_tensor_node_b200.shard import ReceiverShard
from gpu_util import TOL, GpuRun, plan_for, rel_err, workload
from inputs import CONFIGS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cid,n,world", [(4, 1500, 2), (4, 1500, 3), (5, 300, 2), (1, None, 2)])
def test_sharded_local_steps_match_unsharded(cid, n, world):
    c = CONFIGS[cid]
    run = GpuRun(plan_for(cid), workload(cid, n_nodes=n))
    out = run.forward()
    gx, gY, gphi, gA = run.backward()
    N = run.x.shape[0]
    sum_gx, sum_gA = torch.zeros_like(gx), torch.zeros_like(gA)
    for rank in range(world):
        sh = ReceiverShard(run.plan, run.rowptr, run.senders, rank, world)
        sl = slice(sh.e0, sh.e1)
        o = sh.local_forward(run.x, run.Y[sl].clone(), run.phi[sl].clone(), run.A)
        assert rel_err(o[sh.r0:sh.r1].cpu().numpy(), out[sh.r0:sh.r1].cpu().numpy()) <= TOL[c.dtype]
        gout = torch.zeros_like(run.gout)
        gout[sh.r0:sh.r1] = run.gout[sh.r0:sh.r1]
        px, pY, pphi, pA = sh.local_backward(run.x, run.Y[sl].clone(), run.phi[sl].clone(), run.A, gout)
        assert rel_err(pY.cpu().numpy(), gY[sl].cpu().numpy()) <= TOL[c.dtype]
        assert rel_err(pphi.cpu().numpy(), gphi[sl].cpu().numpy()) <= TOL[c.dtype]
        sum_gx += px
        sum_gA += pA
    assert rel_err(sum_gx.cpu().numpy(), gx.cpu().numpy()) <= TOL[c.dtype]
    assert rel_err(sum_gA.cpu().numpy(), gA.cpu().numpy()) <= TOL[c.dtype]
    assert tpc.tp_get_device_error() == 0
