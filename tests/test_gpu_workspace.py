"""Measured tensor-product workspace against the edge count.

The streamed schedule keeps no edge-sized intermediate (Sobek §3.4, Table 2:
W, edge messages and W_bar are not required as complete tensors), and its
bounded receiver state lives under a fixed scratch budget (Sobek App. B.2). So
at a fixed node count the device memory one forward + backward takes beyond its
inputs and outputs must be the same whatever the number of edges.

Measured here at E/4, E/2 and E (a seeded subset of the edges, same nodes) on
the large channelwise and the fully connected workloads at reduced node counts:
  * the peak of the PyTorch allocator during the calls, above what was allocated
    before them (inputs and outputs are allocated beforehand; the binding
    allocates the workspace of tp_conv_workspace_size), is identical for the
    three edge counts and equals the larger of the two workspaces;
  * device memory taken outside the allocator: the drop in free device memory
    over the calls equals the growth of the allocator's reservation, i.e. the
    library itself allocates nothing.
"""
import pytest
import torch

import clebsch_gordan_tensor_node_b200 as tpc
from gpu_util import GpuRun, plan_for, workload

pytestmark = pytest.mark.gpu


def _step(run, out, grads):
    tpc.tp_conv_forward(run.plan, run.x, run.Y, run.phi, run.A, run.rowptr, run.senders, out=out)
    tpc.tp_conv_backward(run.plan, run.x, run.Y, run.phi, run.A, run.rowptr, run.senders, run.colptr,
                         run.srcedge, run.srcrecv, run.gout, out=grads)


def _measure(run):
    out = torch.empty(run.x.shape[0], run.plan.c_out, dtype=run.x.dtype, device=run.x.device)
    grads = (torch.empty_like(run.x), torch.empty_like(run.Y), torch.empty_like(run.phi),
             torch.empty_like(run.A))
    _step(run, out, grads)                 # loads every kernel of the path once
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    res0 = torch.cuda.memory_reserved()
    _step(run, out, grads)
    torch.cuda.synchronize()
    peak = torch.cuda.max_memory_allocated() - base
    free1, _ = torch.cuda.mem_get_info()
    outside = (free0 - free1) - (torch.cuda.memory_reserved() - res0)
    assert tpc.tp_get_device_error() == 0
    return peak, outside


@pytest.mark.parametrize("cid,n", [(4, 20000), (5, 2000)])
def test_workspace_independent_of_edge_count(cid, n):
    plan = plan_for(cid)
    ws = max(plan.workspace_size(n, 0), plan.workspace_size(n, 1))
    peaks = []
    n_edges = []
    for keep in (0.25, 0.5, None):
        run = GpuRun(plan, workload(cid, n_nodes=n, edge_keep=keep))
        n_edges.append(run.senders.numel())
        peak, outside = _measure(run)
        assert outside == 0, f"{outside} bytes of device memory taken outside the allocator"
        peaks.append(peak)
        del run
        torch.cuda.empty_cache()
    assert n_edges[0] < n_edges[1] < n_edges[2]
    assert peaks[0] == peaks[1] == peaks[2], (n_edges, peaks)
    assert ws <= peaks[0] <= ws + (2 << 20), (ws, peaks[0])
