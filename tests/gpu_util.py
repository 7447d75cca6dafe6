"""Helpers of the GPU parity tests: run the library's path on a workload and
compare with the oracle. Imported only by tests."""
from __future__ import annotations

import numpy as np
import torch

import clebsch_gordan_tensor_node_b200 as tpc
from inputs import CONFIGS, make_workload
from oracle.conv import Problem

TOL = {"f32": 1e-4, "f64": 1e-10}


def rel_err(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    scale = np.abs(want).max() if want.size else 0.0
    if scale == 0.0:
        return float(np.abs(got).max()) if got.size else 0.0
    return float(np.abs(got - want).max() / scale)


def problem(cid: int) -> Problem:
    c = CONFIGS[cid]
    return Problem(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.irreps_sh)


def plan_for(cid: int) -> tpc.Plan:
    c = CONFIGS[cid]
    return tpc.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.dtype, irreps_sh=c.irreps_sh)


def workload(cid: int, n_nodes=None, edge_keep=None):
    pr = problem(cid)
    return make_workload(cid, pr.n_w, n_nodes=n_nodes, edge_keep=edge_keep, c_out=pr.c_out)


class GpuRun:
    """Device copies of a workload, its CSR views, and the library's results."""

    def __init__(self, plan: tpc.Plan, wl, dev="cuda"):
        self.plan, self.wl = plan, wl
        N = wl.n_nodes
        self.src = torch.from_numpy(wl.src.astype(np.int32)).to(dev)
        self.dst = torch.from_numpy(wl.dst.astype(np.int32)).to(dev)
        self.rowptr, self.senders, self.perm = tpc.tp_csr_build(self.src, self.dst, N)
        self.colptr, self.srcedge, self.srcrecv = tpc.tp_csr_transpose(self.rowptr, self.senders, N)
        p = self.perm.long()
        self.x = torch.from_numpy(wl.x).to(dev)
        self.Y = torch.from_numpy(wl.Y).to(dev)[p].contiguous()      # CSR edge order
        self.phi = torch.from_numpy(wl.phi).to(dev)[p].contiguous()
        self.A = torch.from_numpy(wl.A).to(dev)
        self.gout = torch.from_numpy(wl.grad_out).to(dev)

    def forward(self, A=None):
        return tpc.tp_conv_forward(self.plan, self.x, self.Y, self.phi, self.A if A is None else A,
                                   self.rowptr, self.senders)

    def backward(self):
        return tpc.tp_conv_backward(self.plan, self.x, self.Y, self.phi, self.A, self.rowptr,
                                    self.senders, self.colptr, self.srcedge, self.srcrecv, self.gout)

    def to_coo(self, t):
        """Rows of an edge-major CSR-order tensor back in COO order, as numpy."""
        out = torch.empty_like(t)
        out[self.perm.long()] = t
        return out.cpu().numpy()
