"""Receiver-range sharding (clebsch_gordan_tensor_node_b200/shard.py) on CPU:
the range split and the masked row pointer, and the whole exchange on two gloo
ranks (127.0.0.1) with the oracle standing in for the local kernels. The
sharded forward and backward must reproduce the unsharded oracle: output rows
and grad_x rows of every rank's range, grad_Y and grad_phi of its edges, and
grad_A summed over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from clebsch_gordan_tensor_node_b200.shard import masked_rowptr, receiver_ranges


def test_receiver_ranges_balance_edges():
    rp = np.array([0, 5, 5, 9, 20, 22, 30, 31, 40], np.int64)
    for world in (1, 2, 3, 4, 8):
        r = receiver_ranges(torch.from_numpy(rp), world)
        assert r[0][0] == 0 and r[-1][1] == 8 and len(r) == world
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
        assert all(a[0] <= a[1] for a in r)
    assert receiver_ranges(torch.from_numpy(rp), 2) == [(0, 4), (4, 8)]


def test_masked_rowptr_keeps_only_the_range():
    rp = torch.tensor([0, 5, 5, 9, 20, 22], dtype=torch.int32)
    m = masked_rowptr(rp, 2, 4)
    assert m.tolist() == [0, 0, 0, 4, 15, 15]
    assert m.dtype == rp.dtype


class _OracleOps:
    """The oracle in the place of the library's kernels (CPU tensors, CSR order)."""

    def __init__(self, pr):
        from oracle import conv
        self.conv, self.pr = conv, pr

    @staticmethod
    def _coo(rowptr, senders):
        rp = rowptr.numpy().astype(np.int64)
        dst = np.repeat(np.arange(len(rp) - 1), np.diff(rp))
        return senders.numpy().astype(np.int64), dst

    def forward(self, plan, x, Y, phi, A, rowptr, senders):
        src, dst = self._coo(rowptr, senders)
        return torch.from_numpy(self.conv.forward(self.pr, x.numpy(), Y.numpy(), phi.numpy(), A.numpy(), src, dst,
                                                  len(rowptr) - 1))

    def backward(self, plan, x, Y, phi, A, rowptr, senders, view, gout):
        src, dst = self._coo(rowptr, senders)
        out = self.conv.backward(self.pr, x.numpy(), Y.numpy(), phi.numpy(), A.numpy(), src, dst, gout.numpy(),
                                 len(rowptr) - 1)
        return tuple(torch.from_numpy(o) for o in out)

    def source_view(self, rowptr, senders, n_nodes):
        return None


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from gpu_util import problem, workload
    from oracle import csr
    cid = 1
    wl = workload(cid)
    pr = problem(cid)
    rp, snd, perm = csr.build(wl.n_nodes, wl.src, wl.dst)
    return wl, pr, rp, snd, perm


def _rank(rank, world, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from clebsch_gordan_tensor_node_b200.shard import ReceiverShard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl, pr, rp, snd, perm = _case()
        rowptr, senders = torch.from_numpy(rp.astype(np.int32)), torch.from_numpy(snd.astype(np.int32))
        sh = ReceiverShard(pr, rowptr, senders, rank, world, ops=_OracleOps(pr))
        Yc, pc = wl.Y[perm], wl.phi[perm]
        sl = slice(sh.e0, sh.e1)
        own = slice(sh.r0, sh.r1)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        out = sh.forward(t(wl.x[own]), t(Yc[sl]), t(pc[sl]), t(wl.A))
        gx, gY, gphi, gA = sh.backward(t(wl.x[own]), t(Yc[sl]), t(pc[sl]), t(wl.A), t(wl.grad_out[own]))
        q.put((rank, sh.r0, sh.r1, sh.e0, sh.e1, out.numpy(), gx.numpy(), gY.numpy(), gphi.numpy(), gA.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_sharded_exchange_on_two_gloo_ranks():
    from oracle import conv
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl, pr, rp, snd, perm = _case()
    want = conv.forward(pr, wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.n_nodes)
    wx, wY, wphi, wA = conv.backward(pr, wl.x, wl.Y, wl.phi, wl.A, wl.src, wl.dst, wl.grad_out, wl.n_nodes)
    wY, wphi = wY[perm], wphi[perm]                      # CSR edge order
    assert res[0][1] == 0 and res[-1][2] == wl.n_nodes and res[0][2] == res[1][1]
    for _, r0, r1, e0, e1, out, gx, gY, gphi, gA in res:
        assert np.allclose(out, want[r0:r1], rtol=0, atol=1e-12)
        assert np.allclose(gx, wx[r0:r1], rtol=0, atol=1e-12)
        assert np.allclose(gY, wY[e0:e1], rtol=0, atol=1e-12)
        assert np.allclose(gphi, wphi[e0:e1], rtol=0, atol=1e-12)
        assert np.allclose(gA, wA, rtol=0, atol=1e-12)
