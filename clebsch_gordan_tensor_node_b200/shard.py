"""Receiver-range sharding of one graph over several GPUs (one process each).

The convolution's output rows are owned by receivers (Sobek §4.1: work is
organised around destination nodes), so contiguous receiver ranges split the
forward with no exchange beyond the sender features: each rank holds the full
receiver CSR, the edge features of its own receivers' edges, and the node rows
of its range. Per call:

* forward: all-gather x; run the library's forward over a row pointer in which
  the receivers outside the rank's range have no edges; keep the rank's rows;
* backward: the edge pass needs only local edges; the source pass, over the
  source view of the local edges, gives each rank a partial x_bar for every
  source, which a reduce-scatter sums onto the owners (the exchange step of the
  source-owned reduction, Sobek §4.3); grad_A is summed by an all-reduce.

Ranges are balanced by edge count. The collectives go through
torch.distributed (NCCL on GPUs, gloo in the CPU tests); the arithmetic is the
library's kernels (`ops` defaults to this package's C-ABI binding).
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple


def receiver_ranges(rowptr, world: int) -> List[Tuple[int, int]]:
    """Contiguous receiver ranges [r0, r1), one per rank, with about equal edge
    counts (cuts at the receivers where the running edge count crosses k E / W)."""
    import numpy as np
    rp = np.asarray(rowptr.cpu() if hasattr(rowptr, "cpu") else rowptr, dtype=np.int64)
    n, e = len(rp) - 1, int(rp[-1])
    cuts = [0]
    for k in range(1, world):
        target = (k * e) // world
        c = int(np.searchsorted(rp, target, side="left"))
        cuts.append(min(max(c, cuts[-1]), n))
    cuts.append(n)
    return [(cuts[k], cuts[k + 1]) for k in range(world)]


def masked_rowptr(rowptr, r0: int, r1: int):
    """Row pointer over all receivers in which only [r0, r1) keep their edges,
    re-based so that the rank's first edge is 0."""
    e0, e1 = int(rowptr[r0]), int(rowptr[r1])
    return (rowptr.clamp(min=e0, max=e1) - e0).to(rowptr.dtype)


class _BindingOps:
    """The library's kernels through the C-ABI binding (CUDA tensors)."""

    def __init__(self):
        from . import tp_conv_backward, tp_conv_forward, tp_csr_transpose
        self.fwd, self.bwd, self.transpose = tp_conv_forward, tp_conv_backward, tp_csr_transpose

    def forward(self, plan, x, Y, phi, A, rowptr, senders):
        return self.fwd(plan, x, Y, phi, A, rowptr, senders)

    def backward(self, plan, x, Y, phi, A, rowptr, senders, view, gout):
        return self.bwd(plan, x, Y, phi, A, rowptr, senders, *view, gout)

    def source_view(self, rowptr, senders, n_nodes):
        return self.transpose(rowptr, senders, n_nodes)


class ReceiverShard:
    """One rank's share of a convolution over a graph split by receiver ranges.

    rowptr, senders: the full receiver CSR (rowptr [N+1], senders [E], global
    node ids), identical on every rank. The rank's edges are the CSR positions
    [rowptr[r0], rowptr[r1]); its edge inputs (Y, phi) are those rows, in
    tensors of their own (the library wants 16-byte aligned buffers, which a
    row slice of the full edge tensors need not be).
    """

    def __init__(self, plan, rowptr, senders, rank: int, world: int, group=None, ops=None,
                 ranges: Optional[Sequence[Tuple[int, int]]] = None):
        self.plan, self.rank, self.world, self.group = plan, rank, world, group
        self.ops = ops if ops is not None else _BindingOps()
        self.n_nodes = rowptr.numel() - 1
        self.ranges = list(ranges) if ranges is not None else receiver_ranges(rowptr, world)
        self.r0, self.r1 = self.ranges[rank]
        self.e0, self.e1 = int(rowptr[self.r0]), int(rowptr[self.r1])
        self.rowptr = masked_rowptr(rowptr, self.r0, self.r1)
        self.senders = senders[self.e0:self.e1].contiguous()
        self.view = self.ops.source_view(self.rowptr, self.senders, self.n_nodes)
        self.rows_max = max(r1 - r0 for r0, r1 in self.ranges)

    # ------------------------------------------------------------------ exchange

    def _all_gather_rows(self, own):
        """[r1 - r0, C] on every rank -> [N, C] (ranges padded to equal length)."""
        import torch
        import torch.distributed as dist
        if self.world == 1:
            return own
        pad = torch.zeros((self.rows_max,) + tuple(own.shape[1:]), dtype=own.dtype, device=own.device)
        pad[: own.shape[0]] = own
        full = torch.empty((self.world * self.rows_max,) + tuple(own.shape[1:]), dtype=own.dtype,
                           device=own.device)
        dist.all_gather_into_tensor(full, pad, group=self.group)
        return torch.cat([full[k * self.rows_max: k * self.rows_max + (r1 - r0)]
                          for k, (r0, r1) in enumerate(self.ranges)])

    def _reduce_scatter_rows(self, part):
        """[N, C] partial sums on every rank -> the sum of the rank's rows."""
        import torch
        import torch.distributed as dist
        if self.world == 1:
            return part
        src = torch.zeros((self.world * self.rows_max,) + tuple(part.shape[1:]), dtype=part.dtype,
                          device=part.device)
        for k, (r0, r1) in enumerate(self.ranges):
            src[k * self.rows_max: k * self.rows_max + (r1 - r0)] = part[r0:r1]
        out = torch.empty((self.rows_max,) + tuple(part.shape[1:]), dtype=part.dtype, device=part.device)
        dist.reduce_scatter_tensor(out, src, group=self.group)
        return out[: self.r1 - self.r0]

    def _all_reduce(self, t):
        import torch.distributed as dist
        if self.world > 1:
            dist.all_reduce(t, group=self.group)
        return t

    # ------------------------------------------------------------------ passes

    def local_forward(self, x_full, Y, phi, A):
        """Output rows of the rank's receivers ([N, C_out]; other rows zero)."""
        return self.ops.forward(self.plan, x_full, Y, phi, A, self.rowptr, self.senders)

    def local_backward(self, x_full, Y, phi, A, gout_full):
        """Partial (x_bar [N, C_in], grad_Y, grad_phi of the rank's edges, grad_A)."""
        return self.ops.backward(self.plan, x_full, Y, phi, A, self.rowptr, self.senders, self.view, gout_full)

    def forward(self, x_own, Y, phi, A):
        """x_own: the rank's node rows [r1 - r0, C_in]; Y, phi: its edges' rows.
        Returns the rank's output rows [r1 - r0, C_out]."""
        out = self.local_forward(self._all_gather_rows(x_own), Y, phi, A)
        return out[self.r0:self.r1]

    def backward(self, x_own, Y, phi, A, gout_own):
        """Returns (grad_x of the rank's rows, grad_Y and grad_phi of its edges,
        grad_A summed over all ranks)."""
        import torch
        x_full = self._all_gather_rows(x_own)
        gout_full = torch.zeros((self.n_nodes, gout_own.shape[1]), dtype=gout_own.dtype, device=gout_own.device)
        gout_full[self.r0:self.r1] = gout_own
        gx, gY, gphi, gA = self.local_backward(x_full, Y, phi, A, gout_full)
        return self._reduce_scatter_rows(gx), gY, gphi, self._all_reduce(gA)
