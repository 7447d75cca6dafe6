"""Receiver CSR and its source transpose (oracle; test infrastructure).

LunaTP §4.1 stores the adjacency by destination node, with the edges of node i in
[rowptr[i], rowptr[i+1]); LunaTP §4.4 and Sobek §4.3 add a source-ordered view so
that the node-feature gradient has one fixed reduction order per source row.
Sobek §4.5 asks for stable views; the reading taken is: within a receiver, edges
keep their input (COO) order; within a source, CSR positions keep ascending order.
"""
from __future__ import annotations

import numpy as np


def build(n_nodes: int, src: np.ndarray, dst: np.ndarray):
    """COO (src -> dst) to receiver CSR: rowptr[N+1], senders[E], perm[E].

    perm[k] is the COO index of the edge stored at CSR position k.
    """
    src = np.asarray(src, dtype=np.int64)
    dst = np.asarray(dst, dtype=np.int64)
    perm = np.argsort(dst, kind="stable")
    counts = np.bincount(dst, minlength=n_nodes)
    rowptr = np.zeros(n_nodes + 1, dtype=np.int64)
    np.cumsum(counts, out=rowptr[1:])
    return rowptr, src[perm], perm


def transpose(n_nodes: int, rowptr: np.ndarray, senders: np.ndarray):
    """Source view of a receiver CSR: colptr[N+1], srcedge[E], srcrecv[E].

    srcedge[k] is the CSR position of the k-th edge in source order, srcrecv[k]
    the receiver of that edge.
    """
    senders = np.asarray(senders, dtype=np.int64)
    srcedge = np.argsort(senders, kind="stable")
    counts = np.bincount(senders, minlength=n_nodes)
    colptr = np.zeros(n_nodes + 1, dtype=np.int64)
    np.cumsum(counts, out=colptr[1:])
    recv = np.repeat(np.arange(n_nodes), np.diff(rowptr))
    return colptr, srcedge, recv[srcedge]
