"""Edge-conditioned Clebsch-Gordan tensor-product convolution on B200 (sm_100a).

Thin binding over libtpconv.so (include/tpconv.h): the functions below carry
the C entry points' names, take PyTorch CUDA tensors for device memory and the
current CUDA stream, and only marshal arguments. Every step of the operator
runs in the library's kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

from ._lib import (TP_F32, TP_F64, TP_UVU, TP_UVU_PATHS, TP_UVW, PathInfo, PlanInfo, TpConvError, check, lib)

__all__ = ["Plan", "tp_conv_plan", "tp_csr_build", "tp_csr_transpose", "tp_conv_forward",
           "tp_conv_backward", "tp_conv_double_backward", "tp_conv_backward_noalloc", "tp_get_device_error",
           "TpConvError"]


def _torch():
    import torch
    return torch


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr() if t is not None and t.numel() > 0 else 0)


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, shape, name):
    torch = _torch()
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


class Plan:
    """One convolution contract (tp_conv_plan). Host-only; owns no device memory."""

    def __init__(self, irreps_in: str, sh_lmax: int, irreps_out: str, n_radial: int,
                 mode: str = "uvu", dtype: str = "f32", irreps_sh: Optional[str] = None):
        self.mode = {"uvu": TP_UVU, "uvw": TP_UVW, "uvu_paths": TP_UVU_PATHS}[mode]
        self.dtype_code = {"f32": TP_F32, "f64": TP_F64}[dtype]
        h = ctypes.c_void_p()
        if irreps_sh is None:
            check(lib().tp_conv_plan(irreps_in.encode(), sh_lmax, irreps_out.encode(), n_radial,
                                     self.mode, self.dtype_code, ctypes.byref(h)), "tp_conv_plan")
        else:
            check(lib().tp_conv_plan_sh(irreps_in.encode(), irreps_sh.encode(), irreps_out.encode(), n_radial,
                                        self.mode, self.dtype_code, ctypes.byref(h)), "tp_conv_plan_sh")
        self._h = h
        info = PlanInfo()
        check(lib().tp_conv_plan_info(h, ctypes.byref(info)), "tp_conv_plan_info")
        self.info = info
        self.c_in, self.c_out, self.dim_y = info.c_in, info.c_out, info.dim_y
        self.n_radial, self.n_paths, self.n_w = info.n_radial, info.n_paths, info.n_w
        self.state_budget = 1 << 30

    @property
    def handle(self):
        return self._h

    @property
    def torch_dtype(self):
        torch = _torch()
        return torch.float32 if self.dtype_code == TP_F32 else torch.float64

    def path(self, index: int) -> PathInfo:
        p = PathInfo()
        check(lib().tp_conv_plan_path(self._h, index, ctypes.byref(p)), "tp_conv_plan_path")
        return p

    def paths(self):
        return [self.path(k) for k in range(self.n_paths)]

    def cg(self, index: int):
        n = check(lib().tp_conv_plan_cg(self._h, index, None, None, None, None, 0), "tp_conv_plan_cg")
        m1, m2, m3 = (ctypes.c_int32 * n)(), (ctypes.c_int32 * n)(), (ctypes.c_int32 * n)()
        c = (ctypes.c_double * n)()
        check(lib().tp_conv_plan_cg(self._h, index, m1, m2, m3, c, n), "tp_conv_plan_cg")
        return [(m1[k], m2[k], m3[k], c[k]) for k in range(n)]

    def set_state_budget(self, nbytes: int) -> None:
        """Bytes of one uvw receiver-state chunk (tp_conv_plan_set_state_budget)."""
        check(lib().tp_conv_plan_set_state_budget(self._h, nbytes), "tp_conv_plan_set_state_budget")
        self.state_budget = nbytes

    def set_schedule(self, schedule: str) -> None:
        """Channelwise forward order: "streamed" (default) or "receiver_state"
        (tp_conv_plan_set_schedule)."""
        code = {"streamed": 0, "receiver_state": 1}[schedule]
        check(lib().tp_conv_plan_set_schedule(self._h, code), "tp_conv_plan_set_schedule")

    def workspace_size(self, n_nodes: int, pass_: int) -> int:
        out = ctypes.c_size_t()
        check(lib().tp_conv_workspace_size(self._h, n_nodes, pass_, ctypes.byref(out)),
              "tp_conv_workspace_size")
        return out.value

    def launch_count(self, n_nodes: int, pass_: int) -> int:
        out = ctypes.c_int()
        check(lib().tp_conv_launch_count(self._h, n_nodes, pass_, ctypes.byref(out)), "tp_conv_launch_count")
        return out.value

    def work_model(self, n_nodes: int, n_edges: int, pass_: int) -> Tuple[float, float]:
        f, b = ctypes.c_double(), ctypes.c_double()
        check(lib().tp_conv_work_model(self._h, n_nodes, n_edges, pass_, ctypes.byref(f), ctypes.byref(b)),
              "tp_conv_work_model")
        return f.value, b.value

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            try:
                lib().tp_conv_plan_destroy(h)
            except Exception:
                pass
            self._h = None


def tp_conv_plan(irreps_in: str, sh_lmax: int, irreps_out: str, n_radial: int, mode: str = "uvu",
                 dtype: str = "f32") -> Plan:
    return Plan(irreps_in, sh_lmax, irreps_out, n_radial, mode, dtype)


def _workspace(nbytes: int, device, ws=None):
    torch = _torch()
    if nbytes == 0:
        return ws, 0
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, ws.numel()


def tp_csr_build(src, dst, n_nodes: int, out=None, ws=None, stream=None):
    """Receiver CSR of (src -> dst): returns (rowptr[N+1], senders[E], perm[E]), int32."""
    torch = _torch()
    E = src.numel()
    _need(src, torch.int32, (E,), "src")
    _need(dst, torch.int32, (E,), "dst")
    dev = src.device
    rowptr, senders, perm = out if out is not None else (
        torch.empty(n_nodes + 1, dtype=torch.int32, device=dev),
        torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E, dtype=torch.int32, device=dev))
    need = ctypes.c_size_t()
    check(lib().tp_csr_workspace_size(n_nodes, ctypes.byref(need)), "tp_csr_workspace_size")
    ws, wsb = _workspace(need.value, dev, ws)
    check(lib().tp_csr_build(n_nodes, E, _ptr(src), _ptr(dst), _ptr(rowptr), _ptr(senders), _ptr(perm),
                             _ptr(ws), wsb, _stream(stream)), "tp_csr_build")
    return rowptr, senders, perm


def tp_csr_transpose(rowptr, senders, n_nodes: int, out=None, ws=None, stream=None):
    """Source view: returns (colptr[N+1], srcedge[E], srcrecv[E]), int32."""
    torch = _torch()
    E = senders.numel()
    dev = senders.device
    colptr, srcedge, srcrecv = out if out is not None else (
        torch.empty(n_nodes + 1, dtype=torch.int32, device=dev),
        torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E, dtype=torch.int32, device=dev))
    need = ctypes.c_size_t()
    check(lib().tp_csr_workspace_size(n_nodes, ctypes.byref(need)), "tp_csr_workspace_size")
    ws, wsb = _workspace(need.value, dev, ws)
    check(lib().tp_csr_transpose(n_nodes, E, _ptr(rowptr), _ptr(senders), _ptr(colptr), _ptr(srcedge),
                                 _ptr(srcrecv), _ptr(ws), wsb, _stream(stream)), "tp_csr_transpose")
    return colptr, srcedge, srcrecv


def tp_conv_forward(plan: Plan, x, Y, phi, A, rowptr, senders, out=None, ws=None, stream=None):
    """out[N, C_out] = the convolution (Y, phi in CSR edge order)."""
    torch = _torch()
    N, E = x.shape[0], senders.numel()
    dt = plan.torch_dtype
    _need(x, dt, (N, plan.c_in), "x")
    _need(Y, dt, (E, plan.dim_y), "Y")
    _need(phi, dt, (E, plan.n_radial), "phi")
    _need(A, dt, (plan.n_radial, plan.n_w), "A")
    _need(rowptr, torch.int32, (N + 1,), "rowptr")
    if out is None:
        out = torch.empty(N, plan.c_out, dtype=dt, device=x.device)
    ws, wsb = _workspace(plan.workspace_size(N, 0), x.device, ws)
    check(lib().tp_conv_forward(plan.handle, _ptr(x), _ptr(Y), _ptr(phi), _ptr(A), _ptr(rowptr),
                                _ptr(senders), N, E, _ptr(out), _ptr(ws), wsb, _stream(stream)),
          "tp_conv_forward")
    return out


def tp_conv_backward(plan: Plan, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv, grad_out,
                     out=None, ws=None, stream=None):
    """Returns (grad_x, grad_Y, grad_phi, grad_A)."""
    torch = _torch()
    N, E = x.shape[0], senders.numel()
    dt = plan.torch_dtype
    _need(grad_out, dt, (N, plan.c_out), "grad_out")
    if out is None:
        out = (torch.empty(N, plan.c_in, dtype=dt, device=x.device),
               torch.empty(E, plan.dim_y, dtype=dt, device=x.device),
               torch.empty(E, plan.n_radial, dtype=dt, device=x.device),
               torch.empty(plan.n_radial, plan.n_w, dtype=dt, device=x.device))
    gx, gY, gphi, gA = out
    ws, wsb = _workspace(plan.workspace_size(N, 1), x.device, ws)
    check(lib().tp_conv_backward(plan.handle, _ptr(x), _ptr(Y), _ptr(phi), _ptr(A), _ptr(rowptr),
                                 _ptr(senders), _ptr(colptr), _ptr(srcedge), _ptr(srcrecv),
                                 _ptr(grad_out), N, E, _ptr(gx), _ptr(gY), _ptr(gphi), _ptr(gA),
                                 _ptr(ws), wsb, _stream(stream)), "tp_conv_backward")
    return gx, gY, gphi, gA


def tp_conv_double_backward(plan: Plan, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv, grad_out,
                            dx, dY, dphi, dA, out=None, ws=None, stream=None):
    """Second-order program along (dx, dY, dphi, dA) with grad_out fixed.
    Returns (d_out, dgrad_x, dgrad_Y, dgrad_phi, dgrad_A)."""
    torch = _torch()
    N, E = x.shape[0], senders.numel()
    dt = plan.torch_dtype
    _need(grad_out, dt, (N, plan.c_out), "grad_out")
    _need(dx, dt, (N, plan.c_in), "dx")
    _need(dY, dt, (E, plan.dim_y), "dY")
    _need(dphi, dt, (E, plan.n_radial), "dphi")
    _need(dA, dt, (plan.n_radial, plan.n_w), "dA")
    if out is None:
        out = (torch.empty(N, plan.c_out, dtype=dt, device=x.device),
               torch.empty(N, plan.c_in, dtype=dt, device=x.device),
               torch.empty(E, plan.dim_y, dtype=dt, device=x.device),
               torch.empty(E, plan.n_radial, dtype=dt, device=x.device),
               torch.empty(plan.n_radial, plan.n_w, dtype=dt, device=x.device))
    ws, wsb = _workspace(plan.workspace_size(N, 2), x.device, ws)
    check(lib().tp_conv_double_backward(plan.handle, _ptr(x), _ptr(Y), _ptr(phi), _ptr(A), _ptr(rowptr),
                                        _ptr(senders), _ptr(colptr), _ptr(srcedge), _ptr(srcrecv),
                                        _ptr(grad_out), _ptr(dx), _ptr(dY), _ptr(dphi), _ptr(dA), N, E,
                                        *[_ptr(t) for t in out], _ptr(ws), wsb, _stream(stream)),
          "tp_conv_double_backward")
    return out


def tp_conv_backward_noalloc(plan: Plan, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv,
                             grad_out, out=None, stream=None):
    """tp_conv_backward without a workspace argument: the library's static
    device scratch holds the grad_A partials (see include/tpconv.h). The output
    tensors are the caller's; pass `out` to avoid any allocation here too."""
    torch = _torch()
    N, E = x.shape[0], senders.numel()
    dt = plan.torch_dtype
    _need(grad_out, dt, (N, plan.c_out), "grad_out")
    if out is None:
        out = (torch.empty(N, plan.c_in, dtype=dt, device=x.device),
               torch.empty(E, plan.dim_y, dtype=dt, device=x.device),
               torch.empty(E, plan.n_radial, dtype=dt, device=x.device),
               torch.empty(plan.n_radial, plan.n_w, dtype=dt, device=x.device))
    gx, gY, gphi, gA = out
    check(lib().tp_conv_backward_noalloc(plan.handle, _ptr(x), _ptr(Y), _ptr(phi), _ptr(A), _ptr(rowptr),
                                         _ptr(senders), _ptr(colptr), _ptr(srcedge), _ptr(srcrecv),
                                         _ptr(grad_out), N, E, _ptr(gx), _ptr(gY), _ptr(gphi), _ptr(gA),
                                         _stream(stream)), "tp_conv_backward_noalloc")
    return gx, gY, gphi, gA


def tp_get_device_error(stream=None) -> int:
    """Synchronise, read and clear the device error word; returns the status code."""
    return lib().tp_get_device_error(_stream(stream))
