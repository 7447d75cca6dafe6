"""Host-side argument validation of the C ABI (include/tpconv.h): every check
runs before any device work, so it is exercised here without a GPU. The
pointers below are never dereferenced: each call fails validation first."""
import ctypes

import pytest

import clebsch_gordan_tensor_node_b200 as tpc
from clebsch_gordan_tensor_node_b200._lib import lib

TP_EINVAL, TP_EWORKSPACE = -1, -4
A16 = 0x10000          # a 16-byte aligned address (never touched)
MIS = 0x10004          # not 16-byte aligned


def _fwd(plan, x=A16, Y=A16, phi=A16, A=A16, rowptr=A16, senders=A16, n=8, e=16, out=A16, ws=None, wsb=0):
    return lib().tp_conv_forward(plan.handle, x, Y, phi, A, rowptr, senders, n, e, out, ws, wsb, None)


def _bwd(plan, n=8, e=16, ws=A16, wsb=0, x=A16, gx=A16):
    return lib().tp_conv_backward(plan.handle, x, A16, A16, A16, A16, A16, A16, A16, A16, A16, n, e, gx, A16,
                                  A16, A16, ws, wsb, None)


@pytest.fixture(scope="module")
def uvu():
    return tpc.Plan("4x0e+4x1o", 1, "4x0e+4x1o", 8, "uvu", "f32")


@pytest.fixture(scope="module")
def uvw():
    return tpc.Plan("4x0e+4x1o", 1, "4x0e+4x1o", 8, "uvw", "f32")


def test_forward_rejects_null_and_misaligned(uvu):
    assert _fwd(uvu, x=None) == TP_EINVAL
    assert _fwd(uvu, out=None) == TP_EINVAL
    assert _fwd(uvu, x=MIS) == TP_EINVAL
    assert _fwd(uvu, A=MIS) == TP_EINVAL
    assert lib().tp_last_error_message()


def test_forward_rejects_bad_sizes(uvu):
    assert _fwd(uvu, n=-1) == TP_EINVAL
    assert _fwd(uvu, e=-5) == TP_EINVAL
    assert _fwd(uvu, n=1 << 31) == TP_EINVAL


def test_uvw_forward_needs_its_workspace(uvw):
    need = uvw.workspace_size(8, 0)
    assert need > 0
    assert _fwd(uvw, ws=A16, wsb=need - 1) == TP_EWORKSPACE


def test_backward_checks_workspace_and_pointers(uvu, uvw):
    for plan in (uvu, uvw):
        need = plan.workspace_size(8, 1)
        assert need > 0
        assert _bwd(plan, wsb=need - 1) == TP_EWORKSPACE
        assert _bwd(plan, wsb=need, x=None) == TP_EINVAL
        assert _bwd(plan, wsb=need, gx=MIS) == TP_EINVAL


def test_null_plan_is_rejected():
    assert lib().tp_conv_forward(None, A16, A16, A16, A16, A16, A16, 8, 16, A16, None, 0, None) == TP_EINVAL
    f = ctypes.c_double()
    assert lib().tp_conv_work_model(None, 8, 16, 0, ctypes.byref(f), ctypes.byref(f)) == TP_EINVAL
