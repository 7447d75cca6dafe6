"""ctypes declarations of libtpconv.so (the C ABI of include/tpconv.h).

Loading fails loudly when the library has not been built: there is no other
implementation behind these names.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_int, c_int32, c_int64, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtpconv.so")

TP_UVU, TP_UVW, TP_UVU_PATHS = 0, 1, 2
TP_F32, TP_F64 = 0, 1
STATUS = {0: "TP_OK", -1: "TP_EINVAL", -2: "TP_EUNSUPPORTED", -3: "TP_ECUDA",
          -4: "TP_EWORKSPACE", -5: "TP_EDEVICE_INDEX", -6: "TP_EDEVICE_CSR", -7: "TP_EDEVICE_TIMEOUT"}


class PlanInfo(ctypes.Structure):
    _fields_ = [("c_in", c_int32), ("c_out", c_int32), ("dim_y", c_int32), ("n_radial", c_int32),
                ("n_paths", c_int32), ("mode", c_int32), ("dtype", c_int32), ("sh_lmax", c_int32),
                ("lmax", c_int32), ("pad", c_int32), ("n_w", c_int64)]


class PathInfo(ctypes.Structure):
    _fields_ = [("l1", c_int32), ("p1", c_int32), ("l2", c_int32), ("p2", c_int32), ("l3", c_int32),
                ("p3", c_int32), ("block_in", c_int32), ("block_out", c_int32), ("mul_in", c_int32),
                ("mul_out", c_int32), ("x_off", c_int32), ("out_off", c_int32), ("w_off", c_int64),
                ("n_w", c_int64), ("nnz", c_int32), ("pad", c_int32)]


# every exported symbol of tpconv.h with (restype, argtypes)
SIGNATURES = {
    "tp_conv_plan": (c_int, [c_char_p, c_int, c_char_p, c_int, c_int, c_int, POINTER(c_void_p)]),
    "tp_conv_plan_sh": (c_int, [c_char_p, c_char_p, c_char_p, c_int, c_int, c_int, POINTER(c_void_p)]),
    "tp_conv_plan_destroy": (c_int, [c_void_p]),
    "tp_conv_plan_info": (c_int, [c_void_p, POINTER(PlanInfo)]),
    "tp_conv_plan_path": (c_int, [c_void_p, c_int, POINTER(PathInfo)]),
    "tp_conv_plan_cg": (c_int, [c_void_p, c_int, POINTER(c_int32), POINTER(c_int32), POINTER(c_int32),
                                POINTER(c_double), c_int]),
    "tp_conv_plan_set_state_budget": (c_int, [c_void_p, c_size_t]),
    "tp_conv_plan_set_schedule": (c_int, [c_void_p, c_int]),
    "tp_conv_work_model": (c_int, [c_void_p, c_int64, c_int64, c_int, POINTER(c_double), POINTER(c_double)]),
    "tp_conv_workspace_size": (c_int, [c_void_p, c_int64, c_int, POINTER(c_size_t)]),
    "tp_conv_launch_count": (c_int, [c_void_p, c_int64, c_int, POINTER(c_int)]),
    "tp_csr_workspace_size": (c_int, [c_int64, POINTER(c_size_t)]),
    "tp_csr_build": (c_int, [c_int64, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_void_p, c_size_t, c_void_p]),
    "tp_csr_transpose": (c_int, [c_int64, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_size_t, c_void_p]),
    "tp_conv_forward": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_int64, c_int64, c_void_p, c_void_p, c_size_t, c_void_p]),
    "tp_conv_backward": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "tp_conv_double_backward": (c_int, [c_void_p] + [c_void_p] * 14 + [c_int64, c_int64] + [c_void_p] * 5
                                + [c_void_p, c_size_t, c_void_p]),
    "tp_conv_backward_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_void_p]),
    "tp_get_device_error": (c_int, [c_void_p]),
    "tp_status_string": (c_char_p, [c_int]),
    "tp_last_error_message": (c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class TpConvError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib().tp_last_error_message().decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")
        self.status = status


def check(status: int, where: str) -> int:
    if status < 0:
        raise TpConvError(status, where)
    return status
