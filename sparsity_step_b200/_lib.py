"""ctypes loader of the in-tree CUDA library ``libbitlinear.so``.

There is no fallback: if the library is missing or fails to load, every entry
point raises. Build it with ``python -m sparsity_step_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libbitlinear.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "bitlinear.h")

BL_OK = 0
STATUS_NAMES = {
    0: "BL_OK", -1: "BL_ERR_INVALID_ARG", -2: "BL_ERR_UNSUPPORTED_SHAPE", -3: "BL_ERR_ALIGNMENT",
    -4: "BL_ERR_RANGE", -5: "BL_ERR_CUDA", -6: "BL_ERR_TIMEOUT", -7: "BL_ERR_WORKSPACE",
}
BL_OUT_BF16 = 0
BL_OUT_F32 = 1

_c = ctypes
_P = _c.c_void_p
_I64 = _c.c_int64
_INT = _c.c_int
_SZ = _c.c_size_t
_F32 = _c.c_float

class BlFwdProblem(ctypes.Structure):
    """bl_fwd_problem of include/bitlinear.h."""
    _fields_ = [("xq", ctypes.c_void_p), ("absmax", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("w_scale", ctypes.c_void_p), ("t", ctypes.c_int64), ("k_in", ctypes.c_int64),
                ("n_out", ctypes.c_int64), ("acc_out", ctypes.c_void_p), ("y_out", ctypes.c_void_p)]


class BlGradWProblem(ctypes.Structure):
    """bl_grad_w_problem of include/bitlinear.h."""
    _fields_ = [("dy", ctypes.c_void_p), ("x", ctypes.c_void_p), ("k_in", ctypes.c_int64), ("n_out", ctypes.c_int64),
                ("grad_w", ctypes.c_void_p), ("grad_w_dtype", ctypes.c_int)]


# name -> (restype, argtypes), in the order of include/bitlinear.h
SIGNATURES = {
    "bitlinear_quant_mask_workspace_size": (_SZ, [_I64, _I64]),
    "bitlinear_quant_mask": (_INT, [_P, _I64, _I64, _INT, _INT, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "bitlinear_sgd_quant_mask": (_INT, [_P, _P, _F32, _I64, _I64, _INT, _INT, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "bitlinear_quant_mask_status": (_INT, [_P, _P]),
    "bitlinear_quant_mask_noalloc": (_INT, [_P, _I64, _I64, _INT, _INT, _P, _P, _P, _P, _P]),
    "bitlinear_act_quant": (_INT, [_P, _I64, _I64, _P, _P, _P]),
    "bitlinear_fwd": (_INT, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _INT, _P]),
    "bitlinear_fwd_grouped": (_INT, [_c.POINTER(BlFwdProblem), _INT, _INT, _P]),
    "bitlinear_bwd_workspace_size": (_SZ, [_I64, _I64, _I64, _INT, _INT]),
    "bitlinear_bwd": (_INT, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _INT, _INT, _P, _SZ, _P]),
    "bitlinear_grad_w_grouped": (_INT, [_P, _INT, _I64, _P]),
    "bitlinear_grad_x_i8_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bitlinear_grad_x_i8": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "bitlinear_mask_threshold_hist": (_INT, [_P, _P, _P, _I64, _I64, _INT, _P, _P]),
    "bitlinear_device_status": (_INT, [_c.POINTER(_c.c_uint)]),
    "bitlinear_last_error": (_c.c_char_p, []),
    "bitlinear_abi_version": (_INT, []),
}

_LIB = None


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")


def header_functions() -> list[str]:
    """Names of the functions include/bitlinear.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"\b(bitlinear_\w+)\s*\(", text)


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparsity_step_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def check(status: int, where: str) -> None:
    if status != BL_OK:
        msg = lib().bitlinear_last_error()
        raise BitLinearError(status, where, msg.decode() if msg else "")
