"""ctypes declarations of the C ABI in include/nerf.h (argument marshalling only).

The names and argument orders are those of the header. Loading fails loudly
when libnerf.so is missing: there is no other implementation behind them.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnerf.so")

NERF_OK = 0
NERF_ERR_INVALID_ARG = 1
NERF_ERR_CUDA = 2
NERF_ERR_UNSUPPORTED = 3
NERF_ERR_OOM = 4
NERF_ERR_TIMEOUT = 5
NERF_ERR_DEVICE_FLAG = 6

NERF_MODEL_MLP, NERF_MODEL_KILONERF, NERF_MODEL_HASHGRID = 0, 1, 2
NERF_SIGMA_RELU, NERF_SIGMA_SOFTPLUS = 0, 1
NERF_FP32, NERF_BF16, NERF_TF32 = 0, 1, 2
NERF_LAST_1E10, NERF_LAST_TO_FAR = 0, 1
TIMED_KINDS = ("network", "composite", "resample", "dir_bias", "march_mask", "march_compact",
               "router", "march_composite")           # NERF_TIMED_* order

_STATUS = {0: "NERF_OK", 1: "NERF_ERR_INVALID_ARG", 2: "NERF_ERR_CUDA", 3: "NERF_ERR_UNSUPPORTED",
           4: "NERF_ERR_OOM", 5: "NERF_ERR_TIMEOUT", 6: "NERF_ERR_DEVICE_FLAG"}


class nerf_config(ctypes.Structure):
    _fields_ = [("model", ctypes.c_int), ("D", ctypes.c_int), ("W", ctypes.c_int),
                ("skip", ctypes.c_int), ("L_pos", ctypes.c_int), ("L_dir", ctypes.c_int),
                ("sigma_act", ctypes.c_int), ("precision", ctypes.c_int),
                ("last_delta_mode", ctypes.c_int), ("white_bkgd", ctypes.c_int),
                ("max_rays", ctypes.c_int64), ("max_samples", ctypes.c_int)]


class nerf_params(ctypes.Structure):
    _fields_ = [("coarse_w", ctypes.c_void_p), ("fine_w", ctypes.c_void_p),
                ("occupancy", ctypes.c_void_p), ("cell_w", ctypes.c_void_p),
                ("hash_table", ctypes.c_void_p), ("hash_mlp", ctypes.c_void_p),
                ("march_step", ctypes.c_float), ("ert_T", ctypes.c_float),
                ("seed", ctypes.c_uint64), ("perturb", ctypes.c_int)]


class nerf_trace(ctypes.Structure):
    _fields_ = [("raw_coarse", ctypes.c_void_p), ("w_coarse", ctypes.c_void_p),
                ("t_fine", ctypes.c_void_p), ("below", ctypes.c_void_p),
                ("t_all", ctypes.c_void_p), ("raw_fine", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float
_I = ctypes.c_int
_U64 = ctypes.c_uint64

# name -> (restype, argtypes), in header order
SIGNATURES = {
    "nerf_create": (_I, [ctypes.POINTER(nerf_config), ctypes.POINTER(_P)]),
    "nerf_destroy": (_I, [_P]),
    "nerf_last_error": (ctypes.c_char_p, [_P]),
    "nerf_sync_status": (_I, [_P, _P]),
    "nerf_raygen": (_I, [_I, _I, _F, _P, _P, _P, _P]),
    "nerf_raygen_batch": (_I, [_I, _I, _F, _I, _P, _P, _P, _P]),
    "nerf_render": (_I, [_P, _P, _P, _I64, _F, _F, _I, _I, ctypes.POINTER(nerf_params),
                         _P, _P, _P, _P]),
    "nerf_render_trace": (_I, [_P, _P, _P, _I64, _F, _F, _I, _I, ctypes.POINTER(nerf_params),
                               _P, _P, _P, ctypes.POINTER(nerf_trace), _P]),
    "nerf_loss_grad": (_I, [_P, _P, _P, _I64, _F, _F, _I, _I, ctypes.POINTER(nerf_params),
                            _P, _P, _P, _P, _P]),
    "nerf_render_host": (_I, [_P, _P, _P, _I64, _F, _F, _I, _I, ctypes.POINTER(nerf_params),
                              _P, _P, _P, _P]),
    "nerf_timing_enable": (_I, [_P, _I]),
    "nerf_timing_read": (_I, [_P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I64)]),
    "nerf_timing_read_kinds": (_I, [_P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I64)]),
    "nerf_test_stratified": (_I, [_P, _P, _I64, _F, _F, _I, _U64, _I, _P, _P, _P]),
    "nerf_test_pe": (_I, [_P, _I64, _I, _P, _P]),
    "nerf_test_mlp": (_I, [_P, _P, _P, _P, _I64, _P, _P]),
    "nerf_test_composite": (_I, [_P, _P, _P, _I64, _I, _F, _I, _F, _I, _I, _P, _P, _P, _P, _P]),
    "nerf_test_sample_pdf": (_I, [_P, _P, _I64, _I, _I, _U64, _I, _P, _P, _P, _P]),
    "nerf_test_march": (_I, [_P, _P, _I64, _F, _F, _I, _P, _P, _P, _P]),
    "nerf_test_route_cells": (_I, [_P, _I64, _P, _P, _P, _P, _P]),
    "nerf_test_hash_encode": (_I, [_P, _I64, _P, _P, _P, _P]),
    "nerf_hash_encode_backward": (_I, [_P, _I64, _P, _P, _I, _P]),
    "nerf_test_sh": (_I, [_P, _I64, _P, _P]),
    "nerf_test_bounded_wait": (_I, [ctypes.c_uint32, _P, _P, _P]),
    "nerf_march_compact_noalloc": (_I, [_P, _P, _I64, _F, _F, _I, _P, _P, _P, _P]),
}

_lib = None


def lib():
    """The loaded libnerf.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python neural_radiance_field_b200/build.py`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class NerfError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


def check(status, ctx=None):
    if status != NERF_OK:
        msg = lib().nerf_last_error(ctx)
        raise NerfError(status, msg.decode() if msg else "")
    return status
