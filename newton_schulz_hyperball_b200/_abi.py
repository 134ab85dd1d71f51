"""ctypes mirror of include/nshb.h.  Argument marshalling only: every computation
happens inside libnshb.so.  Loading fails loudly if the library is missing."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnshb.so")

NSHB_BF16 = 0
NSHB_F32 = 1

NSHB_OK = 0
NSHB_ERR_NULL = 1
NSHB_ERR_SHAPE = 2
NSHB_ERR_DTYPE = 3
NSHB_ERR_PARAM = 4
NSHB_ERR_WORKSPACE = 5
NSHB_ERR_CUDA = 6
NSHB_ERR_DEVICE_TIMEOUT = 7
NSHB_ERR_NONFINITE = 8
NSHB_ERR_ZERO_NORM = 9
NSHB_ERR_UNSUPPORTED = 10

NSHB_DEV_ZERO_NORM_FALLBACK = 0x1
NSHB_DEV_NONFINITE = 0x2
NSHB_DEV_TIMEOUT = 0x4
NSHB_DEV_ZERO_RADIUS = 0x8
NSHB_DEV_NOT_SPD = 0x10

NSHB_PROF_NAMES = ["momentum", "norm", "gram", "poly", "update", "reduce", "finalize", "exact", "apply",
                   "f32gemm", "newton", "adam"]
NSHB_PROF_KINDS = 12

NSHB_OP_MUON = 0
NSHB_OP_HYPERBALL = 1
NSHB_OP_RADIAL_BRAKE = 2
NSHB_OP_HIMUON = 3
NSHB_OP_NEWTON_MUON = 4
NSHB_OP_RELATIVE_UPDATE = 5
NSHB_OP_ADAMH = 6


class nshb_matrix(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("ld", ctypes.c_int64),
        ("w_dtype", ctypes.c_int32),
        ("z_index", ctypes.c_int32),
        ("W", ctypes.c_void_p),
        ("G", ctypes.c_void_p),
        ("M", ctypes.c_void_p),
        ("O_out", ctypes.c_void_p),
    ]


class nshb_params(ctypes.Structure):
    _fields_ = [
        ("beta", ctypes.c_float),
        ("nesterov", ctypes.c_int32),
        ("ns_steps", ctypes.c_int32),
        ("ns_precision", ctypes.c_int32),
        ("coeffs", ctypes.POINTER(ctypes.c_float)),
        ("ns_eps", ctypes.c_float),
        ("lr", ctypes.c_float),
        ("weight_decay", ctypes.c_float),
        ("eta", ctypes.c_float),
        ("rho", ctypes.c_void_p),
        ("hb_eps", ctypes.c_float),
        ("brake_out", ctypes.c_float),
        ("brake_in", ctypes.c_float),
        ("tile", ctypes.c_int32),
        ("ridge_rel", ctypes.c_float),
        ("ns_compensated", ctypes.c_int32),
        ("debug_flags", ctypes.c_uint32),
    ]


class nshb_adam_params(ctypes.Structure):
    _fields_ = [
        ("beta1", ctypes.c_float),
        ("beta2", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("step", ctypes.c_int32),
    ]


# name -> (restype, argtypes)
_P = ctypes.c_void_p
_MATS = ctypes.POINTER(nshb_matrix)
_PAR = ctypes.POINTER(nshb_params)
SIGNATURES = {
    "nshb_default_params": (ctypes.c_int32, [_PAR]),
    "nshb_workspace_size": (ctypes.c_int32, [_MATS, ctypes.c_int32, _PAR, ctypes.c_int32,
                                             ctypes.POINTER(ctypes.c_int64), ctypes.c_int32, ctypes.c_int64,
                                             ctypes.POINTER(ctypes.c_size_t)]),
    "muon_step": (ctypes.c_int32, [_MATS, ctypes.c_int32, _PAR, _P, ctypes.c_size_t, _P]),
    "hyperball_step": (ctypes.c_int32, [_MATS, ctypes.c_int32, _PAR, _P, ctypes.c_size_t, _P]),
    "radial_brake_step": (ctypes.c_int32, [_MATS, ctypes.c_int32, _PAR, _P, ctypes.c_size_t, _P]),
    "relative_update_step": (ctypes.c_int32, [_MATS, ctypes.c_int32, _PAR, _P, ctypes.c_size_t, _P]),
    "nshb_default_adam_params": (ctypes.c_int32, [ctypes.POINTER(nshb_adam_params)]),
    "adamh_step": (ctypes.c_int32, [_MATS, ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p),
                                    ctypes.POINTER(nshb_adam_params), _PAR, _P, ctypes.c_size_t, _P]),
    "himuon_step": (ctypes.c_int32, [_MATS, ctypes.c_int32, _PAR, _P, ctypes.c_size_t, _P]),
    "newton_muon_step": (ctypes.c_int32, [_MATS, ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p),
                                          ctypes.POINTER(ctypes.c_int64), ctypes.c_int32, ctypes.c_int64,
                                          _PAR, _P, ctypes.c_size_t, _P]),
    "nshb_workspace_size_min": (ctypes.c_int32, [_MATS, ctypes.c_int32, _PAR, ctypes.c_int32,
                                                 ctypes.POINTER(ctypes.c_size_t)]),
    "nshb_step_chunked": (ctypes.c_int32, [ctypes.c_int32, _MATS, ctypes.c_int32, _PAR, _P, ctypes.c_size_t, _P,
                                           ctypes.POINTER(ctypes.c_int32)]),
    "nshb_fro_norms": (ctypes.c_int32, [_MATS, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]),
    "nshb_fro_norms_static": (ctypes.c_int32, [_MATS, ctypes.c_int32, _P, _P]),
    "nshb_device_status": (ctypes.c_int32, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "nshb_status_string": (ctypes.c_char_p, [ctypes.c_int32]),
    "nshb_version": (ctypes.c_int32, []),
    "nshb_last_cuda_error": (ctypes.c_int32, []),
    "nshb_profile_enable": (ctypes.c_int32, [ctypes.c_int32]),
    "nshb_profile_read": (ctypes.c_int32, [ctypes.c_int32, ctypes.POINTER(ctypes.c_float),
                                           ctypes.POINTER(ctypes.c_int32)]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m newton_schulz_hyperball_b200.build` "
                          "(the optimizer step has no fallback without the CUDA library)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
