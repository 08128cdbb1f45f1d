"""ctypes loader of libmova.so: argument marshalling only.

The library must have been built (``python -m mixture_value_routing_b200.build``);
importing the compute API without it raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmova.so")

# mova_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_CHECK = range(6)
STATUS_NAMES = {OK: "MOVA_OK", ERR_INVALID_ARG: "MOVA_ERR_INVALID_ARG",
                ERR_UNSUPPORTED: "MOVA_ERR_UNSUPPORTED", ERR_CUDA: "MOVA_ERR_CUDA",
                ERR_TIMEOUT: "MOVA_ERR_TIMEOUT", ERR_DEVICE_CHECK: "MOVA_ERR_DEVICE_CHECK"}
# mova_dtype
F32, BF16, F16, I32, I8 = range(5)
# mova_path
PATH_AUTO, PATH_STREAM, PATH_TENSOR, PATH_TENSOR_1CTA = range(4)
# parts of the workspace (mova_workspace_parts)
WS_PARTS = ("idx", "w", "counts", "offsets", "perm", "pos")
# stage events recorded by the _ex entry points
STAGE_EVENTS = 5
STAGES = ("route", "group", "experts", "combine")

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t


class Options(ctypes.Structure):
    """mova_options (include/mova.h)."""
    _fields_ = [("path", ctypes.c_int), ("events", ctypes.c_void_p),
                ("wv_expert_stride", ctypes.c_longlong), ("router_partitions", ctypes.c_int),
                ("decode_launches", ctypes.c_int), ("router_planes", ctypes.c_void_p)]


SIGNATURES = {
    "mova_status_str": (ctypes.c_char_p, [_i]),
    "mova_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "mova_auto_path": (_i, [_i, _i]),
    "mova_launch_count": (ctypes.c_ulonglong, []),
    "mova_route": (_i, [_vp, _i, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp, _vp]),
    "mova_permute": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mova_value": (_i, [_vp, _i, _vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "mova_value_ex": (_i, [_vp, _i, _vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz,
                           _i, _vp, _vp]),
    "mova_value_routed": (_i, [_vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp,
                               _vp, _sz, _vp]),
    "mova_value_routed_ex": (_i, [_vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp,
                                  _vp, _vp, _sz, _i, _vp, _vp]),
    "mova_get_status": (_i, [_vp, _vp, _vp]),
    "mova_selftest_wait_timeout": (_i, [_vp, ctypes.c_longlong, _vp]),
    "mova_selftest_arm_stream_stall": (_i, [_i, ctypes.c_longlong]),
    "mova_workspace_parts": (_i, [_i, _i, _i, _i, _i, _vp]),
    "mova_router_planes_bytes": (_sz, [_i]),
    "mova_attend_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "mova_value_attend": (_i, [_vp, _vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _sz, _vp]),
    "mova_router_planes": (_i, [_vp, _i, _i, _vp, _vp]),
    "mova_workspace_size_host": (_sz, [_i, _i, _i, _i, _i]),
    "mova_attend_workspace_size_host": (_sz, [_i, _i, _i, _i, _i, _i]),
    "mova_value_routed_host": (_i, [_vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp,
                                    _vp, _sz, _vp]),
    "mova_value_host": (_i, [_vp, _i, _vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "mova_value_attend_host": (_i, [_vp, _vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _sz,
                                    _vp]),
    "mova_value_routed_noalloc": (_i, [_vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp,
                                       _vp]),
    "mova_route_opts": (_i, [_vp, _i, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp]),
    "mova_value_opts": (_i, [_vp, _i, _vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _sz,
                             _vp, _vp]),
    "mova_value_routed_opts": (_i, [_vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp,
                                    _vp, _vp, _sz, _vp, _vp]),
}

_lib = None


class MovaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")
        self.code = code


def load() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mixture_value_routing_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(code: int, where: str) -> None:
    if code != OK:
        raise MovaError(code, where)
