"""ctypes declarations of libmate.so (the C ABI in include/mate.h).

Argument marshalling only. Loading fails loudly when the library has not
been built: there is no fallback implementation of any kernel.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmate.so")

MATE_OK = 0
MATE_ERR_INVALID_ARG = -1
MATE_ERR_UNSUPPORTED = -2
MATE_ERR_CUDA = -3
MATE_ERR_TIMEOUT = -4
MATE_ERR_WORKSPACE = -5

MATE_F32 = 0
MATE_BF16 = 1

MATE_DIR_FWD, MATE_DIR_BWD, MATE_DIR_BI = 1, 2, 3

# every symbol include/mate.h declares
EXPORTS = (
    "mate_bissd_workspace_bytes",
    "mate_bissd_fwd",
    "tesa_fwd",
    "mate_debug_rms_map",
    "mate_debug_tesa_map",
    "mate_debug_fastdiv",
    "mate_last_error",
    "mate_status_string",
    "mate_version",
    "mate_set_phase_hook",
    "mate_kernel_launches",
    "mate_bissd_fwd_noalloc",
    "mate_compose_fwd",
    "mate_frontend_workspace_bytes",
    "mate_frontend_fwd",
    "mate_gate_norm_fwd",
)

NOALLOC_SCRATCH_BYTES = 32 << 20

PHASES = {1: "review_pool", 2: "review_scan", 3: "chunk_state", 4: "state_pass", 5: "chunk_out", 6: "tesa",
          7: "compose", 8: "front_proj", 9: "front_conv", 10: "front_dt", 11: "gate_norm"}
PHASE_HOOK = ctypes.CFUNCTYPE(None, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p)


class mate_ssd_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("nheads", ctypes.c_int), ("headdim", ctypes.c_int),
                ("dstate", ctypes.c_int), ("ngroups", ctypes.c_int), ("chunk", ctypes.c_int),
                ("dtype", ctypes.c_int), ("directions", ctypes.c_int)]


class mate_attn_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("nheads", ctypes.c_int), ("headdim", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class mate_compose_dims(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_int), ("k_ma", ctypes.c_int), ("k_te", ctypes.c_int), ("d_model", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class mate_gate_norm_dims(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_int), ("channels", ctypes.c_int), ("group", ctypes.c_int), ("dtype", ctypes.c_int)]


class mate_frontend_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("d_model", ctypes.c_int), ("nheads", ctypes.c_int), ("headdim", ctypes.c_int),
                ("ngroups", ctypes.c_int), ("dstate", ctypes.c_int), ("dtype", ctypes.c_int)]


class MateError(RuntimeError):
    def __init__(self, fn: str, code: int, text: str):
        super().__init__(f"{fn} returned {code} ({text})")
        self.code = code


_vp = ctypes.c_void_p
_ip = ctypes.POINTER(ctypes.c_int)
_lib = None


def load() -> ctypes.CDLL:
    """Load libmate.so once; raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmate.so not built at {LIB_PATH}; run python -m linear_complexity_video_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    L.mate_bissd_workspace_bytes.argtypes = [ctypes.c_int] * 3 + [_ip, ctypes.POINTER(mate_ssd_dims)]
    L.mate_bissd_workspace_bytes.restype = ctypes.c_size_t
    L.mate_bissd_fwd.argtypes = [_vp] * 6 + [ctypes.c_int] * 4 + [_ip, _vp, ctypes.POINTER(mate_ssd_dims), _vp,
                                                                    ctypes.c_size_t, _vp]
    L.mate_bissd_fwd.restype = ctypes.c_int
    L.tesa_fwd.argtypes = [_vp] * 3 + [ctypes.c_int] * 5 + [_ip, _vp, ctypes.POINTER(mate_attn_dims), _vp]
    L.tesa_fwd.restype = ctypes.c_int
    L.mate_debug_rms_map.argtypes = [ctypes.c_int] * 5 + [_vp, _vp]
    L.mate_debug_rms_map.restype = ctypes.c_int
    L.mate_debug_tesa_map.argtypes = [ctypes.c_int] * 5 + [_ip, _vp, _vp]
    L.mate_debug_tesa_map.restype = ctypes.c_int
    L.mate_last_error.argtypes = [_vp]
    L.mate_last_error.restype = ctypes.c_int
    L.mate_status_string.argtypes = [ctypes.c_int]
    L.mate_status_string.restype = ctypes.c_char_p
    L.mate_debug_fastdiv.argtypes = [_vp, _vp, ctypes.c_size_t, ctypes.c_uint32]
    L.mate_debug_fastdiv.restype = ctypes.c_int
    L.mate_compose_fwd.argtypes = [_vp] * 5 + [ctypes.POINTER(mate_compose_dims), _vp]
    L.mate_compose_fwd.restype = ctypes.c_int
    L.mate_gate_norm_fwd.argtypes = [_vp] * 3 + [ctypes.c_float, _vp, ctypes.POINTER(mate_gate_norm_dims), _vp]
    L.mate_gate_norm_fwd.restype = ctypes.c_int
    L.mate_frontend_workspace_bytes.argtypes = [ctypes.c_int] * 3 + [ctypes.POINTER(mate_frontend_dims)]
    L.mate_frontend_workspace_bytes.restype = ctypes.c_size_t
    L.mate_frontend_fwd.argtypes = [_vp] * 5 + [ctypes.c_int] * 4 + [_vp] * 5 + [ctypes.POINTER(mate_frontend_dims),
                                                                            _vp, ctypes.c_size_t, _vp]
    L.mate_frontend_fwd.restype = ctypes.c_int
    L.mate_version.argtypes = []
    L.mate_version.restype = ctypes.c_int
    L.mate_set_phase_hook.argtypes = [PHASE_HOOK, ctypes.c_void_p]
    L.mate_set_phase_hook.restype = None
    L.mate_bissd_fwd_noalloc.argtypes = [_vp] * 6 + [ctypes.c_int] * 4 + [_ip, _vp, ctypes.POINTER(mate_ssd_dims),
                                                                            _vp]
    L.mate_bissd_fwd_noalloc.restype = ctypes.c_int
    L.mate_kernel_launches.argtypes = []
    L.mate_kernel_launches.restype = ctypes.c_uint64
    _lib = L
    return L


def check(fn: str, code: int) -> None:
    if code != MATE_OK:
        raise MateError(fn, code, load().mate_status_string(code).decode())
