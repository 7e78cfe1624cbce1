"""MATE token-mix core of LinGen on NVIDIA B200 (sm_100a).

The computation lives in libmate.so (C ABI: include/mate.h); this package
only loads it and marshals torch tensors into its calls.
"""
from .api import (bissd, bissd_workspace, block, compose, frontend, gate_norm, linear, mate_bissd_fwd, mate_bissd_workspace_bytes,
                  mate_compose_fwd, mate_debug_rms_map, mate_debug_tesa_map, mate_frontend_fwd,
                  mate_frontend_workspace_bytes, mate_gate_norm_fwd, mate_last_error, mate_version, rms_map, tesa,
                  tesa_fwd, tesa_map)
from ._lib import MateError, load

__all__ = ["bissd", "bissd_workspace", "block", "compose", "frontend", "gate_norm", "linear", "mate_bissd_fwd",
           "mate_bissd_workspace_bytes", "mate_compose_fwd", "mate_frontend_fwd", "mate_gate_norm_fwd",
           "mate_frontend_workspace_bytes", "mate_debug_rms_map", "mate_debug_tesa_map", "mate_last_error", "mate_version", "rms_map", "tesa", "tesa_fwd", "tesa_map",
           "MateError", "load"]
