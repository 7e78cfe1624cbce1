"""Thin PyTorch-facing binding of the C ABI in include/mate.h.

Each function marshals torch CUDA tensors into the pointers and sizes of the
C entry point of the same name and raises ``MateError`` on a non-zero status.
PyTorch supplies device memory and the current stream; every step of the
computation runs in libmate.so. The ``bissd`` / ``tesa`` helpers read the
dims off the tensor shapes and allocate the output and workspace with torch.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import torch

from . import _lib
from ._lib import (MATE_BF16, MATE_DIR_BI, MATE_F32, check, mate_attn_dims, mate_compose_dims, mate_frontend_dims,
                   mate_gate_norm_dims, mate_ssd_dims)

_DT = {torch.float32: MATE_F32, torch.bfloat16: MATE_BF16}


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor]) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    return ctypes.c_void_p(t.data_ptr())


def _int3(v: Optional[Sequence[int]]):
    if v is None:
        return None
    return (ctypes.c_int * 3)(*[int(u) for u in v])


def _require(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def ssd_dims(batch, nheads, headdim, dstate, ngroups, chunk, dtype, directions=MATE_DIR_BI) -> mate_ssd_dims:
    return mate_ssd_dims(batch, nheads, headdim, dstate, ngroups, chunk,
                         _DT[dtype] if isinstance(dtype, torch.dtype) else int(dtype), directions)


def attn_dims(batch, nheads, headdim, dtype) -> mate_attn_dims:
    return mate_attn_dims(batch, nheads, headdim, _DT[dtype] if isinstance(dtype, torch.dtype) else int(dtype))


# ---------------------------------------------------------------------------
# the C entry points, one to one
# ---------------------------------------------------------------------------
def mate_bissd_workspace_bytes(T: int, H: int, W: int, review_pool, dims: mate_ssd_dims) -> int:
    return int(_lib.load().mate_bissd_workspace_bytes(T, H, W, _int3(review_pool), ctypes.byref(dims)))


def mate_bissd_fwd(x, dt, A, B, C, D, T, H, W, scan_mode, review_pool, out, dims: mate_ssd_dims,
                   workspace: torch.Tensor, stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = _lib.load().mate_bissd_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), T, H, W, scan_mode,
                                    _int3(review_pool), _ptr(out), ctypes.byref(dims), _ptr(workspace),
                                    ctypes.c_size_t(ws_bytes), _stream_handle(stream))
    check("mate_bissd_fwd", rc)


def mate_bissd_fwd_noalloc(x, dt, A, B, C, D, T, H, W, scan_mode, review_pool, out, dims: mate_ssd_dims,
                           stream=None) -> None:
    """mate_bissd_fwd with the library's fixed scratch array instead of a caller workspace."""
    rc = _lib.load().mate_bissd_fwd_noalloc(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), T, H, W,
                                            scan_mode, _int3(review_pool), _ptr(out), ctypes.byref(dims),
                                            _stream_handle(stream))
    check("mate_bissd_fwd_noalloc", rc)


def tesa_fwd(q, k, v, T, H, W, Tw, Sw, shift, out, dims: mate_attn_dims, stream=None) -> None:
    rc = _lib.load().tesa_fwd(_ptr(q), _ptr(k), _ptr(v), T, H, W, Tw, Sw, _int3(shift), _ptr(out),
                              ctypes.byref(dims), _stream_handle(stream))
    check("tesa_fwd", rc)


def mate_compose_fwd(y_ma, y_te, w_ma, w_te, out, dims: mate_compose_dims, stream=None) -> None:
    rc = _lib.load().mate_compose_fwd(_ptr(y_ma), _ptr(y_te), _ptr(w_ma), _ptr(w_te), _ptr(out), ctypes.byref(dims),
                                      _stream_handle(stream))
    check("mate_compose_fwd", rc)


def mate_gate_norm_fwd(y, z, w, eps: float, out, dims: mate_gate_norm_dims, stream=None) -> None:
    rc = _lib.load().mate_gate_norm_fwd(_ptr(y), _ptr(z), _ptr(w), float(eps), _ptr(out), ctypes.byref(dims),
                                        _stream_handle(stream))
    check("mate_gate_norm_fwd", rc)


def mate_debug_rms_map(T, H, W, scan_mode, flip, out, stream=None) -> None:
    check("mate_debug_rms_map",
          _lib.load().mate_debug_rms_map(T, H, W, scan_mode, int(flip), _ptr(out), _stream_handle(stream)))


def mate_debug_tesa_map(T, H, W, Tw, Sw, shift, out, stream=None) -> None:
    check("mate_debug_tesa_map",
          _lib.load().mate_debug_tesa_map(T, H, W, Tw, Sw, _int3(shift), _ptr(out), _stream_handle(stream)))


def mate_last_error(stream=None) -> int:
    return int(_lib.load().mate_last_error(_stream_handle(stream)))


def mate_version() -> int:
    return int(_lib.load().mate_version())


# ---------------------------------------------------------------------------
# shape-reading helpers
# ---------------------------------------------------------------------------
def bissd_workspace(x: torch.Tensor, B: torch.Tensor, review_pool=None, chunk: int = 256,
                    directions: int = MATE_DIR_BI) -> torch.Tensor:
    b, T, H, W, nh, P = x.shape
    G, Ns = B.shape[4:]
    dims = ssd_dims(b, nh, P, Ns, G, chunk, x.dtype, directions)
    n = mate_bissd_workspace_bytes(T, H, W, review_pool, dims)
    if n == 0:
        raise ValueError("unsupported bi-SSD dims")
    return torch.empty(n, dtype=torch.uint8, device=x.device)


def bissd(x, dt, A, B, C, D, scan_mode: int, review_pool=None, chunk: int = 256, directions: int = MATE_DIR_BI,
          out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """MA-branch token mix. x: (batch, T, H, W, nh, P); dt: (batch, T, H, W, nh) fp32;
    A, D: (nh,) fp32; B, C: (batch, T, H, W, G, Ns). Returns out shaped like x."""
    for t, n in ((x, "x"), (B, "B"), (C, "C")):
        _require(t, n, x.dtype)
    for t, n in ((dt, "dt"), (A, "A"), (D, "D")):
        _require(t, n, torch.float32)
    b, T, H, W, nh, P = x.shape
    G, Ns = B.shape[4:]
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = bissd_workspace(x, B, review_pool, chunk, directions)
    dims = ssd_dims(b, nh, P, Ns, G, chunk, x.dtype, directions)
    mate_bissd_fwd(x, dt, A, B, C, D, T, H, W, scan_mode, review_pool, out, dims, workspace, stream)
    return out


def tesa(q, k, v, Tw: int, Sw: int, shift=(0, 0, 0), out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """TE-branch window attention. q, k, v: (batch, T, H, W, nh, d). Returns out shaped like q."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n, q.dtype)
    b, T, H, W, nh, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    tesa_fwd(q, k, v, T, H, W, Tw, Sw, shift, out, attn_dims(b, nh, d, q.dtype), stream)
    return out


def compose(y_ma, y_te, w_ma, w_te, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """MATE composition: out = y_ma w_ma^T + y_te w_te^T (bf16). y_ma: (..., k_ma), the bi-SSD
    output with its heads flattened; y_te: (..., k_te), the TESA output likewise; w_ma: (d_model,
    k_ma), w_te: (d_model, k_te). Returns (..., d_model)."""
    for t, n in ((y_ma, "y_ma"), (y_te, "y_te"), (w_ma, "w_ma"), (w_te, "w_te")):
        _require(t, n, torch.bfloat16)
    lead = y_ma.shape[:-1]
    if y_te.shape[:-1] != lead:
        raise ValueError("y_ma and y_te must cover the same tokens")
    M = 1
    for s in lead:
        M *= int(s)
    N = int(w_ma.shape[0])
    if out is None:
        out = torch.empty(*lead, N, dtype=torch.bfloat16, device=y_ma.device)
    dims = mate_compose_dims(M, int(y_ma.shape[-1]), int(y_te.shape[-1]), N, MATE_BF16)
    mate_compose_fwd(y_ma, y_te, w_ma, w_te, out, dims, stream)
    return out


def gate_norm(y, z, w, group: int, eps: float = 1e-5, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """MA-branch output side: out = y SiLU(z) / sqrt(mean over each group of `group` channels
    of (y SiLU(z))^2 + eps) * w (bf16). y: (..., C), the bi-SSD output with its heads flattened;
    z: (..., C), the front-end's z; w: (C,) fp32. Returns (..., C)."""
    _require(y, "y", torch.bfloat16)
    _require(z, "z", torch.bfloat16)
    _require(w, "w", torch.float32)
    if z.shape != y.shape or w.shape != (y.shape[-1],):
        raise ValueError("y and z must have one shape and w one entry per channel")
    M = 1
    for s in y.shape[:-1]:
        M *= int(s)
    if out is None:
        out = torch.empty_like(y)
    dims = mate_gate_norm_dims(M, int(y.shape[-1]), int(group), MATE_BF16)
    mate_gate_norm_fwd(y, z, w, eps, out, dims, stream)
    return out


def linear(x, w, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """x w^T on the tensor cores (bf16): the composition GEMM with one input part.
    x: (..., K); w: (N, K) in the nn.Linear layout. Returns (..., N)."""
    _require(x, "x", torch.bfloat16)
    _require(w, "w", torch.bfloat16)
    M = 1
    for s in x.shape[:-1]:
        M *= int(s)
    N = int(w.shape[0])
    if out is None:
        out = torch.empty(*x.shape[:-1], N, dtype=torch.bfloat16, device=x.device)
    mate_compose_fwd(x, None, w, None, out, mate_compose_dims(M, int(x.shape[-1]), 0, N, MATE_BF16), stream)
    return out


def block(u, weights, *, scan_mode: int, review_pool, chunk: int, nheads: int, headdim: int, ngroups: int,
          dstate: int, attn_heads: int, attn_dim: int, Tw: int, Sw: int, shift, eps: float = 1e-5, stream=None,
          keep: bool = False):
    """One MATE token mixer, every step in the library's kernels. u: (batch, T, H, W, d_model) bf16.
        MA-branch: z, x, dt, B, C = front-end(u); y = bi-SSD(x, dt, A, B, C, D) in the RMS order
                   `scan_mode` with review tokens; y_ma = gated norm(y, z)
        TE-branch: q, k, v = u w_q^T, u w_k^T, u w_v^T; y_te = TESA(q, k, v)
        out = y_ma w_ma^T + y_te w_te^T
    weights: w_in, conv_w, conv_b, dt_bias, A, D, norm_w, w_q, w_k, w_v, w_ma, w_te (as
    workloads.generate_block draws them). Returns out (batch, T, H, W, d_model), and with
    `keep` also a dict of the intermediate tensors."""
    w = weights
    b, T, H, W, _ = u.shape
    z, x, dt, B, C = frontend(u, w["w_in"], w["conv_w"], w["conv_b"], w["dt_bias"], scan_mode, nheads, headdim,
                              ngroups, dstate, stream=stream)
    y = bissd(x, dt, w["A"], B, C, w["D"], scan_mode, review_pool, chunk=chunk, stream=stream)
    d_inner = nheads * headdim
    y_ma = gate_norm(y.view(b, T, H, W, d_inner), z, w["norm_w"], d_inner // ngroups, eps, stream=stream)
    q, k, v = (linear(u, w[n], stream=stream).view(b, T, H, W, attn_heads, attn_dim) for n in ("w_q", "w_k", "w_v"))
    y_te = tesa(q, k, v, Tw, Sw, shift, stream=stream)
    out = compose(y_ma, y_te.view(b, T, H, W, attn_heads * attn_dim), w["w_ma"], w["w_te"], stream=stream)
    if keep:
        return out, dict(z=z, x=x, dt=dt, B=B, C=C, y=y, y_ma=y_ma, q=q, k=k, v=v, y_te=y_te)
    return out


def mate_frontend_workspace_bytes(T: int, H: int, W: int, dims: mate_frontend_dims) -> int:
    return int(_lib.load().mate_frontend_workspace_bytes(T, H, W, ctypes.byref(dims)))


def mate_frontend_fwd(u, w_in, conv_w, conv_b, dt_bias, T, H, W, scan_mode, z, x, dt, B, C,
                      dims: mate_frontend_dims, workspace, stream=None) -> None:
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = _lib.load().mate_frontend_fwd(_ptr(u), _ptr(w_in), _ptr(conv_w), _ptr(conv_b), _ptr(dt_bias), T, H, W,
                                       scan_mode, _ptr(z), _ptr(x), _ptr(dt), _ptr(B), _ptr(C), ctypes.byref(dims),
                                       _ptr(workspace), nbytes, _stream_handle(stream))
    check("mate_frontend_fwd", rc)


def frontend(u, w_in, conv_w, conv_b, dt_bias, scan_mode: int, nheads: int, headdim: int, ngroups: int, dstate: int,
             stream=None):
    """MA-branch front-end. u: (batch, T, H, W, d_model) bf16; w_in: (d_inner + dc + nheads, d_model)
    bf16; conv_w: (dc, 4), conv_b: (dc), dt_bias: (nheads) fp32. Returns z, x, dt, B, C shaped as
    mate_bissd_fwd and the gate take them."""
    _require(u, "u", torch.bfloat16)
    _require(w_in, "w_in", torch.bfloat16)
    for t, n in ((conv_w, "conv_w"), (conv_b, "conv_b"), (dt_bias, "dt_bias")):
        _require(t, n, torch.float32)
    b, T, H, W, dm = u.shape
    dims = mate_frontend_dims(b, dm, nheads, headdim, ngroups, dstate, MATE_BF16)
    nbytes = mate_frontend_workspace_bytes(T, H, W, dims)
    if nbytes == 0:
        raise ValueError("unsupported front-end dims")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=u.device)
    kw = dict(dtype=torch.bfloat16, device=u.device)
    z = torch.empty(b, T, H, W, nheads * headdim, **kw)
    x = torch.empty(b, T, H, W, nheads, headdim, **kw)
    dt = torch.empty(b, T, H, W, nheads, dtype=torch.float32, device=u.device)
    Bm = torch.empty(b, T, H, W, ngroups, dstate, **kw)
    Cm = torch.empty(b, T, H, W, ngroups, dstate, **kw)
    mate_frontend_fwd(u, w_in, conv_w, conv_b, dt_bias, T, H, W, scan_mode, z, x, dt, Bm, Cm, dims, ws, stream)
    return z, x, dt, Bm, Cm


def rms_map(T: int, H: int, W: int, scan_mode: int, flip: bool = False, device="cuda") -> torch.Tensor:
    out = torch.empty(T * H * W, dtype=torch.int32, device=device)
    mate_debug_rms_map(T, H, W, scan_mode, flip, out)
    return out


def tesa_map(T: int, H: int, W: int, Tw: int, Sw: int, shift, device="cuda") -> torch.Tensor:
    out = torch.empty(T * H * W, dtype=torch.int32, device=device)
    mate_debug_tesa_map(T, H, W, Tw, Sw, shift, out)
    return out
