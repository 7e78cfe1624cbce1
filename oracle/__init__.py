"""Python access to the fp64 CPU oracle (``mate_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline use this package; the product path never imports it.

The wrapper marshals arrays only: every step of the computation runs in the
C file, except the MA-branch front-end (Oracle.frontend), written with numpy. Inputs are upcast to float64 exactly (bf16 and fp32 values are
representable in fp64), so the oracle sees the very values the GPU sees.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "mate_oracle.c")
BUILD_DIR = os.path.join(_HERE, "_build")
DEFAULT_LIB = os.path.join(BUILD_DIR, "liboracle.so")

_i32p = ctypes.POINTER(ctypes.c_int32)
_f64p = ctypes.POINTER(ctypes.c_double)
_intp = ctypes.POINTER(ctypes.c_int)


def build(source: str = SOURCE, out: str = DEFAULT_LIB, extra: Sequence[str] = ()) -> str:
    """Compile the oracle into a shared library (gcc, -O2, OpenMP, IEEE fp64)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (os.path.exists(out) and not extra and source == SOURCE
            and os.path.getmtime(out) >= os.path.getmtime(source)):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", *extra, source, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor: exact upcast, then numpy
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


class Oracle:
    """ctypes handle on one build of the oracle library."""

    def __init__(self, lib_path: Optional[str] = None):
        path = lib_path or build()
        self.path = path
        self.lib = ctypes.CDLL(path)
        L = self.lib
        L.oracle_unroll.argtypes = [ctypes.c_int] * 3 + [_intp, _i32p]
        L.oracle_rms_sequence.argtypes = [ctypes.c_int] * 5 + [_i32p]
        L.oracle_avg_pool.argtypes = [_f64p] + [ctypes.c_int] * 7 + [_f64p]
        L.oracle_ssd_scan.argtypes = [ctypes.c_int64] + [ctypes.c_int] * 4 + [_f64p] * 6 + [_f64p]
        L.oracle_bissd.argtypes = [ctypes.c_int] * 8 + [_f64p] * 6 + [ctypes.c_int, _intp, _f64p]
        L.oracle_tesa_window_ids.argtypes = [ctypes.c_int] * 5 + [_intp, _i32p]
        L.oracle_tesa.argtypes = [ctypes.c_int] * 6 + [_f64p] * 3 + [ctypes.c_int] * 2 + [_intp, _f64p]
        L.oracle_compose.argtypes = [ctypes.c_int64] + [ctypes.c_int] * 3 + [_f64p] * 5
        L.oracle_gate_norm.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_double] + [_f64p] * 4
        for f in ("oracle_unroll", "oracle_rms_sequence", "oracle_avg_pool", "oracle_ssd_scan",
                  "oracle_bissd", "oracle_tesa_window_ids", "oracle_tesa", "oracle_compose",
                  "oracle_gate_norm"):
            getattr(L, f).restype = ctypes.c_int

    # ---- Rotary Major Scan -------------------------------------------------
    def unroll(self, T: int, H: int, W: int, priority: Sequence[int]) -> np.ndarray:
        seq = np.empty(T * H * W, dtype=np.int32)
        pr = (ctypes.c_int * 3)(*priority)
        rc = self.lib.oracle_unroll(T, H, W, pr, _ptr(seq, _i32p))
        if rc:
            raise ValueError(f"oracle_unroll rc={rc}")
        return seq

    def rms_sequence(self, T: int, H: int, W: int, mode: int, flip: bool = False) -> np.ndarray:
        seq = np.empty(T * H * W, dtype=np.int32)
        rc = self.lib.oracle_rms_sequence(T, H, W, mode, int(bool(flip)), _ptr(seq, _i32p))
        if rc:
            raise ValueError(f"oracle_rms_sequence rc={rc}")
        return seq

    def avg_pool(self, grid, pool) -> np.ndarray:
        g = _f64(grid)
        T, H, W = g.shape[:3]
        ch = int(np.prod(g.shape[3:])) if g.ndim > 3 else 1
        pt, ph, pw = pool
        out = np.empty((T // pt, H // ph, W // pw) + g.shape[3:], dtype=np.float64)
        rc = self.lib.oracle_avg_pool(_ptr(g, _f64p), T, H, W, ch, pt, ph, pw, _ptr(out, _f64p))
        if rc:
            raise ValueError(f"oracle_avg_pool rc={rc}")
        return out

    # ---- SSD ---------------------------------------------------------------
    def ssd_scan(self, x, dt, A, B, C, D) -> np.ndarray:
        """One-direction scan of an explicit sequence. x: (L, nh, P); dt: (L, nh);
        B, C: (L, G, Ns); A, D: (nh,)."""
        x, dt, A, B, C, D = map(_f64, (x, dt, A, B, C, D))
        L, nh, P = x.shape
        G, Ns = B.shape[1:]
        y = np.empty_like(x)
        rc = self.lib.oracle_ssd_scan(L, nh, P, Ns, G, _ptr(x, _f64p), _ptr(dt, _f64p), _ptr(A, _f64p),
                                      _ptr(B, _f64p), _ptr(C, _f64p), _ptr(D, _f64p), _ptr(y, _f64p))
        if rc:
            raise ValueError(f"oracle_ssd_scan rc={rc}")
        return y

    def bissd(self, x, dt, A, B, C, D, mode: int, pool=None) -> np.ndarray:
        """x: (batch, T, H, W, nh, P); dt: (batch, T, H, W, nh); B, C: (batch, T, H, W, G, Ns)."""
        x, dt, A, B, C, D = map(_f64, (x, dt, A, B, C, D))
        b, T, H, W, nh, P = x.shape
        G, Ns = B.shape[4:]
        out = np.empty_like(x)
        pl = (ctypes.c_int * 3)(*(pool if pool else (0, 0, 0)))
        rc = self.lib.oracle_bissd(b, T, H, W, nh, P, Ns, G, _ptr(x, _f64p), _ptr(dt, _f64p), _ptr(A, _f64p),
                                   _ptr(B, _f64p), _ptr(C, _f64p), _ptr(D, _f64p), mode, pl, _ptr(out, _f64p))
        if rc:
            raise ValueError(f"oracle_bissd rc={rc}")
        return out

    # ---- TESA --------------------------------------------------------------
    def tesa_window_ids(self, T: int, H: int, W: int, Tw: int, Sw: int, shift) -> np.ndarray:
        win = np.empty(T * H * W, dtype=np.int32)
        sh = (ctypes.c_int * 3)(*shift)
        rc = self.lib.oracle_tesa_window_ids(T, H, W, Tw, Sw, sh, _ptr(win, _i32p))
        if rc < 0:
            raise ValueError(f"oracle_tesa_window_ids rc={rc}")
        return win

    def tesa(self, q, k, v, Tw: int, Sw: int, shift) -> np.ndarray:
        q, k, v = map(_f64, (q, k, v))
        b, T, H, W, nh, d = q.shape
        out = np.empty_like(q)
        sh = (ctypes.c_int * 3)(*shift)
        rc = self.lib.oracle_tesa(b, T, H, W, nh, d, _ptr(q, _f64p), _ptr(k, _f64p), _ptr(v, _f64p),
                                  Tw, Sw, sh, _ptr(out, _f64p))
        if rc < 0:
            raise ValueError(f"oracle_tesa rc={rc}")
        return out


    # ---- MATE composition --------------------------------------------------
    def compose(self, y_ma, y_te, w_ma, w_te) -> np.ndarray:
        """out = y_ma w_ma^T + y_te w_te^T. y_ma: (..., K1), y_te: (..., K2) over the same
        leading shape; w_ma: (N, K1), w_te: (N, K2). Returns (..., N)."""
        y1, y2, w1, w2 = map(_f64, (y_ma, y_te, w_ma, w_te))
        lead = y1.shape[:-1]
        K1, K2, N = y1.shape[-1], y2.shape[-1], w1.shape[0]
        M = int(np.prod(lead)) if lead else 1
        y1 = np.ascontiguousarray(y1.reshape(M, K1))
        y2 = np.ascontiguousarray(y2.reshape(M, K2))
        out = np.empty((M, N), dtype=np.float64)
        rc = self.lib.oracle_compose(M, K1, K2, N, _ptr(y1, _f64p), _ptr(y2, _f64p), _ptr(w1, _f64p),
                                     _ptr(w2, _f64p), _ptr(out, _f64p))
        if rc:
            raise ValueError(f"oracle_compose rc={rc}")
        return out.reshape(*lead, N)


    def gate_norm(self, y, z, w, group: int, eps: float) -> np.ndarray:
        """Gated RMS norm of the MA-branch output (reading R9): v = y SiLU(z), each group of
        `group` channels divided by sqrt(mean(v^2) + eps), times w. y, z: (..., C); w: (C,).
        Returns (..., C)."""
        y, z, w = map(_f64, (y, z, w))
        lead, C = y.shape[:-1], y.shape[-1]
        M = int(np.prod(lead)) if lead else 1
        y = np.ascontiguousarray(y.reshape(M, C))
        z = np.ascontiguousarray(z.reshape(M, C))
        out = np.empty((M, C), dtype=np.float64)
        rc = self.lib.oracle_gate_norm(M, C, group, ctypes.c_double(eps), _ptr(y, _f64p), _ptr(z, _f64p),
                                       _ptr(np.ascontiguousarray(w), _f64p), _ptr(out, _f64p))
        if rc:
            raise ValueError(f"oracle_gate_norm rc={rc}")
        return out.reshape(*lead, C)

    # ---- MA-branch front-end ------------------------------------------------
    def frontend(self, u, w_in, conv_w, conv_b, dt_bias, mode: int, nheads: int, headdim: int, ngroups: int,
                 dstate: int, positions=None):
        """The standard Mamba2 input side ([Review] section 三, MA-Branch item 1, bidirectional
        Mamba2; the pages give no more of the block; reading R8 of the C oracle's header):
            [z | xBC_pre | dt_raw] = u w_in^T
            xBC[n] = SiLU(conv_b + sum_{k=0..3} conv_w[:, k] xBC_pre[n - 3 + k])   along the scan
                     order of `mode` (positions before 0 are zero)
            dt = softplus(dt_raw + dt_bias)
        u: (batch, T, H, W, d_model). Returns z, x, dt, B, C in grid order, shaped as the SSD takes
        them. With `positions` (scan positions), only those tokens are produced, as arrays
        (batch, len(positions), ...) in the order given: the projection is then taken of those
        tokens and their three predecessors only."""
        u, w, cw, cb, db = map(_f64, (u, w_in, conv_w, conv_b, dt_bias))
        b, T, H, W, dm = u.shape
        N = T * H * W
        d_inner, gns = nheads * headdim, ngroups * dstate
        dc = d_inner + 2 * gns
        order = self.rms_sequence(T, H, W, mode).astype(np.int64)   # scan position -> grid offset
        flat = u.reshape(b, N, dm)
        if positions is None:
            pos = np.arange(N)
        else:
            pos = np.asarray(positions, dtype=np.int64)
        # the tokens needed: each output position and its three predecessors in scan order
        need = np.unique(np.concatenate([pos - k for k in range(4)]))
        need = need[need >= 0]
        proj = flat[:, order[need], :] @ w.T                  # (b, len(need), d_inner + dc + nheads)
        at = {int(p): i for i, p in enumerate(need)}
        def pre(p):  # xBC_pre at scan position p (zero before the sequence)
            return proj[:, at[p], d_inner:d_inner + dc] if p >= 0 else np.zeros((b, dc))
        conv = np.empty((b, len(pos), dc))
        for j, p in enumerate(pos):
            acc = cb.copy()[None, :].repeat(b, axis=0)
            for k in range(4):
                acc = acc + cw[:, k][None, :] * pre(int(p) - 3 + k)
            conv[:, j] = acc
        act = conv / (1.0 + np.exp(-conv))                    # SiLU
        rows = np.array([at[int(p)] for p in pos])
        z = proj[:, rows, :d_inner]
        dt = np.logaddexp(0.0, proj[:, rows, d_inner + dc:] + db[None, None, :])  # softplus
        x, Bm, Cm = act[..., :d_inner], act[..., d_inner:d_inner + gns], act[..., d_inner + gns:]
        if positions is not None:
            return (z, x.reshape(b, -1, nheads, headdim), dt, Bm.reshape(b, -1, ngroups, dstate),
                    Cm.reshape(b, -1, ngroups, dstate))
        # scatter the scan-ordered results back to grid order
        def grid(a):
            g = np.empty_like(a)
            g[:, order] = a
            return g
        shp = (b, T, H, W)
        return (grid(z).reshape(*shp, d_inner), grid(x).reshape(*shp, nheads, headdim), grid(dt).reshape(*shp, nheads),
                grid(Bm).reshape(*shp, ngroups, dstate), grid(Cm).reshape(*shp, ngroups, dstate))


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle built from the committed source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
