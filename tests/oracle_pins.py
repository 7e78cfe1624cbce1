"""Pins that tie the fp64 oracle to something other than itself.

Each pin takes an ``oracle.Oracle`` handle and raises AssertionError when the
oracle disagrees with a fact fixed by the pages or by mathematics:
hand-written golden fixtures (tests/golden, each with its citation), closed
forms, the quadratic "dual" forms of the scan written independently here
with numpy, textbook softmax attention, and invariants. The mutant test
builds deliberately broken copies of the oracle and checks that every
mutant trips at least one pin.
"""
from __future__ import annotations

import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
MODE_CODE = {"SR": 0, "SC": 1, "TR": 2, "TC": 3}


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------------------
# independent restatements used by the pins (numpy, written from the
# definitions, not from the oracle's C code)
# ---------------------------------------------------------------------------
def scan_order_by_transpose(T, H, W, mode):
    """Scan order by moving the axes into priority order (slowest first) and
    flattening; returns seq[n] = grid offset."""
    g = np.arange(T * H * W).reshape(T, H, W)
    perm = {0: (0, 1, 2), 1: (0, 2, 1), 2: (1, 2, 0), 3: (2, 1, 0)}[mode]
    return np.ascontiguousarray(g.transpose(perm)).reshape(-1)


def dual_forward(x, dt, A, B, C, D):
    """Causal quadratic form of one scan direction:
    y_i = sum_{j<=i} (C_i . B_j) exp(A sum_{k=j+1..i} dt_k) dt_j x_j + D x_i.
    x: (L, nh, P); dt: (L, nh); B, C: (L, G, Ns)."""
    L, nh, P = x.shape
    G = B.shape[1]
    y = np.zeros_like(x)
    for h in range(nh):
        g = h // (nh // G)
        cs = np.concatenate([[0.0], np.cumsum(dt[:, h])])  # cs[i+1] = sum_{k<=i} dt_k
        S = C[:, g, :] @ B[:, g, :].T                         # S[i, j] = C_i . B_j
        seg = cs[1:, None] - cs[None, 1:]                    # sum_{k=j+1..i} dt_k
        low = np.tril(np.ones((L, L), bool))
        Lmat = np.where(low, np.exp(A[h] * np.where(low, seg, 0.0)), 0.0)
        M = S * Lmat * dt[None, :, h]
        y[:, h, :] = M @ x[:, h, :] + D[h] * x[:, h, :]
    return y


def dual_backward(x, dt, A, B, C, D):
    """Anti-causal quadratic form of the flipped direction, in original order:
    y_i = sum_{j>=i} (C_i . B_j) exp(A sum_{k=i..j-1} dt_k) dt_j x_j + D x_i."""
    L, nh, P = x.shape
    G = B.shape[1]
    y = np.zeros_like(x)
    for h in range(nh):
        g = h // (nh // G)
        cs = np.concatenate([[0.0], np.cumsum(dt[:, h])])   # cs[i] = sum_{k<i} dt_k
        S = C[:, g, :] @ B[:, g, :].T
        seg = cs[None, :-1] - cs[:-1, None]                   # [i, j] -> sum_{k=i..j-1} dt_k
        U = np.triu(np.ones((L, L), bool))
        Lmat = np.where(U, np.exp(A[h] * np.where(U, seg, 0.0)), 0.0)
        M = S * Lmat * dt[None, :, h]
        y[:, h, :] = M @ x[:, h, :] + D[h] * x[:, h, :]
    return y


def window_index(c, S, s):
    """Window number along one axis when boundaries sit at coordinates = s (mod S)."""
    return (c + (S - s) % S) // S


def block_mask_attention(q, k, v, Tw, Sw, shift):
    """Full attention over the whole grid with a block mask that keeps only
    pairs in the same window. q, k, v: (T, H, W, nh, d)."""
    T, H, W, nh, d = q.shape
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    nht = window_index(H - 1, Sw, shift[1]) + 1
    nwt = window_index(W - 1, Sw, shift[2]) + 1
    wid = ((window_index(t, Tw, shift[0]) * nht + window_index(h, Sw, shift[1])) * nwt
           + window_index(w, Sw, shift[2])).reshape(-1)
    same = wid[:, None] == wid[None, :]
    Q = q.reshape(-1, nh, d)
    K = k.reshape(-1, nh, d)
    V = v.reshape(-1, nh, d)
    out = np.empty_like(Q)
    for hd in range(nh):
        s = Q[:, hd] @ K[:, hd].T / np.sqrt(d)
        s = np.where(same, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, hd] = p @ V[:, hd]
    return out.reshape(q.shape)


def _rng(seed):
    return np.random.default_rng(seed)


def _ssd_inputs(rng, L, nh, P, Ns, G, a_scale=1.0):
    x = rng.standard_normal((L, nh, P))
    dt = np.log1p(np.exp(rng.standard_normal((L, nh)) - 2.0))
    A = -np.exp(rng.uniform(0, np.log(4.0), nh)) * a_scale
    B = rng.standard_normal((L, G, Ns)) / np.sqrt(Ns)
    C = rng.standard_normal((L, G, Ns)) / np.sqrt(Ns)
    D = rng.standard_normal(nh)
    return x, dt, A, B, C, D


def _grid_inputs(rng, T, H, W, nh, P, Ns, G, batch=1):
    x = rng.standard_normal((batch, T, H, W, nh, P))
    dt = np.log1p(np.exp(rng.standard_normal((batch, T, H, W, nh)) - 2.0))
    A = -np.exp(rng.uniform(0, np.log(4.0), nh))
    B = rng.standard_normal((batch, T, H, W, G, Ns)) / np.sqrt(Ns)
    C = rng.standard_normal((batch, T, H, W, G, Ns)) / np.sqrt(Ns)
    D = rng.standard_normal(nh)
    return x, dt, A, B, C, D


def _close(a, b, tol=1e-10, what=""):
    a = np.asarray(a)
    b = np.asarray(b)
    err = np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)
    assert err <= tol, f"{what}: relative max error {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------------------
# Rotary Major Scan
# ---------------------------------------------------------------------------
def pin_rms_golden(o):
    for row in _read_golden("rms_T2_H2_W3.txt"):
        mode = MODE_CODE[row[0]]
        want = np.array([int(v) for v in row[1:]])
        got = o.rms_sequence(2, 2, 3, mode)
        assert np.array_equal(got, want), f"mode {row[0]}: {got} != {want}"


def pin_rms_flip_golden(o):
    seq = o.rms_sequence(2, 2, 3, 0)
    flipped = o.rms_sequence(2, 2, 3, 0, flip=True)
    for n_l, n_flip in _read_golden("flip_N12.txt"):
        assert flipped[int(n_flip)] == seq[int(n_l) - 1]


def pin_rms_properties(o):
    for (T, H, W) in [(3, 4, 5), (1, 7, 2), (4, 4, 4), (2, 6, 3)]:
        N = T * H * W
        for mode in range(4):
            seq = o.rms_sequence(T, H, W, mode)
            assert np.array_equal(np.sort(seq), np.arange(N)), "not a bijection"
            assert np.array_equal(seq, scan_order_by_transpose(T, H, W, mode)), f"mode {mode} order"
            fl = o.rms_sequence(T, H, W, mode, flip=True)
            assert np.array_equal(fl, seq[::-1]), "flip is not n -> N-1-n"
        assert np.array_equal(o.rms_sequence(T, H, W, 0), np.arange(N)), "SR is not the identity"
    # spatial-column on a square frame is the per-frame transpose
    T, S = 3, 4
    g = np.arange(T * S * S).reshape(T, S, S)
    assert np.array_equal(o.rms_sequence(T, S, S, 1), g.transpose(0, 2, 1).reshape(-1))


# ---------------------------------------------------------------------------
# pooling
# ---------------------------------------------------------------------------
def pin_pool(o):
    rng = _rng(1)
    g = rng.standard_normal((4, 6, 8, 3))
    got = o.avg_pool(g, (2, 3, 4))
    want = g.reshape(2, 2, 2, 3, 2, 4, 3).mean(axis=(1, 3, 5))
    _close(got, want, 1e-14, "pool vs reshape-mean")
    c = np.full((4, 6, 8, 2), 3.25)
    _close(o.avg_pool(c, (4, 2, 8)), np.full((1, 3, 1, 2), 3.25), 1e-15, "pool of a constant")
    _close(o.avg_pool(g, (1, 1, 1)), g, 0.0, "pool {1,1,1}")


# ---------------------------------------------------------------------------
# one-direction scan
# ---------------------------------------------------------------------------
def pin_scan_dual(o):
    rng = _rng(2)
    for (L, nh, P, Ns, G) in [(13, 3, 4, 5, 1), (9, 4, 3, 2, 2), (1, 2, 2, 3, 1)]:
        x, dt, A, B, C, D = _ssd_inputs(rng, L, nh, P, Ns, G)
        _close(o.ssd_scan(x, dt, A, B, C, D), dual_forward(x, dt, A, B, C, D), 1e-11, "scan vs dual")


def pin_scan_closed_forms(o):
    rng = _rng(3)
    L, nh, P, Ns = 11, 2, 3, 4
    x, dt, A, B, C, D = _ssd_inputs(rng, L, nh, P, Ns, 1)
    # A = 0, dt = 1: linear attention, y_i = C_i . sum_{j<=i} B_j x_j^T + D x_i
    ones = np.ones_like(dt)
    zeros = np.zeros_like(A)
    y = o.ssd_scan(x, ones, zeros, B, C, D)
    kv = np.cumsum(B[:, 0, :, None, None] * x[:, None, :, :], axis=0)  # kv[i,n,h,p] = sum_{j<=i} B_j[n] x_j[h,p]
    want = np.einsum("in,inhp->ihp", C[:, 0, :], kv) + D[None, :, None] * x
    _close(y, want, 1e-12, "linear-attention closed form")
    # dt*A -> -inf: only the diagonal survives, y_i = dt_i (C_i . B_i) x_i + D x_i
    Abig = np.full(nh, -1e6)
    y = o.ssd_scan(x, dt, Abig, B, C, D)
    cb = np.sum(C[:, 0, :] * B[:, 0, :], axis=1)
    want = dt[:, :, None] * cb[:, None, None] * x + D[None, :, None] * x
    _close(y, want, 1e-12, "diagonal-only closed form")
    # a single token: y = dt (C . B) x + D x
    y = o.ssd_scan(x[:1], dt[:1], A, B[:1], C[:1], D)
    _close(y, dt[:1, :, None] * cb[:1, None, None] * x[:1] + D[None, :, None] * x[:1], 1e-13, "L = 1")


# ---------------------------------------------------------------------------
# bidirectional scan in RMS order, with and without review tokens
# ---------------------------------------------------------------------------
def _seq_of(a, order):
    """Grid tensor (T, H, W, ...) -> sequence (N, ...) in the given order."""
    return a.reshape((-1,) + a.shape[3:])[order]


def pin_bissd_dual(o):
    rng = _rng(4)
    T, H, W, nh, P, Ns = 2, 3, 4, 2, 3, 4
    x, dt, A, B, C, D = _grid_inputs(rng, T, H, W, nh, P, Ns, 1, batch=2)
    for mode in range(4):
        out = o.bissd(x, dt, A, B, C, D, mode)
        order = scan_order_by_transpose(T, H, W, mode)
        for b in range(2):
            xs, ds, Bs, Cs = (_seq_of(a[b], order) for a in (x, dt, B, C))
            y = dual_forward(xs, ds, A, Bs, Cs, D) + dual_backward(xs, ds, A, Bs, Cs, D)
            want = np.empty_like(y)
            want[order] = y
            _close(out[b].reshape(y.shape), want, 1e-11, f"bissd mode {mode} vs duals")


def pin_bissd_flip_equivariance(o):
    rng = _rng(5)
    x, dt, A, B, C, D = _grid_inputs(rng, 3, 2, 4, 2, 2, 3, 1)
    rev = lambda a: a[:, ::-1, ::-1, ::-1].copy()  # reversing every axis flips every scan
    for mode in range(4):
        y = o.bissd(x, dt, A, B, C, D, mode)
        yr = o.bissd(rev(x), rev(dt), A, rev(B), rev(C), D, mode)
        _close(yr, rev(y), 1e-12, f"bi(flip) = flip(bi), mode {mode}")


def pin_bissd_review(o):
    rng = _rng(6)
    T, H, W, nh, P, Ns = 4, 4, 6, 2, 3, 4
    pool = (2, 2, 3)
    x, dt, A, B, C, D = _grid_inputs(rng, T, H, W, nh, P, Ns, 1)
    Tp, Hp, Wp = T // 2, H // 2, W // 3

    def pooled(a):
        s = a[0].shape[3:]
        return a[0].reshape((Tp, 2, Hp, 2, Wp, 3) + s).mean(axis=(1, 3, 5))

    for mode in range(4):
        out = o.bissd(x, dt, A, B, C, D, mode, pool)
        order = scan_order_by_transpose(T, H, W, mode)
        porder = scan_order_by_transpose(Tp, Hp, Wp, mode)
        Xs = [_seq_of(a[0], order) for a in (x, dt, B, C)]
        Rs = [_seq_of(pooled(a), porder) for a in (x, dt, B, C)]
        pre = [np.concatenate([r, r[::-1]]) for r in Rs]
        Lp = pre[0].shape[0]
        fwd = dual_forward(*[np.concatenate([p_, s_]) for p_, s_ in zip(pre[:2], Xs[:2])], A,
                           *[np.concatenate([p_, s_]) for p_, s_ in zip(pre[2:], Xs[2:])], D)[Lp:]
        bwd = dual_forward(*[np.concatenate([p_, s_[::-1]]) for p_, s_ in zip(pre[:2], Xs[:2])], A,
                           *[np.concatenate([p_, s_[::-1]]) for p_, s_ in zip(pre[2:], Xs[2:])], D)[Lp:][::-1]
        want = np.empty_like(fwd)
        want[order] = fwd + bwd
        _close(out[0].reshape(want.shape), want, 1e-11, f"review prefix, mode {mode}")
    # pool {1,1,1}: R is the scan sequence itself
    out1 = o.bissd(x, dt, A, B, C, D, 2, (1, 1, 1))
    order = scan_order_by_transpose(T, H, W, 2)
    Xs = [_seq_of(a[0], order) for a in (x, dt, B, C)]
    fwd = dual_forward(*(np.concatenate([s_, s_[::-1], s_]) for s_ in Xs[:2]), A,
                       *(np.concatenate([s_, s_[::-1], s_]) for s_ in Xs[2:]), D)[2 * len(order):]
    bwd = dual_forward(*(np.concatenate([s_, s_[::-1], s_[::-1]]) for s_ in Xs[:2]), A,
                       *(np.concatenate([s_, s_[::-1], s_[::-1]]) for s_ in Xs[2:]), D)[2 * len(order):][::-1]
    want = np.empty_like(fwd)
    want[order] = fwd + bwd
    _close(out1[0].reshape(want.shape), want, 1e-11, "pool {1,1,1}")


# ---------------------------------------------------------------------------
# TESA
# ---------------------------------------------------------------------------
def pin_tesa_golden(o):
    rows = _read_golden("tesa_windows_T4_H5_W6_Tw3_Sw4_shift1_1_3.txt")
    want = np.zeros((4, 5, 6), dtype=np.int64)
    for r in rows:
        t, h = int(r[0]), int(r[1])
        want[t, h] = [int(v) for v in r[2:]]
    got = o.tesa_window_ids(4, 5, 6, 3, 4, (1, 1, 3)).reshape(4, 5, 6)
    assert np.array_equal(got, want), "TESA window partition differs from the hand-written fixture"


def pin_tesa_tiling(o):
    for (T, H, W, Tw, Sw, sh) in [(4, 8, 8, 2, 4, (1, 2, 2)), (5, 7, 9, 2, 4, (1, 3, 1)), (3, 4, 4, 3, 4, (0, 0, 0))]:
        wid = o.tesa_window_ids(T, H, W, Tw, Sw, sh)
        n = wid.max() + 1
        counts = np.bincount(wid, minlength=n)
        assert counts.sum() == T * H * W and (counts > 0).all(), "windows do not tile the grid once"
        nt = len(set(window_index(np.arange(T), Tw, sh[0])))
        nh = len(set(window_index(np.arange(H), Sw, sh[1])))
        nw = len(set(window_index(np.arange(W), Sw, sh[2])))
        assert n == nt * nh * nw, "window count"
        assert counts.max() <= Tw * Sw * Sw, "a window is larger than Tw x Sw x Sw"


def pin_tesa_block_mask(o):
    rng = _rng(7)
    for (T, H, W, Tw, Sw, sh) in [(4, 8, 8, 2, 4, (1, 2, 2)), (3, 5, 6, 2, 4, (1, 1, 3)), (2, 4, 4, 2, 4, (0, 0, 0))]:
        q, k, v = (rng.standard_normal((1, T, H, W, 2, 5)) for _ in range(3))
        got = o.tesa(q, k, v, Tw, Sw, sh)
        _close(got[0], block_mask_attention(q[0], k[0], v[0], Tw, Sw, sh), 1e-12, f"TESA block mask {sh}")


def pin_tesa_special(o):
    rng = _rng(8)
    T, H, W, nh, d = 2, 4, 4, 2, 6
    q, k, v = (rng.standard_normal((1, T, H, W, nh, d)) for _ in range(3))
    # one window covering the grid: textbook softmax attention
    got = o.tesa(q, k, v, T, H, (0, 0, 0))
    tq, tk, tv = (torch.from_numpy(a.reshape(T * H * W, nh, d).transpose(1, 0, 2).copy()) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).numpy().transpose(1, 0, 2)
    _close(got.reshape(T * H * W, nh, d), ref, 1e-12, "whole-grid window vs SDPA")
    # 1 x 1 x 1 windows: every token attends only to itself
    _close(o.tesa(q, k, v, 1, 1, (0, 0, 0)), v, 1e-15, "1x1x1 window")
    # q = 0: uniform weights, the window mean of v
    got = o.tesa(np.zeros_like(q), k, v, 2, 2, (0, 0, 0))
    m = v[0].reshape(1, 2, 2, 2, 2, 2, nh, d).mean(axis=(1, 3, 5), keepdims=True)
    want = np.broadcast_to(m, (1, 2, 2, 2, 2, 2, nh, d)).reshape(T, H, W, nh, d)
    _close(got[0], want, 1e-13, "q = 0 gives the window mean")


def pin_zigzag(o):
    """The zigzag comparison order (mode 4). The pages name the Zigzag scan
    (QbitAI method section; paper review 5.5 Table 2) without defining it; the
    reading is the 3D boustrophedon. These properties fix that order
    uniquely: a bijection that starts at grid token 0 and first moves along
    +W; frames visited whole and in time order, each row (t, h) visited
    whole along W; every step to a neighbouring token (one unit in one
    axis). The flip is the reversal, as for the RMS orders."""
    for (T, H, W) in [(2, 2, 3), (3, 4, 5), (1, 5, 1), (4, 1, 6), (3, 3, 2), (2, 7, 4)]:
        N = T * H * W
        seq = o.rms_sequence(T, H, W, 4)
        assert np.array_equal(np.sort(seq), np.arange(N)), "not a bijection"
        t, h, w = seq // (H * W), (seq // W) % H, seq % W
        assert seq[0] == 0 and (N == 1 or W == 1 or seq[1] == 1), "does not start at token 0 along +W"
        assert np.all(t == np.repeat(np.arange(T), H * W)), "frames not whole and in time order"
        rows = (t * H + h).reshape(T * H, W)
        assert np.all(rows == rows[:, :1]), "a row is not visited whole along W"
        if N > 1:
            step = np.abs(np.diff(t)) + np.abs(np.diff(h)) + np.abs(np.diff(w))
            assert np.all(step == 1), "a step does not move to a neighbouring token"
        assert np.array_equal(o.rms_sequence(T, H, W, 4, flip=True), seq[::-1]), "flip is not n -> N-1-n"
    # 2 x 2 x 3 written out by hand: frame 0 rows h = 0 (w ->), h = 1 (w <-);
    # frame 1 rows h = 1 (w ->), h = 0 (w <-)
    assert o.rms_sequence(2, 2, 3, 4).tolist() == [0, 1, 2, 5, 4, 3, 9, 10, 11, 8, 7, 6]


def pin_compose(o):
    """MATE composition (reading R7): a tiny case written out by hand, the
    two-part split (each branch alone, zeros in the other, adds up to the
    whole), and agreement with numpy's float64 matmul on a random case."""
    y1, y2 = np.array([[2.0]]), np.array([[3.0]])
    w1, w2 = np.array([[1.0], [4.0]]), np.array([[5.0], [6.0]])
    assert o.compose(y1, y2, w1, w2).tolist() == [[2 * 1 + 3 * 5, 2 * 4 + 3 * 6]]
    rng = np.random.default_rng(4)
    y1, y2 = rng.standard_normal((2, 3, 5, 24)), rng.standard_normal((2, 3, 5, 16))
    w1, w2 = rng.standard_normal((7, 24)), rng.standard_normal((7, 16))
    full = o.compose(y1, y2, w1, w2)
    assert full.shape == (2, 3, 5, 7)
    parts = o.compose(y1, np.zeros_like(y2), w1, w2) + o.compose(np.zeros_like(y1), y2, w1, w2)
    _close(full, parts, 1e-12, "the two branches do not add up")
    _close(full, y1 @ w1.T + y2 @ w2.T, 1e-12, "composition against numpy matmul")
    # each projection is applied to its own branch: swapping the weights changes the result
    assert not np.allclose(full, y1 @ w1.T + y2 @ (w2[::-1]).T)


def pin_frontend(o):
    """MA-branch front-end (reading R8). In spatial-row order the scan is the grid order, so
    each channel's conv is numpy's full convolution with the reversed taps, cut to the
    sequence (the causal conv); an impulse placed at one scan position of the temporal-column
    order reaches exactly that position and the next three, in scan order, through the taps
    w3, w2, w1, w0; z is the plain projection; dt is softplus(dt_raw + bias); the sampled form
    agrees with the full one."""
    rng = np.random.default_rng(6)
    b, T, H, W, dm, nh, P, G, Ns = 2, 2, 3, 4, 16, 2, 4, 1, 4
    d_inner, dc = nh * P, nh * P + 2 * G * Ns
    u = rng.standard_normal((b, T, H, W, dm))
    w_in = rng.standard_normal((d_inner + dc + nh, dm)) / 4
    cw, cb, db = rng.standard_normal((dc, 4)), rng.standard_normal(dc), rng.standard_normal(nh)
    z, x, dt, Bm, Cm = o.frontend(u, w_in, cw, cb, db, 0, nh, P, G, Ns)
    proj = u.reshape(b, -1, dm) @ w_in.T
    _close(z.reshape(b, -1, d_inner), proj[..., :d_inner], 1e-12, "z is not the projection")
    _close(dt.reshape(b, -1, nh), np.log1p(np.exp(proj[..., d_inner + dc:] + db)), 1e-12, "dt softplus")
    N = T * H * W
    act = np.concatenate([x.reshape(b, N, -1), Bm.reshape(b, N, -1), Cm.reshape(b, N, -1)], axis=-1)
    for bb in range(b):
        for c in range(dc):
            v = np.convolve(proj[bb, :, d_inner + c], cw[c, ::-1])[:N] + cb[c]
            _close(act[bb, :, c], v / (1 + np.exp(-v)), 1e-12, "causal conv in scan order")
    # impulse in temporal-column order: u chosen so that xBC_pre is one hot at scan position p
    T, H, W, dm = 4, 3, 2, 8
    w_in = np.zeros((d_inner + dc + nh, dm))
    w_in[d_inner, 0] = 1.0                  # channel 0 of xBC_pre reads u[..., 0]
    order = o.rms_sequence(T, H, W, 3)
    p = 5
    u = np.zeros((1, T, H, W, dm))
    u.reshape(1, -1, dm)[0, order[p], 0] = 1.0
    cw, cb = rng.standard_normal((dc, 4)), np.zeros(dc)
    z, x, dt, Bm, Cm = o.frontend(u, w_in, cw, cb, np.zeros(nh), 3, nh, P, G, Ns)
    got = x.reshape(1, -1, d_inner)[0, order, 0]    # channel 0 along the scan
    want = np.zeros(T * H * W)
    for j in range(4):
        v = cw[0, 3 - j]
        want[p + j] = v / (1 + np.exp(-v))
    _close(got, want, 1e-12, "impulse response along the scan order")
    # the sampled form gives the same rows
    pos = [0, 3, 11, 23]
    zs, xs, dts, Bs, Cs = o.frontend(u, w_in, cw, cb, np.zeros(nh), 3, nh, P, G, Ns, positions=pos)
    _close(xs.reshape(1, len(pos), -1), x.reshape(1, -1, d_inner)[:, order[pos]], 1e-12, "sampled rows")


def pin_gate_norm(o):
    """MA-branch output side (reading R9). Against torch's float64 rms_norm of y * silu(z)
    taken group by group (the library special case); a group whose gated values are all
    one constant c has the closed form c w / sqrt(c^2 + eps); with eps = 0 every group's
    mean square of out / w is exactly 1; and SiLU written as z (1 + tanh(z / 2)) / 2, not
    the oracle's form, gives the ratios inside a group."""
    rng = np.random.default_rng(7)
    M, C, group, eps = 6, 24, 8, 0.5
    y, z, w = rng.standard_normal((M, C)), rng.standard_normal((M, C)) * 2, rng.standard_normal(C)
    got = o.gate_norm(y, z, w, group, eps)
    yt, zt = torch.from_numpy(y), torch.from_numpy(z)
    v = (yt * torch.nn.functional.silu(zt)).reshape(M, C // group, group)
    want = torch.nn.functional.rms_norm(v, (group,), eps=eps).reshape(M, C) * torch.from_numpy(w)
    _close(got, want.numpy(), 1e-12, "gate norm against torch rms_norm of y silu(z)")
    # every group's gated values equal to one constant c
    silu = 0.5 * z * (1.0 + np.tanh(0.5 * z))
    c = np.repeat(rng.uniform(0.2, 2.0, (M, C // group)), group, axis=1)
    yc = c / silu
    _close(o.gate_norm(yc, z, w, group, eps), c * w / np.sqrt(c * c + eps), 1e-10, "constant group closed form")
    # eps = 0: unit mean square per group, and the in-group ratios of the gated values
    g0 = o.gate_norm(y, z, w, group, 0.0) / w
    _close(np.mean(g0.reshape(M, C // group, group) ** 2, axis=-1), np.ones((M, C // group)), 1e-12,
           "mean square per group")
    gated = (y * silu).reshape(M, C // group, group)
    ratio = g0.reshape(M, C // group, group) / gated
    _close(ratio, np.repeat(ratio[..., :1], group, axis=-1), 1e-10, "one scale per group")
    # the group size matters
    assert not np.allclose(o.gate_norm(y, z, w, C, eps), got)


ALL_PINS = [pin_rms_golden, pin_rms_flip_golden, pin_rms_properties, pin_zigzag, pin_compose, pin_frontend,
            pin_gate_norm, pin_pool,
            pin_scan_dual,
            pin_scan_closed_forms, pin_bissd_dual, pin_bissd_flip_equivariance, pin_bissd_review,
            pin_tesa_golden, pin_tesa_tiling, pin_tesa_block_mask, pin_tesa_special]
