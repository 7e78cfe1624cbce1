"""Helpers shared by the GPU parity tests: device copies, the error metric
and sampled-head oracle calls."""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref) -> float:
    """max |got - ref| / max |ref|, the parity metric for floating point."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def to_dev(d):
    return {k: v.cuda() for k, v in d.items()}


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def oracle_bissd_heads(inp, mode, pool, heads):
    """Oracle output for a subset of SSD heads (heads are independent)."""
    hs = list(heads)
    x = inp["x"][..., hs, :]
    dt = inp["dt"][..., hs]
    A = inp["A"][hs]
    D = inp["D"][hs]
    nh = inp["x"].shape[4]
    G = inp["B"].shape[4]
    if G == 1:
        B, C = inp["B"], inp["C"]
        return oracle.get().bissd(x, dt, A, B, C, D, mode, pool)
    # one head at a time so that each keeps its own group
    outs = []
    for h in hs:
        g = h // (nh // G)
        outs.append(oracle.get().bissd(inp["x"][..., [h], :], inp["dt"][..., [h]], inp["A"][[h]],
                                       inp["B"][..., [g], :], inp["C"][..., [g], :], inp["D"][[h]], mode, pool))
    return np.concatenate(outs, axis=4)


def oracle_tesa_heads(inp, Tw, Sw, shift, heads):
    hs = list(heads)
    return oracle.get().tesa(inp["q"][..., hs, :], inp["k"][..., hs, :], inp["v"][..., hs, :], Tw, Sw, shift)
