"""Planted mistakes in the oracle must trip at least one pin (CPU only).

Each case patches one plausible slip into a private copy of the oracle's C
source (a dropped term, a wrong index or order, a transposed operand, a
wrong convention), builds it, and runs every pin against it. A mutant that
no pin catches means the pins leave that part of the oracle unchecked.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins

MUTANTS = [
    ("decay ignores dt", "const double decay = exp(dtt * A);", "const double decay = exp(A);"),
    ("dropped D*x term", "yt[p] = acc + D * xt[p];", "yt[p] = acc;"),
    ("C and B swapped in the readout", "acc += (*hpn) * Ct[n];", "acc += (*hpn) * Bt[n];"),
    ("readout before the state update",
     "*hpn = decay * (*hpn) + dtt * xt[p] * Bt[n];\n                acc += (*hpn) * Ct[n];",
     "acc += (*hpn) * Ct[n];\n                *hpn = decay * (*hpn) + dtt * xt[p] * Bt[n];"),
    ("input not scaled by dt", "dtt * xt[p] * Bt[n]", "xt[p] * Bt[n]"),
    ("spatial-column priorities equal spatial-row", "{AXIS_H, AXIS_W, AXIS_T}, /* 1", "{AXIS_W, AXIS_H, AXIS_T}, /* 1"),
    ("temporal-row and temporal-column exchanged", "{AXIS_T, AXIS_W, AXIS_H}, /* 2", "{AXIS_T, AXIS_H, AXIS_W}, /* 2"),
    ("flipped outputs not flipped back", "yb + (Lp + (N - 1 - n)) * wx", "yb + (Lp + n) * wx"),
    ("review prefix [R, R] instead of [R, flip(R)]", "hi = Lp - 1 - i;", "hi = Np + i;"),
    ("pool divides by a wrong count", "inv = 1.0 / ((double)pt * ph * pw);", "inv = 1.0 / ((double)pt * ph);"),
    ("pooled grid unrolled in grid order", "if (review) oracle_rms_sequence(Tp, Hp, Wp, mode, 0, porder);",
     "if (review) oracle_rms_sequence(Tp, Hp, Wp, 0, 0, porder);"),
    ("zigzag rows all walked the same way", "const int w = (row % 2 == 0) ? j : W - 1 - j;", "const int w = j;"),
    ("zigzag odd frames not reversed", "const int h = (t % 2 == 0) ? i : H - 1 - i;", "const int h = i;"),
    ("composition drops the TE branch", "out[i * N + n] = s1 + s2;", "out[i * N + n] = s1;"),
    ("composition reads w1 transposed", "s1 += y1[i * K1 + k] * w1[(int64_t)n * K1 + k];",
     "s1 += y1[i * K1 + k] * w1[(int64_t)(k % N) * K1 + n % K1];"),
    ("gate norm without the gate", "const double v = y[i * C + k] * zk / (1.0 + exp(-zk));",
     "const double v = y[i * C + k];"),
    ("gate norm with a sigmoid gate", "const double v = y[i * C + k] * zk / (1.0 + exp(-zk));",
     "const double v = y[i * C + k] / (1.0 + exp(-zk));"),
    ("gate norm over the sum, not the mean", "1.0 / sqrt(ss / group + eps);", "1.0 / sqrt(ss + eps);"),
    ("gate norm eps outside the root", "1.0 / sqrt(ss / group + eps);", "1.0 / (sqrt(ss / group) + eps);"),
    ("gate norm without its weight", "out[i * C + k] = out[i * C + k] * w[k] * inv;",
     "out[i * C + k] = out[i * C + k] * inv;"),
    ("softmax without 1/sqrt(d)", "const double scale = 1.0 / sqrt((double)d);", "const double scale = 1.0;"),
    ("window boundaries at -shift", "for (int b = s; b < Lx; b += S) starts[n++] = b;",
     "for (int b = (S - s) % S; b < Lx; b += S) starts[n++] = b;"),
    ("attention averages k instead of v", "const double *vj = vb +", "const double *vj = kb +"),
    ("bidirectional difference instead of sum", "o[k] = f[k] + r[k];", "o[k] = f[k] - r[k];"),
]


@pytest.mark.parametrize("name,orig,mutated", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, orig, mutated):
    src = open(oracle.SOURCE).read()
    assert src.count(orig) == 1, f"mutation anchor not found exactly once: {orig!r}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(orig, mutated))
    lib = oracle.build(str(path), str(tmp_path / "libmutant.so"), extra=("-DORACLE_MUTANT",))
    o = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutant '{name}'"


# The front-end part of the oracle is written with numpy (Oracle.frontend); its
# mutants patch that method's source and rebind it on an oracle instance.
PY_MUTANTS = [
    ("front-end taps reversed", "acc = acc + cw[:, k][None, :] * pre(int(p) - 3 + k)",
     "acc = acc + cw[:, 3 - k][None, :] * pre(int(p) - 3 + k)"),
    ("front-end conv in grid order", "order = self.rms_sequence(T, H, W, mode).astype(np.int64)",
     "order = np.arange(T * H * W)"),
    ("front-end dt without its bias", "proj[:, rows, d_inner + dc:] + db[None, None, :]", "proj[:, rows, d_inner + dc:]"),
    ("front-end without SiLU", "act = conv / (1.0 + np.exp(-conv))", "act = conv"),
]


@pytest.mark.parametrize("name,orig,mutated", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_python_mutant_is_caught(name, orig, mutated):
    import inspect
    import textwrap
    import types

    src = inspect.getsource(oracle.Oracle.frontend)
    assert src.count(orig) == 1, f"mutation anchor not found exactly once: {orig!r}"
    ns = {}
    exec(textwrap.dedent(src.replace(orig, mutated)), dict(vars(oracle)), ns)
    o = oracle.Oracle()
    o.frontend = types.MethodType(ns["frontend"], o)
    with pytest.raises((AssertionError, ValueError, KeyError)):
        oracle_pins.pin_frontend(o)
