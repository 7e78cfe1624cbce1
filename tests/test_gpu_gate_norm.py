"""The MA-branch output side (mate_gate_norm_fwd) against the fp64 oracle:
out = y SiLU(z) / sqrt(mean over each channel group of (y SiLU(z))^2 + eps) * w,
bf16 in and out, fp32 arithmetic.

Tolerance, element by element: the oracle sees the same bf16 inputs, so the
difference is the kernel's single bf16 rounding of each output (at most 2^-8 of
its magnitude) plus fp32 arithmetic and the fast exponential and divide in SiLU
(relative errors near 2^-21): |got - ref| <= 4.5e-3 |ref| + 1e-6 max|ref|."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import host64, to_dev

pytestmark = pytest.mark.gpu

mate = pytest.importorskip("linear_complexity_video_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mate.load()


def _check(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    bound = 4.5e-3 * np.abs(ref) + 1e-6 * np.max(np.abs(ref))
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} elements off, worst {np.max(np.abs(got - ref) - bound):.3e} over the bound"


def _case(tokens, channels, group, eps=1e-5, seed=0, rows=None):
    inp = workloads.generate_gate_norm(tokens, channels, seed=seed)
    dev = to_dev(inp)
    out = mate.gate_norm(dev["y"], dev["z"], dev["w"], group, eps)
    assert mate.mate_last_error() == 0
    got = host64(out)
    y, z = inp["y"], inp["z"]
    if rows is not None:
        got, y, z = got[rows], y[rows], z[rows]
    _check(got, oracle.get().gate_norm(y, z, inp["w"], group, eps))


@pytest.mark.parametrize("shape", [
    (1, 8, 8),            # one vector, one group
    (37, 256, 8),         # one group per vector
    (37, 256, 64),        # several groups a row
    (300, 5120, 5120),    # the 80 x 64 channels, one group (ngroups = 1)
    (129, 5120, 2560),    # two groups (ngroups = 2)
    (50, 8192, 1024),     # the widest row the kernel takes
    (64, 1000, 40),       # a row that is no multiple of the CTA's 1,024 channels
])
def test_gate_norm_matches_oracle(shape):
    _case(*shape, seed=sum(shape))


def test_gate_norm_eps_matters():
    # eps comparable to the mean square: the oracle decides where it enters
    _case(40, 512, 128, eps=0.75, seed=5)


def test_gate_norm_extremes():
    # z far negative (the gate closes: SiLU -> 0^-) and far positive (SiLU(z) -> z), y large
    inp = workloads.generate_gate_norm(16, 1024, seed=6)
    inp["z"][:4] = -30.0
    inp["z"][4:8] = 40.0
    inp["y"][8:] = inp["y"][8:] * 3000.0
    dev = to_dev(inp)
    out = mate.gate_norm(dev["y"], dev["z"], dev["w"], 256, 1e-5)
    _check(host64(out), oracle.get().gate_norm(inp["y"], inp["z"], inp["w"], 256, 1e-5))


def test_gate_norm_full_size_sampled_rows():
    # the 131k-token grid x 5,120 channels; the oracle checks 64 rows, both ends included
    tokens = workloads.CONFIGS["512p-68s"].tokens
    rows = np.unique(np.concatenate([[0, 1, tokens - 2, tokens - 1], np.random.default_rng(1).integers(0, tokens, 60)]))
    _case(tokens, 5120, 5120, seed=2, rows=rows)


def test_gate_norm_of_the_branch_outputs():
    # the front-end's z and the bi-SSD's y on a small grid, shapes as the kernels produce them
    cfg = workloads.CONFIGS["512p-17s"].with_(T=4, H=16, W=16, nheads=8)
    fr = workloads.generate_frontend(cfg, seed=1, d_model=256)
    dev = to_dev(fr)
    z, x, dt, B, C = mate.frontend(dev["u"], dev["w_in"], dev["conv_w"], dev["conv_b"], dev["dt_bias"],
                                   cfg.modes[0], cfg.nheads, cfg.headdim, cfg.ngroups, cfg.dstate)
    ssd = workloads.generate(cfg, seed=1, parts=("ssd",))
    A, D = ssd["A"].cuda(), ssd["D"].cuda()
    y = mate.bissd(x, dt, A, B, C, D, cfg.modes[0], None, chunk=512)
    C_ = cfg.nheads * cfg.headdim
    w = (1.0 + torch.randn(C_, generator=torch.Generator().manual_seed(9)) / 10).float()
    out = mate.gate_norm(y.reshape(*y.shape[:-2], C_), z, w.cuda(), C_, 1e-5)
    assert mate.mate_last_error() == 0
    ref = oracle.get().gate_norm(host64(y).reshape(-1, C_), host64(z).reshape(-1, C_), w, C_, 1e-5)
    _check(host64(out).reshape(-1, C_), ref)


def test_gate_norm_rejects_overlap():
    y = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    z = torch.zeros_like(y)
    w = torch.ones(64, device="cuda")
    with pytest.raises(mate.MateError):
        mate.gate_norm(y, z, w, 64, 1e-5, out=y)
