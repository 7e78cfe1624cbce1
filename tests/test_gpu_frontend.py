"""MA-branch front-end on the GPU (mate_frontend_fwd: three tensor-core GEMMs for
in_proj, the causal conv along the scan order with SiLU, softplus for dt)
against the fp64 oracle, every output within max|d| / max|ref| <= 2e-2."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, host64, oracle_bissd_heads, rel_err, to_dev

pytestmark = pytest.mark.gpu

mate = pytest.importorskip("linear_complexity_video_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mate.load()


def _run(cfg, mode, d_model, seed=0):
    inp = workloads.generate_frontend(cfg, seed=seed, d_model=d_model)
    dev = to_dev(inp)
    outs = mate.frontend(dev["u"], dev["w_in"], dev["conv_w"], dev["conv_b"], dev["dt_bias"], mode, cfg.nheads,
                         cfg.headdim, cfg.ngroups, cfg.dstate)
    assert mate.mate_last_error() == 0
    return inp, outs


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
def test_frontend_small_matches_oracle(mode):
    # 120 tokens per batch element (a partial conv block and GEMM tile), 8 heads of 64
    cfg = workloads.CONFIGS["tiny"].with_(T=3, H=5, W=8, batch=2, nheads=8, headdim=64, dstate=64, ngroups=1)
    inp, outs = _run(cfg, mode, 256, seed=mode)
    ref = oracle.get().frontend(inp["u"], inp["w_in"], inp["conv_w"], inp["conv_b"], inp["dt_bias"], mode,
                                cfg.nheads, cfg.headdim, cfg.ngroups, cfg.dstate)
    for name, got, want in zip("z x dt B C".split(), outs, ref):
        assert got.shape == want.shape, name
        assert rel_err(host64(got), want) <= TOL["bf16"], name


def test_frontend_ragged_channels():
    # 544 conv channels (d_state 16): the last warp of a CTA holds channels past the end
    cfg = workloads.CONFIGS["tiny"].with_(T=2, H=6, W=11, batch=1, nheads=8, headdim=64, dstate=16, ngroups=1)
    inp, outs = _run(cfg, 1, 128, seed=11)
    ref = oracle.get().frontend(inp["u"], inp["w_in"], inp["conv_w"], inp["conv_b"], inp["dt_bias"], 1,
                                cfg.nheads, cfg.headdim, cfg.ngroups, cfg.dstate)
    for name, got, want in zip("z x dt B C".split(), outs, ref):
        assert rel_err(host64(got), want) <= TOL["bf16"], name


def test_frontend_block_widths():
    # d_model 2560, 80 heads of 64, d_state 64 (10,448 in_proj rows) on a 4x8x8 grid in TC order
    cfg = workloads.CONFIGS["512p-68s"].with_(T=4, H=8, W=8)
    inp, outs = _run(cfg, 3, workloads.D_MODEL, seed=5)
    ref = oracle.get().frontend(inp["u"], inp["w_in"], inp["conv_w"], inp["conv_b"], inp["dt_bias"], 3,
                                cfg.nheads, cfg.headdim, cfg.ngroups, cfg.dstate)
    for name, got, want in zip("z x dt B C".split(), outs, ref):
        assert rel_err(host64(got), want) <= TOL["bf16"], name


@pytest.mark.slow
def test_frontend_full_size_sampled_positions():
    # the 131k grid; the oracle produces 40 scan positions (the first ones, both ends of
    # a 128-position block, and random ones) from those tokens and their predecessors
    cfg = workloads.CONFIGS["512p-68s"]
    inp, outs = _run(cfg, 3, workloads.D_MODEL, seed=6)
    N = cfg.T * cfg.H * cfg.W
    pos = np.unique(np.concatenate([[0, 1, 2, 3, 127, 128, 129, N - 1], np.random.default_rng(1).integers(0, N, 32)]))
    ref = oracle.get().frontend(inp["u"], inp["w_in"], inp["conv_w"], inp["conv_b"], inp["dt_bias"], 3,
                                cfg.nheads, cfg.headdim, cfg.ngroups, cfg.dstate, positions=pos)
    order = oracle.get().rms_sequence(cfg.T, cfg.H, cfg.W, 3)[pos]
    for name, got, want in zip("z x dt B C".split(), outs, ref):
        g = host64(got).reshape(cfg.batch, N, *got.shape[4:])[:, order]
        assert rel_err(g, want) <= TOL["bf16"], name


def test_frontend_feeds_the_scan():
    # the front-end's outputs through the bi-SSD against the oracle chain (front-end, then
    # bi-SSD) on a small grid, with review tokens
    cfg = workloads.CONFIGS["512p-17s"].with_(T=4, H=16, W=16, nheads=8)
    inp, (z, x, dt, Bm, Cm) = _run(cfg, 2, 256, seed=7)
    ssd = workloads.generate(cfg, seed=7, parts=("ssd",))
    dev = to_dev(ssd)
    y = mate.bissd(x, dt, dev["A"], Bm, Cm, dev["D"], 2, (2, 4, 4), chunk=512)
    assert mate.mate_last_error() == 0
    _, xr, dtr, Br, Cr = oracle.get().frontend(inp["u"], inp["w_in"], inp["conv_w"], inp["conv_b"],
                                               inp["dt_bias"], 2, cfg.nheads, cfg.headdim, cfg.ngroups, cfg.dstate)
    ref = oracle_bissd_heads(dict(x=xr, dt=dtr, A=ssd["A"], B=Br, C=Cr, D=ssd["D"]), 2, (2, 4, 4),
                             range(cfg.nheads))
    assert rel_err(host64(y), ref) <= TOL["bf16"]
