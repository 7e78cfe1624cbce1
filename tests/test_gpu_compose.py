"""MATE composition on the tensor cores (mate_compose_fwd) against the fp64
oracle: out = y_ma w_ma^T + y_te w_te^T, bf16 storage, fp32 accumulation,
within max|d| / max|ref| <= 2e-2."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, host64, rel_err, to_dev

pytestmark = pytest.mark.gpu

mate = pytest.importorskip("linear_complexity_video_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mate.load()


def _case(tokens, k_ma, k_te, d_model, seed=0, rows=None):
    inp = workloads.generate_compose(tokens, k_ma, k_te, d_model, seed=seed)
    dev = to_dev(inp)
    out = mate.compose(dev["y_ma"], dev["y_te"], dev["w_ma"], dev["w_te"])
    assert mate.mate_last_error() == 0
    got = host64(out)
    if rows is not None:
        got = got[rows]
        inp = dict(inp, y_ma=inp["y_ma"][rows], y_te=inp["y_te"][rows])
    ref = oracle.get().compose(inp["y_ma"], inp["y_te"], inp["w_ma"], inp["w_te"])
    return rel_err(got, ref)


@pytest.mark.parametrize("shape", [
    (128, 64, 64, 256),      # one tile, one K step per branch
    (300, 320, 192, 320),    # ragged rows, a partial column tile
    (1000, 5120, 2560, 2560),  # the block's widths: 80 x 64 and 20 x 128 channels to 2560
    (77, 0, 2560, 512),      # the TE branch alone
    (200, 5120, 0, 2560),    # the MA branch alone
])
def test_compose_matches_oracle(shape):
    assert _case(*shape) <= TOL["bf16"]


def test_compose_full_size_sampled_rows():
    # the 131k-token grid; the oracle checks 64 rows spread over it, including both ends
    tokens = workloads.CONFIGS["512p-68s"].tokens
    rows = np.unique(np.concatenate([[0, 1, 127, 128, tokens - 1], np.random.default_rng(0).integers(0, tokens, 59)]))
    assert _case(tokens, 5120, 2560, 2560, seed=1, rows=rows) <= TOL["bf16"]


def test_compose_of_the_branch_outputs():
    # the composition of the two kernels' own outputs on a small grid (shapes as produced)
    cfg = workloads.CONFIGS["512p-17s"].with_(T=4, H=16, W=16, nheads=4, attn_heads=2)
    inp = workloads.generate(cfg, seed=3)
    dev = to_dev(inp)
    y_ma = mate.bissd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], cfg.modes[0], None, chunk=512)
    y_te = mate.tesa(dev["q"], dev["k"], dev["v"], cfg.Tw, cfg.Sw, cfg.shift)
    w = to_dev(workloads.generate_compose(1, 4 * 64, 2 * 128, 512, seed=3))
    y1 = y_ma.reshape(*y_ma.shape[:4], -1)
    y2 = y_te.reshape(*y_te.shape[:4], -1)
    out = mate.compose(y1, y2, w["w_ma"], w["w_te"])
    assert mate.mate_last_error() == 0 and out.shape == (*y_ma.shape[:4], 512)
    ref = oracle.get().compose(host64(y1), host64(y2), host64(w["w_ma"]), host64(w["w_te"]))
    assert rel_err(host64(out), ref) <= TOL["bf16"]
