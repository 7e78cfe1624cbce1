"""One MATE token mixer through the library (api.block): the front-end, the bi-SSD, the
gated norm, the TE-branch projections, TESA and the composition, on a small grid.

Each stage is checked against the fp64 oracle fed the GPU's own bf16 inputs to that
stage (so every check is one kernel against its definition, within the bf16 bound
max|d| / max|ref| <= 2e-2), and the block output against the oracle run on u alone,
the whole chain in fp64: there the GPU's bf16 roundings of every intermediate add up
(eleven of them, each <= 2^-8 relative), so the bound is 6e-2."""
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


def _spec(cfg):
    return dict(scan_mode=cfg.modes[0], review_pool=cfg.review, chunk=cfg.chunk, nheads=cfg.nheads,
                headdim=cfg.headdim, ngroups=cfg.ngroups, dstate=cfg.dstate, attn_heads=cfg.attn_heads,
                attn_dim=cfg.attn_dim, Tw=cfg.Tw, Sw=cfg.Sw, shift=cfg.shift)


@pytest.mark.parametrize("name", ["512p-17s", "512p-68s"])
def test_block_stages_and_output(name):
    # the grid shrunk to 8 x 16 x 16 (2,048 tokens, four 512-token chunks), 8 SSD heads,
    # 2 TESA heads, model width 256; each config's own scan order, review box and shift
    cfg = workloads.CONFIGS[name].with_(T=8, H=16, W=16, nheads=8, attn_heads=2)
    p = workloads.generate_block(cfg, seed=3, d_model=256)
    dev = to_dev(p)
    out, mid = mate.block(dev["u"], dev, keep=True, **_spec(cfg))
    torch.cuda.synchronize()
    assert mate.mate_last_error() == 0
    o = oracle.get()
    h = {k: host64(v) for k, v in mid.items()}
    b, T, H, W = cfg.batch, cfg.T, cfg.H, cfg.W
    d_inner, te = cfg.nheads * cfg.headdim, cfg.attn_heads * cfg.attn_dim
    # stage by stage, each from the GPU's inputs to it
    ref = o.frontend(p["u"], p["w_in"], p["conv_w"], p["conv_b"], p["dt_bias"], cfg.modes[0], cfg.nheads, cfg.headdim,
                     cfg.ngroups, cfg.dstate)
    for n, r in zip("z x dt B C".split(), ref):
        assert rel_err(h[n], r) <= TOL["bf16"], n
    y_ref = o.bissd(h["x"], h["dt"], p["A"], h["B"], h["C"], p["D"], cfg.modes[0], cfg.review)
    assert rel_err(h["y"], y_ref) <= TOL["bf16"], "bi-SSD"
    g_ref = o.gate_norm(h["y"].reshape(-1, d_inner), h["z"].reshape(-1, d_inner), p["norm_w"], d_inner, 1e-5)
    assert rel_err(h["y_ma"].reshape(-1, d_inner), g_ref) <= TOL["bf16"], "gated norm"
    u64 = host64(dev["u"]).reshape(-1, 256)
    for n, wn in (("q", "w_q"), ("k", "w_k"), ("v", "w_v")):
        r = o.compose(u64, np.zeros((u64.shape[0], 0)), host64(dev[wn]), np.zeros((te, 0)))
        assert rel_err(h[n].reshape(-1, te), r) <= TOL["bf16"], n
    t_ref = o.tesa(h["q"], h["k"], h["v"], cfg.Tw, cfg.Sw, cfg.shift)
    assert rel_err(h["y_te"], t_ref) <= TOL["bf16"], "TESA"
    c_ref = o.compose(h["y_ma"].reshape(-1, d_inner), h["y_te"].reshape(-1, te), p["w_ma"], p["w_te"])
    got = host64(out).reshape(-1, 256)
    assert rel_err(got, c_ref) <= TOL["bf16"], "composition"
    # the whole chain in fp64 from u
    z, x, dt, B, C = ref
    y = o.bissd(x, dt, p["A"], B, C, p["D"], cfg.modes[0], cfg.review)
    y_ma = o.gate_norm(y.reshape(-1, d_inner), z.reshape(-1, d_inner), p["norm_w"], d_inner, 1e-5)
    qkv = [(u64 @ host64(dev[n]).T).reshape(b, T, H, W, cfg.attn_heads, cfg.attn_dim) for n in ("w_q", "w_k", "w_v")]
    y_te = o.tesa(*qkv, cfg.Tw, cfg.Sw, cfg.shift)
    full = o.compose(y_ma, y_te.reshape(-1, te), p["w_ma"], p["w_te"])
    assert rel_err(got, full) <= 6e-2
