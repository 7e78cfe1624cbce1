"""Tensor-core (tcgen05) paths against the fp64 oracle (needs a B200).

The bf16 / head dim 64 / d_state 64 bi-SSD and the bf16 / head dim 128 /
128-token-window TESA run on the tensor-core kernels; these cases stress
their tiling: every chunk length the kernel takes, ragged tails, partial
windows, batch > 1, long memory and the wide-decay fallback of the factored
exponentials.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from gpu_util import TOL, host64, oracle_bissd_heads, oracle_tesa_heads, rel_err, to_dev

pytestmark = pytest.mark.gpu

mate = pytest.importorskip("linear_complexity_video_b200")

BF16_SSD = workloads.CONFIGS["256p-17s"].with_(nheads=4)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mate.load()


def _run_ssd(cfg, inp, mode, pool, chunk, heads=None):
    dev = to_dev(inp)
    out = mate.bissd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], mode, pool, chunk=chunk)
    assert mate.mate_last_error() == 0
    heads = list(range(cfg.nheads)) if heads is None else heads
    ref = oracle_bissd_heads(inp, mode, pool, heads)
    return rel_err(host64(out)[..., heads, :], ref)


@pytest.mark.parametrize("chunk", [128, 256, 384, 512])
@pytest.mark.parametrize("mode", [0, 3])
def test_ssd_tc_chunks(chunk, mode):
    cfg = BF16_SSD.with_(T=8, H=16, W=16)
    inp = workloads.generate(cfg, seed=1, parts=("ssd",))
    assert _run_ssd(cfg, inp, mode, (2, 4, 4), chunk) <= TOL["bf16"]


@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_ssd_tc_ragged_batch2(mode):
    # 5*9*11 = 495 tokens: the last 512-token chunk is partial, inside a sub-chunk
    cfg = BF16_SSD.with_(T=5, H=9, W=11, batch=2, nheads=3)
    inp = workloads.generate(cfg, seed=2, parts=("ssd",))
    assert _run_ssd(cfg, inp, mode, None, 512) <= TOL["bf16"]
    assert _run_ssd(cfg, inp, mode, (5, 3, 11), 256) <= TOL["bf16"]


@pytest.mark.parametrize("mode", [0, 2])
def test_ssd_tc_tma_rows_batch2(mode):
    # 8x16x16 grid: every 128-position sub-chunk is a box of the grid in SR (16 w x 8 h)
    # and TR (8 t x 16 w), so the rows come by TMA, one launch per batch element
    cfg = BF16_SSD.with_(T=8, H=16, W=16, batch=2, nheads=3)
    inp = workloads.generate(cfg, seed=6, parts=("ssd",))
    assert _run_ssd(cfg, inp, mode, (2, 4, 4), 512) <= TOL["bf16"]


def test_ssd_tc_tma_rows_past_the_end():
    # 9x16x16 = 2304 tokens in SR order: boxes again, and the last 512-token chunk has two
    # sub-chunks wholly past the sequence end, which the TMA fills with zeros
    cfg = BF16_SSD.with_(T=9, H=16, W=16, nheads=3)
    inp = workloads.generate(cfg, seed=7, parts=("ssd",))
    assert _run_ssd(cfg, inp, 0, None, 512) <= TOL["bf16"]
    assert _run_ssd(cfg, inp, 1, (3, 4, 4), 256) <= TOL["bf16"]


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
def test_ssd_tc_review_runs(mode):
    # review boxes 4 or 8 tokens long on the scan's fastest axis: runs of 4 or 8 rows of a
    # sub-chunk share one box, and their sums are taken where the chunk states are; box
    # rows by TMA (8x16x16), gathered rows (4x12x20), and two groups of two heads
    cfg = BF16_SSD.with_(T=8, H=16, W=16, batch=2, nheads=4)
    inp = workloads.generate(cfg, seed=8, parts=("ssd",))
    assert _run_ssd(cfg, inp, mode, (8, 8, 8), 512) <= TOL["bf16"]
    assert _run_ssd(cfg, inp, mode, (4, 4, 4), 256) <= TOL["bf16"]
    cfg = BF16_SSD.with_(T=4, H=12, W=20, nheads=4, ngroups=2)
    inp = workloads.generate(cfg, seed=9, parts=("ssd",))
    assert _run_ssd(cfg, inp, mode, (4, 4, 4), 512) <= TOL["bf16"]
    assert _run_ssd(cfg, inp, mode, (2, 4, 4), 384) <= TOL["bf16"]


def test_ssd_tc_zigzag_odd_rows():
    # the zigzag comparison order with an odd row count per frame (the row walking
    # direction then flips parity from frame to frame), a ragged last chunk, batch 2
    cfg = BF16_SSD.with_(T=3, H=5, W=24, batch=2, nheads=4)
    inp = workloads.generate(cfg, seed=12, parts=("ssd",))
    assert _run_ssd(cfg, inp, 4, None, 512) <= TOL["bf16"]
    assert _run_ssd(cfg, inp, 4, (1, 5, 8), 256) <= TOL["bf16"]
    assert _run_ssd(cfg, inp, 4, (3, 1, 3), 128) <= TOL["bf16"]


@pytest.mark.parametrize("chunk", [128, 384, 512])
def test_ssd_tc_many_items_per_cta(chunk):
    # 32x16x16 grid, 16 heads, batch 2, TC order (TMA row boxes): 352 to 1,024 (head,
    # chunk) items per batch element, so each persistent chunk_out CTA walks several
    # with one to four sub-chunks each (its next item's dt and rows requested during the
    # current one); with 384 the last chunk is a third full; review runs of 8 along t
    cfg = workloads.CONFIGS["256p-17s"].with_(nheads=16, batch=2)
    inp = workloads.generate(cfg, seed=13, parts=("ssd",))
    assert _run_ssd(cfg, inp, 3, (8, 4, 4), chunk, heads=[0, 7, 15]) <= TOL["bf16"]


def test_ssd_tc_review_extremes():
    # one review cell per token (2,048 cells: the cell weights do not fit in shared memory
    # and every h_init part spans several tiles) and one cell for the whole grid (three of
    # the four h_init parts are empty), with pooling runs of 8 along t in TC order
    cfg = BF16_SSD.with_(T=8, H=16, W=16, nheads=4)
    inp = workloads.generate(cfg, seed=10, parts=("ssd",))
    assert _run_ssd(cfg, inp, 0, (1, 1, 1), 512) <= TOL["bf16"]
    assert _run_ssd(cfg, inp, 0, (8, 16, 16), 512) <= TOL["bf16"]
    assert _run_ssd(cfg, inp, 3, (8, 16, 16), 256) <= TOL["bf16"]


def test_ssd_tc_groups():
    cfg = BF16_SSD.with_(T=4, H=8, W=16, nheads=4, ngroups=2)
    inp = workloads.generate(cfg, seed=3, parts=("ssd",))
    assert _run_ssd(cfg, inp, 2, (2, 2, 2), 512) <= TOL["bf16"]


def test_ssd_tc_long_memory():
    # A / 256: a state survives thousands of tokens, so lost chunk or sub-chunk
    # states would show
    cfg = BF16_SSD.with_(T=16, H=16, W=16, variant="long_memory")
    inp = workloads.generate(cfg, seed=4, parts=("ssd",))
    assert _run_ssd(cfg, inp, 3, (4, 4, 4), 512) <= TOL["bf16"]
    assert _run_ssd(cfg, inp, 0, None, 128) <= TOL["bf16"]


def test_ssd_tc_wide_decay_fallback():
    # dt around 2 and |A| up to 16: the decay range inside a 128-token sub-chunk
    # exceeds what factored fp32 exponentials can hold, so the kernel must
    # exponentiate every element exactly
    cfg = BF16_SSD.with_(T=4, H=8, W=16)
    inp = workloads.generate(cfg, seed=5, parts=("ssd",))
    g = torch.Generator().manual_seed(11)
    inp["dt"] = torch.nn.functional.softplus(torch.randn(inp["dt"].shape, generator=g) + 1.5).float()
    assert _run_ssd(cfg, inp, 1, None, 256) <= TOL["bf16"]


def _run_tesa(cfg, heads=None, seed=0):
    inp = workloads.generate(cfg, seed=seed, parts=("attn",))
    dev = to_dev(inp)
    out = mate.tesa(dev["q"], dev["k"], dev["v"], cfg.Tw, cfg.Sw, cfg.shift)
    assert mate.mate_last_error() == 0
    heads = list(range(cfg.attn_heads)) if heads is None else heads
    ref = oracle_tesa_heads(inp, cfg.Tw, cfg.Sw, cfg.shift, heads)
    return rel_err(host64(out)[..., heads, :], ref)


@pytest.mark.parametrize("shift", [(0, 0, 0), (1, 4, 4), (1, 3, 5), (0, 7, 1)])
def test_tesa_tc_partial_windows(shift):
    cfg = workloads.CONFIGS["256p-17s"].with_(T=5, H=12, W=20, batch=2, attn_heads=3, shift=shift)
    assert _run_tesa(cfg) <= TOL["bf16"]


def test_tesa_tc_other_window_shapes():
    # 128-token windows of another shape: 8 x 4 x 4
    cfg = workloads.CONFIGS["256p-17s"].with_(T=16, H=8, W=12, attn_heads=2, Tw=8, Sw=4, shift=(3, 1, 2))
    assert _run_tesa(cfg) <= TOL["bf16"]


def test_tesa_tc_large_logits():
    # scaled-up q: softmax close to one-hot, so the max subtraction matters
    cfg = workloads.CONFIGS["256p-17s"].with_(T=4, H=16, W=16, attn_heads=2)
    inp = workloads.generate(cfg, seed=9, parts=("attn",))
    inp["q"] = (inp["q"].float() * 8).to(torch.bfloat16)
    dev = to_dev(inp)
    out = mate.tesa(dev["q"], dev["k"], dev["v"], cfg.Tw, cfg.Sw, cfg.shift)
    ref = oracle_tesa_heads(inp, cfg.Tw, cfg.Sw, cfg.shift, [0, 1])
    assert rel_err(host64(out), ref) <= TOL["bf16"]
