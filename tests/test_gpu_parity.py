"""GPU path against the fp64 oracle, through the C ABI (needs a B200).

Parity bar: index maps bit-exact; floating point max|d|/max|ref| <= 1e-4
for fp32 storage and <= 2e-2 for bf16 storage (fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, host64, oracle_bissd_heads, oracle_tesa_heads, rel_err, to_dev

pytestmark = pytest.mark.gpu

mate = pytest.importorskip("linear_complexity_video_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mate.load()


# ---------------------------------------------------------------------------
# index maps: bit exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("grid", [(2, 2, 3), (4, 8, 8), (3, 5, 7), (128, 32, 32), (1, 1, 1), (32, 48, 48)])
@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("flip", [False, True])
def test_rms_map_bit_exact(grid, mode, flip):
    T, H, W = grid
    got = mate.rms_map(T, H, W, mode, flip).cpu().numpy()
    want = oracle.get().rms_sequence(T, H, W, mode, flip)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("case", [
    (4, 8, 8, 2, 4, (1, 2, 2)), (32, 32, 32, 2, 8, (1, 4, 4)), (128, 32, 32, 2, 8, (1, 4, 4)),
    (32, 48, 48, 2, 8, (0, 0, 0)), (5, 7, 9, 2, 4, (1, 3, 1)), (4, 5, 6, 3, 4, (1, 1, 3)), (3, 3, 3, 4, 8, (3, 7, 5))])
def test_tesa_map_bit_exact(case):
    T, H, W, Tw, Sw, sh = case
    got = mate.tesa_map(T, H, W, Tw, Sw, sh).cpu().numpy()
    want = oracle.get().tesa_window_ids(T, H, W, Tw, Sw, sh)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------------------
# bi-SSD
# ---------------------------------------------------------------------------
def _bissd_case(cfg, mode, pool, chunk=None, heads=None, seed=0):
    inp = workloads.generate(cfg, seed=seed, parts=("ssd",))
    dev = to_dev(inp)
    out = mate.bissd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], mode, pool,
                     chunk=chunk or cfg.chunk)
    assert mate.mate_last_error() == 0
    heads = list(range(cfg.nheads)) if heads is None else heads
    ref = oracle_bissd_heads(inp, mode, pool, heads)
    got = host64(out)[..., heads, :]
    return rel_err(got, ref)


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
def test_bissd_tiny_fp32(mode):
    cfg = workloads.CONFIGS["tiny"]
    assert _bissd_case(cfg, mode, cfg.review) <= TOL["f32"]


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
def test_bissd_tiny_no_review(mode):
    cfg = workloads.CONFIGS["tiny"]
    assert _bissd_case(cfg, mode, None) <= TOL["f32"]


@pytest.mark.parametrize("chunk", [1, 7, 16, 32, 64, 256])
def test_bissd_independent_of_chunk(chunk):
    cfg = workloads.CONFIGS["tiny"]
    assert _bissd_case(cfg, 2, cfg.review, chunk=chunk) <= TOL["f32"]


def test_bissd_long_memory_fp32():
    # states must survive many chunks: a lost inter-chunk state would show
    cfg = workloads.CONFIGS["tiny"].with_(variant="long_memory", T=8)
    assert _bissd_case(cfg, 3, cfg.review, chunk=16) <= TOL["f32"]


def test_bissd_ragged_and_groups():
    # 105 tokens (not a multiple of the chunk), 4 heads in 2 B/C groups, batch 2
    cfg = workloads.CONFIGS["tiny"].with_(T=3, H=5, W=7, batch=2, nheads=4, ngroups=2, headdim=32, dstate=16)
    for mode in range(5):
        assert _bissd_case(cfg, mode, (3, 5, 7), chunk=32) <= TOL["f32"]
        assert _bissd_case(cfg, mode, None, chunk=32) <= TOL["f32"]


def test_bissd_single_token():
    cfg = workloads.CONFIGS["tiny"].with_(T=1, H=1, W=1, batch=2)
    assert _bissd_case(cfg, 0, (1, 1, 1)) <= TOL["f32"]
    assert _bissd_case(cfg, 1, None) <= TOL["f32"]


def test_bissd_directions_add_up():
    cfg = workloads.CONFIGS["tiny"]
    dev = to_dev(workloads.generate(cfg, parts=("ssd",)))
    args = (dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], 3, cfg.review)
    bi = mate.bissd(*args, chunk=32, directions=3)
    f = mate.bissd(*args, chunk=32, directions=1)
    b = mate.bissd(*args, chunk=32, directions=2)
    assert rel_err(host64(f + b), host64(bi)) <= 1e-6
    # Without review tokens, the flipped scan of a grid equals the forward scan of the grid
    # reversed on every axis. (With review tokens it does not: reversing the grid reverses R,
    # and the prefix [flip(R), R] differs from [R, flip(R)].)
    rev = lambda t: t.flip(1, 2, 3).contiguous()
    b0 = mate.bissd(*args[:7], None, chunk=32, directions=2)
    fr = mate.bissd(rev(dev["x"]), rev(dev["dt"]), dev["A"], rev(dev["B"]), rev(dev["C"]), dev["D"], 3, None,
                    chunk=32, directions=1)
    assert rel_err(host64(rev(fr)), host64(b0)) <= 1e-5


def test_bissd_256p_bf16():
    cfg = workloads.CONFIGS["256p-17s"]
    assert _bissd_case(cfg, 0, None, heads=[0, 1, 41, 79]) <= TOL["bf16"]


@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_bissd_512p_17s_bf16(mode):
    cfg = workloads.CONFIGS["512p-17s"]
    assert _bissd_case(cfg, mode, cfg.review, heads=[0, 23, 79]) <= TOL["bf16"]


@pytest.mark.slow
def test_bissd_512p_68s_bf16_full_size():
    cfg = workloads.CONFIGS["512p-68s"]
    assert _bissd_case(cfg, 3, cfg.review, heads=[5, 66]) <= TOL["bf16"]


@pytest.mark.slow
def test_bissd_512p_68s_zigzag_full_size():
    # the zigzag comparison order on the 131k grid (gathered rows, review runs along W)
    cfg = workloads.CONFIGS["512p-68s"]
    assert _bissd_case(cfg, workloads.ZZ, cfg.review, heads=[17]) <= TOL["bf16"]


@pytest.mark.slow
@pytest.mark.parametrize("mode", [0, 3])
def test_bissd_768p_bf16_full_size(mode):
    # SR rows are gathered (W = 48 is no divisor of 128); TC rows come as TMA boxes,
    # one launch per batch element
    cfg = workloads.CONFIGS["768p-17s"]
    assert _bissd_case(cfg, mode, None, heads=[11, 70]) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# TESA
# ---------------------------------------------------------------------------
def _tesa_case(cfg, heads=None, seed=0):
    inp = workloads.generate(cfg, seed=seed, parts=("attn",))
    dev = to_dev(inp)
    out = mate.tesa(dev["q"], dev["k"], dev["v"], cfg.Tw, cfg.Sw, cfg.shift)
    heads = list(range(cfg.attn_heads)) if heads is None else heads
    ref = oracle_tesa_heads(inp, cfg.Tw, cfg.Sw, cfg.shift, heads)
    return rel_err(host64(out)[..., heads, :], ref)


def test_tesa_tiny_fp32():
    assert _tesa_case(workloads.CONFIGS["tiny"]) <= TOL["f32"]


@pytest.mark.parametrize("shift", [(0, 0, 0), (1, 2, 2), (1, 3, 1), (0, 1, 0)])
def test_tesa_partial_windows_fp32(shift):
    cfg = workloads.CONFIGS["tiny"].with_(T=5, H=7, W=9, batch=2)
    assert _tesa_case(cfg.with_(shift=shift)) <= TOL["f32"]


def test_tesa_256p_bf16():
    assert _tesa_case(workloads.CONFIGS["256p-17s"], heads=[0, 7, 19]) <= TOL["bf16"]


def test_tesa_512p_17s_bf16_shifted():
    assert _tesa_case(workloads.CONFIGS["512p-17s"], heads=[0, 19]) <= TOL["bf16"]


@pytest.mark.slow
def test_tesa_512p_68s_bf16_full_size():
    assert _tesa_case(workloads.CONFIGS["512p-68s"], heads=[3]) <= TOL["bf16"]


@pytest.mark.slow
def test_tesa_768p_bf16_full_size():
    assert _tesa_case(workloads.CONFIGS["768p-17s"], heads=[12]) <= TOL["bf16"]


def test_inputs_not_written():
    cfg = workloads.CONFIGS["tiny"]
    dev = to_dev(workloads.generate(cfg))
    before = {k: v.clone() for k, v in dev.items()}
    mate.bissd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], 1, cfg.review, chunk=32)
    mate.tesa(dev["q"], dev["k"], dev["v"], cfg.Tw, cfg.Sw, cfg.shift)
    torch.cuda.synchronize()
    for k in dev:
        assert torch.equal(before[k], dev[k]), f"{k} was written"
