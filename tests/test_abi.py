"""The C ABI library: it loads, exports every declared symbol and rejects bad
arguments on the host (no GPU needed: these calls return before touching
CUDA)."""
import ctypes
import os
import re

import pytest

import linear_complexity_video_b200 as mate
from linear_complexity_video_b200 import _lib, api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            src = "\n".join(ln for ln in src.splitlines() if not ln.lstrip().startswith(("typedef", "#")))
            names.update(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(\w+)\s*\(", src, flags=re.M))
    return names


def test_library_loads():
    L = mate.load()
    assert mate.mate_version() >= 100
    assert L.mate_status_string(0) == b"ok"


def test_every_declared_symbol_is_exported():
    L = mate.load()
    names = declared_functions()
    assert {"mate_bissd_fwd", "tesa_fwd", "mate_bissd_workspace_bytes"} <= names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert set(_lib.EXPORTS) == names, "binding list and header disagree"


def _dims(**kw):
    base = dict(batch=1, nheads=2, headdim=16, dstate=16, ngroups=1, chunk=32, dtype=0, directions=3)
    base.update(kw)
    return _lib.mate_ssd_dims(**base)


def test_workspace_query_rejects_bad_dims():
    ok = api.mate_bissd_workspace_bytes(4, 8, 8, (2, 4, 4), _dims())
    assert ok > 0
    assert api.mate_bissd_workspace_bytes(4, 8, 8, (3, 4, 4), _dims()) == 0      # pool does not divide T
    assert api.mate_bissd_workspace_bytes(4, 8, 8, None, _dims(headdim=48)) == 0  # unsupported head dim
    assert api.mate_bissd_workspace_bytes(4, 8, 8, None, _dims(nheads=3, ngroups=2)) == 0
    assert api.mate_bissd_workspace_bytes(4, 8, 8, None, _dims(chunk=512)) == 0   # CUDA-core path: chunk <= 256
    assert api.mate_bissd_workspace_bytes(4, 8, 8, None, _dims(chunk=2048)) == 0
    # the bf16, 64 x 64 tensor-core path takes chunks of 128..512 tokens
    tc = dict(nheads=4, headdim=64, dstate=64, dtype=1)
    assert api.mate_bissd_workspace_bytes(4, 8, 8, None, _dims(chunk=512, **tc)) > 0
    assert api.mate_bissd_workspace_bytes(4, 8, 8, None, _dims(chunk=640, **tc)) == 0
    assert api.mate_bissd_workspace_bytes(0, 8, 8, None, _dims()) == 0


def test_workspace_grows_linearly_in_tokens():
    d = _dims(nheads=80, headdim=64, dstate=64, chunk=256, dtype=1)
    w1 = api.mate_bissd_workspace_bytes(32, 32, 32, None, d)
    w4 = api.mate_bissd_workspace_bytes(128, 32, 32, None, d)
    assert abs(w4 / w1 - 4.0) < 0.01


def _call_bissd(L, ptr=1, T=4, dims=None, ws=1 << 20, ws_ptr=256, mode=0, pool=None, align=256):
    p = ctypes.c_void_p(ptr * align)
    f = ctypes.c_void_p(ptr * align + (1 << 30))
    dims = dims or _dims()
    pool_arr = (ctypes.c_int * 3)(*pool) if pool else None
    out = ctypes.c_void_p((ptr * align + (2 << 30)) if ptr else 0)
    return L.mate_bissd_fwd(p, f, f, p, p, f, T, 8, 8, mode, pool_arr, out, ctypes.byref(dims),
                            ctypes.c_void_p(ws_ptr + (3 << 30) if ws_ptr else 0), ctypes.c_size_t(ws), None)


def test_bissd_argument_errors_on_host():
    L = mate.load()
    assert _call_bissd(L, ptr=0) == _lib.MATE_ERR_INVALID_ARG                      # null pointers
    assert _call_bissd(L, mode=7) == _lib.MATE_ERR_INVALID_ARG                     # bad scan mode
    assert _call_bissd(L, pool=(3, 4, 4)) == _lib.MATE_ERR_INVALID_ARG             # pool must divide
    assert _call_bissd(L, dims=_dims(dtype=5)) == _lib.MATE_ERR_UNSUPPORTED
    assert _call_bissd(L, align=2) == _lib.MATE_ERR_INVALID_ARG                    # misaligned x
    assert _call_bissd(L, ws=16) == _lib.MATE_ERR_WORKSPACE                        # workspace too small
    assert _call_bissd(L, ws_ptr=0) == _lib.MATE_ERR_WORKSPACE                     # no workspace


def test_tesa_argument_errors_on_host():
    L = mate.load()
    d = _lib.mate_attn_dims(1, 2, 16, 0)
    p = ctypes.c_void_p(1 << 20)
    o = ctypes.c_void_p(1 << 32)
    sh = lambda *v: (ctypes.c_int * 3)(*v)
    assert L.tesa_fwd(p, p, p, 4, 8, 8, 2, 4, sh(2, 0, 0), o, ctypes.byref(d), None) == _lib.MATE_ERR_INVALID_ARG
    assert L.tesa_fwd(p, p, p, 4, 8, 8, 2, 4, sh(0, -1, 0), o, ctypes.byref(d), None) == _lib.MATE_ERR_INVALID_ARG
    assert L.tesa_fwd(p, p, p, 4, 8, 8, 2, 4, None, o, ctypes.byref(d), None) == _lib.MATE_ERR_INVALID_ARG
    d48 = _lib.mate_attn_dims(1, 2, 48, 0)
    assert L.tesa_fwd(p, p, p, 4, 8, 8, 2, 4, sh(0, 0, 0), o, ctypes.byref(d48), None) == _lib.MATE_ERR_UNSUPPORTED
    # out overlapping q
    assert L.tesa_fwd(p, p, p, 4, 8, 8, 2, 4, sh(0, 0, 0), p, ctypes.byref(d), None) == _lib.MATE_ERR_INVALID_ARG


def test_debug_map_argument_errors_on_host():
    L = mate.load()
    assert L.mate_debug_rms_map(4, 8, 8, 9, 0, ctypes.c_void_p(256), None) == _lib.MATE_ERR_INVALID_ARG
    assert L.mate_debug_rms_map(4, 8, 8, 0, 0, None, None) == _lib.MATE_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(ImportError):
        _lib.load()


def test_dispatch_by_storage_type():
    """bf16 runs on the tensor-core kernels only and fp32 on the CUDA-core kernels
    only: shapes the kernels of that storage type cannot take are refused on the
    host, never sent to the other kernels."""
    tc = dict(nheads=4, headdim=64, dstate=64, dtype=1)
    ws = api.mate_bissd_workspace_bytes
    for chunk in (128, 256, 384, 512):
        assert ws(4, 8, 16, None, _dims(chunk=chunk, **tc)) > 0
    for chunk in (64, 200, 640, 1024):                                   # not 128..512 in steps of 128
        assert ws(4, 8, 16, None, _dims(chunk=chunk, **tc)) == 0
    assert ws(4, 8, 16, None, _dims(chunk=256, **dict(tc, headdim=32))) == 0   # bf16 needs 64 x 64
    assert ws(4, 8, 16, None, _dims(chunk=256, **dict(tc, dstate=16))) == 0
    assert ws(4, 8, 16, None, _dims(chunk=256, directions=1, **tc)) == 0       # bf16: both directions only
    assert ws(4, 8, 16, None, _dims(chunk=256)) > 0                             # fp32: CUDA-core kernels
    assert ws(4, 8, 16, None, _dims(chunk=256, directions=1)) > 0
    assert ws(4, 8, 16, None, _dims(chunk=384)) == 0                            # fp32: chunk <= 256
    L = mate.load()
    assert _call_bissd(L, dims=_dims(chunk=256, **dict(tc, headdim=32))) == _lib.MATE_ERR_UNSUPPORTED
    assert _call_bissd(L, dims=_dims(chunk=200, **tc)) == _lib.MATE_ERR_UNSUPPORTED
    # bf16 attention: head dim 128 and 128-token windows only
    p = ctypes.c_void_p(1 << 20)
    o = ctypes.c_void_p(1 << 32)
    sh = (ctypes.c_int * 3)(0, 0, 0)
    for dims, Tw, Sw in (((1, 2, 64, 1), 2, 8), ((1, 2, 128, 1), 2, 4)):
        d = _lib.mate_attn_dims(*dims)
        assert L.tesa_fwd(p, p, p, 4, 8, 8, Tw, Sw, sh, o, ctypes.byref(d), None) == _lib.MATE_ERR_UNSUPPORTED


def test_workspace_layout_by_storage_type():
    """Chunk states take 2 bytes per element for bf16 storage and 4 for fp32;
    bf16 storage adds dt in scan order (fp32, padded to whole chunks)."""
    def expected(nchunks, nh, state_bytes, chunk):
        align = lambda v: (v + 255) // 256 * 256
        states = align(nchunks * nh * 64 * 64 * state_bytes)
        dt_scan = align(nchunks * chunk * nh * 4) if state_bytes == 2 else 0
        return 2 * states + align(nchunks * nh * 4) + dt_scan
    # 2,048 tokens, chunk 256 -> 8 chunks, 4 heads of 64 x 64, no review tokens
    assert api.mate_bissd_workspace_bytes(8, 16, 16, None, _dims(nheads=4, headdim=64, dstate=64, chunk=256,
                                                                 dtype=1)) == expected(8, 4, 2, 256)
    assert api.mate_bissd_workspace_bytes(8, 16, 16, None, _dims(nheads=4, headdim=64, dstate=64, chunk=256,
                                                                 dtype=0)) == expected(8, 4, 4, 256)
    # 1,200 tokens, chunk 512 -> 3 chunks (the last one partial): dt padded to 1,536 positions
    assert api.mate_bissd_workspace_bytes(5, 12, 20, None, _dims(nheads=4, headdim=64, dstate=64, chunk=512,
                                                                 dtype=1)) == expected(3, 4, 2, 512)


def test_fastdiv_matches_integer_division():
    """The kernels' multiply-high division (Granlund and Montgomery 1994,
    figure 4.1) against exact integer division: every divisor the index maps
    can meet on small grids, powers of two and their neighbours, large odd
    divisors, and dividends at the ends of the range."""
    import numpy as np

    L = mate.load()
    rng = np.random.default_rng(0)
    top = (1 << 31) - 1
    divisors = list(range(1, 300)) + [(1 << k) + e for k in range(1, 31) for e in (-1, 0, 1)] + \
        [top, top - 1, 1_000_003, 73_728, 147_456, 2_359_296]
    for d in divisors:
        if not 1 <= d <= top:
            continue
        n = np.concatenate([np.arange(0, 2048, dtype=np.uint64),
                            rng.integers(0, 1 << 31, 4096, dtype=np.uint64),
                            np.array([top, top - 1, d, d - 1, d + 1, 2 * d - 1, top // d * d, top // d * d - 1],
                                     dtype=np.uint64)])
        n = n[n <= top].astype(np.uint32)
        q = np.empty_like(n)
        assert L.mate_debug_fastdiv(n.ctypes.data, q.ctypes.data, n.size, d) == _lib.MATE_OK
        assert np.array_equal(q, n // np.uint32(d)), d


def test_fastdiv_rejects_out_of_range():
    import numpy as np

    L = mate.load()
    n = np.array([1 << 31], dtype=np.uint32)
    q = np.zeros(1, dtype=np.uint32)
    assert L.mate_debug_fastdiv(n.ctypes.data, q.ctypes.data, 1, 3) == _lib.MATE_ERR_INVALID_ARG
    n[0] = 5
    assert L.mate_debug_fastdiv(n.ctypes.data, q.ctypes.data, 1, 0) == _lib.MATE_ERR_INVALID_ARG
    assert L.mate_debug_fastdiv(n.ctypes.data, q.ctypes.data, 1, 1 << 31) == _lib.MATE_ERR_INVALID_ARG
    assert L.mate_debug_fastdiv(None, None, 1, 3) == _lib.MATE_ERR_INVALID_ARG
    assert q[0] == 0


def test_compose_rejects_bad_arguments():
    """mate_compose_fwd checks its sizes, dtype and pointers before any CUDA call."""
    L = mate.load()
    p = ctypes.c_void_p(256)
    ok = _lib.mate_compose_dims(128, 5120, 2560, 2560, _lib.MATE_BF16)
    assert L.mate_compose_fwd(p, p, p, p, p, None, None) == _lib.MATE_ERR_INVALID_ARG
    for bad in [(0, 64, 64, 64), (128, 0, 0, 64), (128, 64, 64, 0), (128, -64, 64, 64)]:
        d = _lib.mate_compose_dims(*bad, _lib.MATE_BF16)
        assert L.mate_compose_fwd(p, p, p, p, p, ctypes.byref(d), None) == _lib.MATE_ERR_INVALID_ARG, bad
    for bad in [(128, 5000, 2560, 2560), (128, 5120, 2560, 2500), (128, 5120, 100, 2560)]:
        d = _lib.mate_compose_dims(*bad, _lib.MATE_BF16)
        assert L.mate_compose_fwd(p, p, p, p, p, ctypes.byref(d), None) == _lib.MATE_ERR_UNSUPPORTED, bad
    d = _lib.mate_compose_dims(128, 5120, 2560, 2560, _lib.MATE_F32)
    assert L.mate_compose_fwd(p, p, p, p, p, ctypes.byref(d), None) == _lib.MATE_ERR_UNSUPPORTED
    assert L.mate_compose_fwd(p, p, p, p, None, ctypes.byref(ok), None) == _lib.MATE_ERR_INVALID_ARG
    assert L.mate_compose_fwd(None, p, p, p, p, ctypes.byref(ok), None) == _lib.MATE_ERR_INVALID_ARG
    q = ctypes.c_void_p(264)  # 8-byte aligned only
    assert L.mate_compose_fwd(q, p, p, p, p, ctypes.byref(ok), None) == _lib.MATE_ERR_INVALID_ARG
    # one branch absent: its pointers may be null
    one = _lib.mate_compose_dims(128, 0, 2560, 2560, _lib.MATE_BF16)
    r = ctypes.c_void_p(1 << 40)
    assert L.mate_compose_fwd(None, p, None, r, None, ctypes.byref(one), None) == _lib.MATE_ERR_INVALID_ARG


def test_gate_norm_rejects_bad_arguments():
    """mate_gate_norm_fwd checks its sizes, eps, dtype, pointers and overlaps before any CUDA call."""
    L = mate.load()
    base = 1 << 40
    y, z, w, o = (ctypes.c_void_p(base + i * (1 << 32)) for i in range(4))
    ok = _lib.mate_gate_norm_dims(128, 5120, 5120, _lib.MATE_BF16)
    f = ctypes.c_float
    assert L.mate_gate_norm_fwd(y, z, w, f(1e-5), o, None, None) == _lib.MATE_ERR_INVALID_ARG
    for bad in [(0, 64, 64), (128, 0, 64), (128, 64, 0), (-1, 64, 64)]:
        d = _lib.mate_gate_norm_dims(*bad, _lib.MATE_BF16)
        assert L.mate_gate_norm_fwd(y, z, w, f(1e-5), o, ctypes.byref(d), None) == _lib.MATE_ERR_INVALID_ARG, bad
    # group not dividing the row, not a multiple of 8, or a row beyond 8192 channels
    for bad in [(128, 5120, 3000), (128, 120, 12), (128, 16384, 16384)]:
        d = _lib.mate_gate_norm_dims(*bad, _lib.MATE_BF16)
        assert L.mate_gate_norm_fwd(y, z, w, f(1e-5), o, ctypes.byref(d), None) == _lib.MATE_ERR_UNSUPPORTED, bad
    d = _lib.mate_gate_norm_dims(128, 5120, 5120, _lib.MATE_F32)
    assert L.mate_gate_norm_fwd(y, z, w, f(1e-5), o, ctypes.byref(d), None) == _lib.MATE_ERR_UNSUPPORTED
    for eps in (-1.0, float("nan"), float("inf")):
        assert L.mate_gate_norm_fwd(y, z, w, f(eps), o, ctypes.byref(ok), None) == _lib.MATE_ERR_INVALID_ARG, eps
    assert L.mate_gate_norm_fwd(y, z, None, f(1e-5), o, ctypes.byref(ok), None) == _lib.MATE_ERR_INVALID_ARG
    assert L.mate_gate_norm_fwd(y, z, w, f(1e-5), ctypes.c_void_p(base + 8), ctypes.byref(ok), None) == \
        _lib.MATE_ERR_INVALID_ARG  # misaligned
    # out overlapping y (one row past its start) or w
    assert L.mate_gate_norm_fwd(y, z, w, f(1e-5), ctypes.c_void_p(base + 5120 * 2), ctypes.byref(ok), None) == \
        _lib.MATE_ERR_INVALID_ARG
    assert L.mate_gate_norm_fwd(y, z, o, f(1e-5), o, ctypes.byref(ok), None) == _lib.MATE_ERR_INVALID_ARG


def test_python_entry_points_refuse_host_tensors():
    """The binding has no CPU path: host tensors are refused before any library call."""
    import torch
    import workloads

    cfg = workloads.CONFIGS["tiny"]
    inp = workloads.generate(cfg, seed=0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mate.bissd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], 0, None, chunk=32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mate.tesa(inp["q"], inp["k"], inp["v"], cfg.Tw, cfg.Sw, cfg.shift)
    y = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mate.gate_norm(y, y, torch.ones(64), 64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mate.linear(y, torch.zeros(64, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA tensor"):
        mate.compose(y, y, torch.zeros(64, 64, dtype=torch.bfloat16), torch.zeros(64, 64, dtype=torch.bfloat16))
    blk = workloads.generate_block(workloads.CONFIGS["tiny"].with_(nheads=8, headdim=16, dstate=16), d_model=64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mate.block(blk["u"], blk, scan_mode=0, review_pool=None, chunk=32, nheads=8, headdim=16, ngroups=1,
                   dstate=16, attn_heads=2, attn_dim=16, Tw=2, Sw=4, shift=(0, 0, 0))


def test_frontend_rejects_bad_arguments():
    """mate_frontend_fwd and its workspace query check sizes, dtype, scan mode, pointers,
    workspace and overlaps before any CUDA call."""
    L = mate.load()
    T, H, W = 4, 8, 8
    ok = _lib.mate_frontend_dims(1, 256, 8, 64, 1, 64, _lib.MATE_BF16)
    M, dc, nh = T * H * W, 8 * 64 + 2 * 64, 8

    def up(n):
        return (n + 255) // 256 * 256

    assert L.mate_frontend_workspace_bytes(T, H, W, ctypes.byref(ok)) == up(M * dc * 2) + up(M * nh * 2)
    for bad, why in [((1, 256, 6, 64, 1, 64), "heads not a multiple of 8"), ((1, 100, 8, 64, 1, 64), "d_model"),
                     ((1, 256, 8, 64, 3, 64), "groups not dividing heads"), ((0, 256, 8, 64, 1, 64), "batch")]:
        d = _lib.mate_frontend_dims(*bad, _lib.MATE_BF16)
        assert L.mate_frontend_workspace_bytes(T, H, W, ctypes.byref(d)) == 0, why
    # distinct fake device addresses, 4 GB apart (nothing is dereferenced before the checks)
    u, w_in, cw, cb, db, z, x, dt, B, C, ws = (ctypes.c_void_p((1 << 40) + i * (1 << 32)) for i in range(11))
    nbytes = L.mate_frontend_workspace_bytes(T, H, W, ctypes.byref(ok))

    def call(d=ok, mode=0, **kw):
        a = dict(u=u, w_in=w_in, cw=cw, cb=cb, db=db, z=z, x=x, dt=dt, B=B, C=C, ws=ws, n=nbytes)
        a.update(kw)
        return L.mate_frontend_fwd(a["u"], a["w_in"], a["cw"], a["cb"], a["db"], T, H, W, mode, a["z"], a["x"], a["dt"],
                                   a["B"], a["C"], ctypes.byref(d) if d is not None else None, a["ws"],
                                   ctypes.c_size_t(a["n"]), None)

    assert call(d=None) == _lib.MATE_ERR_INVALID_ARG
    assert call(mode=5) == _lib.MATE_ERR_INVALID_ARG
    assert call(d=_lib.mate_frontend_dims(1, 256, 6, 64, 1, 64, _lib.MATE_BF16)) == _lib.MATE_ERR_UNSUPPORTED
    assert call(d=_lib.mate_frontend_dims(1, 256, 8, 64, 1, 64, _lib.MATE_F32)) == _lib.MATE_ERR_UNSUPPORTED
    assert call(u=None) == _lib.MATE_ERR_INVALID_ARG
    assert call(x=ctypes.c_void_p((1 << 40) + 6 * (1 << 32) + 8)) == _lib.MATE_ERR_INVALID_ARG  # misaligned bf16
    assert call(n=nbytes - 1) == _lib.MATE_ERR_WORKSPACE
    assert call(ws=None) == _lib.MATE_ERR_WORKSPACE
    assert call(x=z) == _lib.MATE_ERR_INVALID_ARG          # two outputs overlap
    assert call(dt=u) == _lib.MATE_ERR_INVALID_ARG         # an output over an input
