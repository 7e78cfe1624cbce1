"""The allocation-free bi-SSD entry point (mate_bissd_fwd_noalloc).

It exists for callers that cannot allocate device memory on their call path
(a plugin whose host owns the device memory pool, code that must avoid the
implicit synchronisation of cudaMalloc/cudaFree, a fixed memory budget). It
takes its scratch from a fixed array inside the library instead of a caller
workspace, so its results must match mate_bissd_fwd's on the same inputs,
call after call. This file is collected last so that a run stopping at the
first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import workloads
from gpu_util import TOL, host64, rel_err, to_dev

pytestmark = pytest.mark.gpu

mate = pytest.importorskip("linear_complexity_video_b200")
from linear_complexity_video_b200 import _lib, api  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mate.load()


def _noalloc_call(L, dev, cfg, mode, pool, out):
    dims = api.ssd_dims(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate, cfg.ngroups, cfg.chunk, cfg.torch_dtype)
    pool_arr = (ctypes.c_int * 3)(*pool) if pool else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return L.mate_bissd_fwd_noalloc(p(dev["x"]), p(dev["dt"]), p(dev["A"]), p(dev["B"]), p(dev["C"]), p(dev["D"]),
                                    cfg.T, cfg.H, cfg.W, mode, pool_arr, p(out), ctypes.byref(dims), stream)


# 256p-17s at all 80 heads needs 20 MiB with its states sized at bf16 (the
# tensor-core path's storage); sized at fp32 it would not fit in 32 MiB.
@pytest.mark.parametrize("name,heads,mode", [("tiny", None, 2), ("512p-17s", 4, 3), ("256p-17s", None, 0)])
def test_noalloc_matches_workspace_entry_point(name, heads, mode):
    cfg = workloads.CONFIGS[name]
    if heads is not None:
        cfg = cfg.with_(nheads=heads)
    dev = to_dev(workloads.generate(cfg, seed=3, parts=("ssd",)))
    need = api.mate_bissd_workspace_bytes(cfg.T, cfg.H, cfg.W, cfg.review,
                                          api.ssd_dims(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate,
                                                       cfg.ngroups, cfg.chunk, cfg.torch_dtype))
    assert 0 < need <= _lib.NOALLOC_SCRATCH_BYTES
    ref = mate.bissd(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], mode, cfg.review, chunk=cfg.chunk)
    torch.cuda.synchronize()
    L = mate.load()
    for _ in range(2):  # two calls in a row share the same scratch array
        out = torch.full_like(dev["x"], float("nan"))
        assert _noalloc_call(L, dev, cfg, mode, cfg.review, out) == _lib.MATE_OK
        torch.cuda.synchronize()
        assert mate.mate_last_error() == 0
        assert rel_err(host64(out), host64(ref)) <= TOL[cfg.dtype]


def test_noalloc_rejects_sizes_beyond_its_scratch():
    cfg = workloads.CONFIGS["512p-17s"].with_(review=None)
    dims = api.ssd_dims(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate, cfg.ngroups, cfg.chunk, cfg.torch_dtype)
    assert api.mate_bissd_workspace_bytes(cfg.T, cfg.H, cfg.W, cfg.review, dims) > _lib.NOALLOC_SCRATCH_BYTES
    dev = to_dev(workloads.generate(cfg.with_(T=1), parts=("ssd",)))  # pointers only; nothing may be written
    out = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    L = mate.load()
    assert _noalloc_call(L, dev, cfg, 0, None, out) == _lib.MATE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert out.item() == 0
