"""Throughput of the MATE token mix on B200: one step = review pooling and
prefix scan, the bidirectional SSD scan and TESA over one batch of a
synthetic latent grid.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl mate|reference]
    python bench.py --report | --component compose|frontend|gate_norm|block [--config NAME]

Prints one JSON line (rank 0). With N > 1 (torchrun, one rank per GPU; a
plain `python bench.py --gpus N` starts the N ranks itself) every rank
processes its own batch element drawn with its own seed: the path has no
exchange step, so this is weak scaling with no collective on the data path;
the NCCL group only carries the barrier and the max-over-ranks time.

--impl reference times the fp64 CPU oracle (the only other code this script
may run) on the same workload, one bounded sample per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# algorithmic bytes per token of each kernel (one read of what the step
# must read, one write of what it must write)
# ---------------------------------------------------------------------------
def elem_bytes(cfg):
    return 4 if cfg.dtype == "f32" else 2


def algorithmic_bytes(cfg):
    e = elem_bytes(cfg)
    x = cfg.nheads * cfg.headdim * e
    dt = cfg.nheads * 4
    bc = cfg.ngroups * cfg.dstate * e
    per_tok = {
        # a separate pooling pass over x, dt, B: only where the box sums cannot be taken
        # inside chunk_state, so not part of the path's minimum
        "review_pool": (x + dt + bc) if cfg.review else 0,
        "chunk_state": x + dt + bc,                          # x, dt, B
        "chunk_out": 2 * x + dt + 2 * bc,                    # x, dt, B, C in; y out
        "tesa": 4 * cfg.attn_heads * cfg.attn_dim * e,       # q, k, v in; out
    }
    per_tok["bissd"] = 2 * x + dt + 2 * bc                   # the MA-branch as one op
    return per_tok


def mma_flops(cfg):
    """Tensor-core flops per token of each kernel, as the kernels issue them
    (bf16 path: 128-token sub-chunks, both scan directions).
    chunk_state: one MMA [U_f^T; U_b^T] (2P x 128) . B (128 x Ns) per sub-chunk.
    chunk_out: that MMA again, S = C B^T (128 x 128 x Ns), M x (128 x P x 128)
    and R_f C h_f^T + R_b C h_b^T (2 x 128 x P x Ns) per sub-chunk.
    tesa: Q K^T and P V over every key of the token's window."""
    P, Ns, nh = cfg.headdim, cfg.dstate, cfg.nheads
    q = 128
    state = 2 * (2 * P) * Ns
    out = state + 2 * q * Ns + 2 * q * P + 2 * (2 * P * Ns)
    win = cfg.Tw * cfg.Sw * cfg.Sw
    f = {"review_pool": 0, "chunk_state": nh * state, "state_pass": 0, "chunk_out": nh * out,
         "tesa": cfg.attn_heads * 4 * cfg.attn_dim * win}
    f["bissd"] = f["chunk_state"] + f["chunk_out"]
    return f


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid):
        self.uuid = device_uuid
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle as it stands on a bounded sample of the workload
# ---------------------------------------------------------------------------
def oracle_sample(cfg, threads=None):
    """Time the fp64 oracle on a head subset of the full grid and scale to the
    whole workload (heads are independent, so cost is linear in heads).
    Returns (Mtokens/s, cores, description)."""
    import oracle

    threads = threads or min(os.cpu_count() or 1, 16)
    os.environ.setdefault("OMP_NUM_THREADS", str(threads))
    o = oracle.get()
    ssd_heads = min(cfg.nheads, threads)
    attn_heads = min(cfg.attn_heads, 2)
    inp = workloads.generate(cfg.with_(batch=1), seed=0)
    x = inp["x"][..., :ssd_heads, :]
    dt = inp["dt"][..., :ssd_heads]
    A = inp["A"][:ssd_heads]
    D = inp["D"][:ssd_heads]
    mode = cfg.modes[0]
    t0 = time.perf_counter()
    o.bissd(x, dt, A, inp["B"], inp["C"], D, mode, cfg.review)
    t_ssd = time.perf_counter() - t0
    q, k, v = (inp[n][..., :attn_heads, :] for n in ("q", "k", "v"))
    t0 = time.perf_counter()
    o.tesa(q, k, v, cfg.Tw, cfg.Sw, cfg.shift)
    t_attn = time.perf_counter() - t0
    t_full = t_ssd * cfg.nheads / ssd_heads + t_attn * cfg.attn_heads / attn_heads
    desc = (f"{cfg.name} grid {cfg.T}x{cfg.H}x{cfg.W}, 1 batch element: bi-SSD on {ssd_heads}/{cfg.nheads} heads "
            f"({t_ssd:.2f} s), TESA on {attn_heads}/{cfg.attn_heads} heads ({t_attn:.2f} s), "
            f"scaled by head count to the full step")
    return cfg.N / t_full / 1e6, threads, desc


# ---------------------------------------------------------------------------
# multi-rank plumbing (weak scaling over independent grids, no data exchange)
# ---------------------------------------------------------------------------
def rank_seed(rank: int, base: int = 0) -> int:
    """Each rank draws its own grid: seed = base + rank."""
    return base + rank


def max_over_ranks(ms: float, dist, device=None) -> float:
    """The step time of the job is the slowest rank's (max all-reduce)."""
    if dist is None:
        return ms
    import torch

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job Mtokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms_per_step / 1e3) / 1e6


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def run_mate(args, cfg, rank, world, dist):
    import ctypes

    import torch

    import linear_complexity_video_b200 as mate
    from linear_complexity_video_b200 import _lib, api

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    L = mate.load()
    stream = torch.cuda.current_stream()
    mode = cfg.modes[0]

    host = workloads.generate(cfg, seed=rank_seed(rank))
    d = {k: v.to(dev) for k, v in host.items()}
    out_ssd = torch.empty_like(d["x"])
    out_att = torch.empty_like(d["q"])
    ws = api.bissd_workspace(d["x"], d["B"], cfg.review, cfg.chunk)
    sdims = api.ssd_dims(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate, cfg.ngroups, cfg.chunk, cfg.torch_dtype)
    adims = api.attn_dims(cfg.batch, cfg.attn_heads, cfg.attn_dim, cfg.torch_dtype)

    def step(src, o_ssd, o_att, workspace, strm=None):
        strm = strm or stream
        api.mate_bissd_fwd(src["x"], src["dt"], src["A"], src["B"], src["C"], src["D"], cfg.T, cfg.H, cfg.W, mode,
                           cfg.review, o_ssd, sdims, workspace, strm)
        api.tesa_fwd(src["q"], src["k"], src["v"], cfg.T, cfg.H, cfg.W, cfg.Tw, cfg.Sw, cfg.shift, o_att, adims,
                     strm)

    # phase events recorded through the library's enqueue-time hook
    marks = []

    def hook(phase, is_end, strm, user):
        # recorded on the stream the library launches that phase on (a phase may run
        # on the library's side stream)
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(torch.cuda.ExternalStream(strm) if strm and strm != stream.cuda_stream else stream)
        marks.append((phase, is_end, ev))

    hook_c = _lib.PHASE_HOOK(hook)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step(d, out_ssd, out_att, ws)
    torch.cuda.synchronize()
    rc = mate.mate_last_error()
    if rc != 0:
        raise RuntimeError(f"device error word {rc}")

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}") if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    launches0 = L.mate_kernel_launches()
    L.mate_set_phase_hook(hook_c, None)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step(d, out_ssd, out_att, ws)
    ev1.record(stream)
    torch.cuda.synchronize()
    L.mate_set_phase_hook(_lib.PHASE_HOOK(), None)
    launches = L.mate_kernel_launches() - launches0
    barrier()
    clocks = sampler.stop() if sampler else None
    ms_step = max_over_ranks(ev0.elapsed_time(ev1), dist, dev) / args.steps

    # per-phase average duration on this rank
    phase_ms = {}
    open_ev = {}
    for phase, is_end, ev in marks:
        if not is_end:
            open_ev[phase] = ev
        else:
            phase_ms.setdefault(_lib.PHASES[phase], []).append(open_ev.pop(phase).elapsed_time(ev))
    # a phase may launch once per batch element: per-step totals, and per-launch averages
    phase_avg = {k: sum(v) / args.steps for k, v in phase_ms.items()}
    phase_launch_avg = {k: sum(v) / len(v) for k, v in phase_ms.items()}
    launches_per_step = {k: len(v) / args.steps for k, v in phase_ms.items()}

    # end to end through the public API with host buffers: every step copies its
    # inputs from pinned host memory and its outputs back. Steps are pipelined over
    # three streams (copies in, compute, copies out) and two sets of device buffers,
    # as a serving loop would run them: step i's inputs travel while step i-1
    # computes and step i-2's outputs travel back.
    e2e = None
    if not args.no_e2e:
        pinned = {k: v.pin_memory() for k, v in host.items()}
        h_out = [(torch.empty(out_ssd.shape, dtype=out_ssd.dtype).pin_memory(),
                  torch.empty(out_att.shape, dtype=out_att.dtype).pin_memory()) for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in pinned.values())
        d2h = sum(t.numel() * t.element_size() for t in h_out[0])
        dsets = [d, {k: torch.empty_like(v) for k, v in d.items()}]
        osets = [(out_ssd, out_att), (torch.empty_like(out_ssd), torch.empty_like(out_att))]
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        started = [False, False]

        def e2e_step(i):
            j = i % 2
            if started[j]:
                s_in.wait_event(ev_cmp[j])    # step i-2 has read this input set
            with torch.cuda.stream(s_in):
                for k_, v_ in pinned.items():
                    dsets[j][k_].copy_(v_, non_blocking=True)
            ev_in[j].record(s_in)
            s_cmp.wait_event(ev_in[j])
            if started[j]:
                s_cmp.wait_event(ev_out[j])   # step i-2's outputs have left this set
            step(dsets[j], osets[j][0], osets[j][1], ws, s_cmp)
            ev_cmp[j].record(s_cmp)
            s_out.wait_event(ev_cmp[j])
            with torch.cuda.stream(s_out):
                h_out[j][0].copy_(osets[j][0], non_blocking=True)
                h_out[j][1].copy_(osets[j][1], non_blocking=True)
            ev_out[j].record(s_out)
            started[j] = True

        k_e2e = max(1, min(args.steps, args.e2e_steps))
        for i in range(min(args.warmup, 2)):
            e2e_step(i)
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(k_e2e):
            e2e_step(i)
        s_in.wait_event(ev_out[(k_e2e - 1) % 2])
        s_in.wait_event(ev_out[k_e2e % 2])
        e1.record(s_in)
        torch.cuda.synchronize()
        te = max_over_ranks(e0.elapsed_time(e1) / k_e2e, dist, dev)
        e2e = {"value": job_throughput(cfg.tokens, world, te), "unit": "Mtokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": k_e2e,
               "pipelined": "copies in, compute and copies out of consecutive steps overlap (3 streams)"}
        del dsets, osets, h_out

    result = None
    if rank == 0:
        peaks, peak_src = load_peaks()
        per_tok = algorithmic_bytes(cfg)
        # dominant kernel by time
        dom = max(phase_avg, key=lambda k: phase_avg[k])
        dom_bytes = per_tok.get(dom, 0) * cfg.tokens / launches_per_step[dom]   # per launch
        achieved = dom_bytes / (phase_launch_avg[dom] / 1e3) / 1e9
        peak = float(peaks["hbm_gbs"])
        tc_peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
        flops = mma_flops(cfg)
        dom_flops = flops.get(dom, 0) * cfg.tokens / launches_per_step[dom]
        tensor_tflops = dom_flops / (phase_launch_avg[dom] / 1e3) / 1e12
        path_bytes = (per_tok["bissd"] + per_tok["tesa"]) * cfg.tokens
        path_flops = (flops["bissd"] + flops["tesa"]) * cfg.tokens
        path_gbs = path_bytes / (ms_step / 1e3) / 1e9
        path_tflops = path_flops / (ms_step / 1e3) / 1e12
        value = job_throughput(cfg.tokens, world, ms_step)
        traffic = load_traffic(dom, cfg)
        result = {
            "metric": "MATE token-mix Mtokens/s on 1 B200 (bi-SSD+TESA)",
            "value": value,
            "unit": "Mtokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if cfg.dtype == "bf16" else "f32",
            "data": "synthetic (seeded, per rank)",
            "config": {"workload": f"{cfg.name}: grid T={cfg.T} H={cfg.H} W={cfg.W} x batch {cfg.batch}, "
                                   f"SSD {cfg.nheads}x{cfg.headdim} d_state {cfg.dstate} chunk {cfg.chunk}, "
                                   f"scan {workloads.MODE_NAMES[mode]}, review pool {cfg.review}, "
                                   f"TESA {cfg.attn_heads}x{cfg.attn_dim} window {cfg.Tw}x{cfg.Sw}x{cfg.Sw} "
                                   f"shift {cfg.shift}",
                       "tokens_per_rank": cfg.tokens, "global_tokens": cfg.tokens * world,
                       "parallelism": f"dp{world} (independent grids)",
                       "l2": f"inputs larger than L2 ({cfg.tokens * per_tok['bissd'] / 1e9:.2f} GB per bi-SSD pass "
                             f"> {L2_BYTES / 1e6:.0f} MB); no flush"},
            "phase_ms": {k: round(v, 4) for k, v in phase_avg.items()},
            "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_bytes_per_launch": dom_bytes, "launches_per_step": launches_per_step[dom],
                         "peak_source": peak_src,
                         "tensor_tflops": tensor_tflops, "tensor_peak": tc_peak,
                         "tensor_frac": tensor_tflops / tc_peak, "mma_flops_per_launch": dom_flops,
                         "path_frac": path_gbs / peak, "path_gbs": path_gbs,
                         "path_tensor_frac": path_tflops / tc_peak,
                         "path_bytes_per_step": path_bytes, "path_mma_flops_per_step": path_flops},
            "gpu_launches": int(launches),
            "clocks": clocks,
            "e2e": e2e,
        }
    return result


def time_config(cfg, mode, steps, warmup, seed=0):
    """Device time (ms) of one step of cfg in scan order `mode`, plus per-phase ms."""
    import torch

    import linear_complexity_video_b200 as mate
    from linear_complexity_video_b200 import _lib, api

    stream = torch.cuda.current_stream()
    d = {k: v.cuda() for k, v in workloads.generate(cfg, seed=seed).items()}
    out_ssd = torch.empty_like(d["x"])
    out_att = torch.empty_like(d["q"])
    ws = api.bissd_workspace(d["x"], d["B"], cfg.review, cfg.chunk)
    sdims = api.ssd_dims(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate, cfg.ngroups, cfg.chunk, cfg.torch_dtype)
    adims = api.attn_dims(cfg.batch, cfg.attn_heads, cfg.attn_dim, cfg.torch_dtype)

    def step():
        api.mate_bissd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], cfg.T, cfg.H, cfg.W, mode, cfg.review,
                           out_ssd, sdims, ws, stream)
        api.tesa_fwd(d["q"], d["k"], d["v"], cfg.T, cfg.H, cfg.W, cfg.Tw, cfg.Sw, cfg.shift, out_att, adims, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    marks = []

    def hook(phase, is_end, strm, user):
        # recorded on the stream the library launches that phase on (a phase may run
        # on the library's side stream)
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(torch.cuda.ExternalStream(strm) if strm and strm != stream.cuda_stream else stream)
        marks.append((phase, is_end, ev))

    L = mate.load()
    hook_c = _lib.PHASE_HOOK(hook)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    # one more pass with the phase hook for the per-kernel split
    L.mate_set_phase_hook(hook_c, None)
    step()
    torch.cuda.synchronize()
    L.mate_set_phase_hook(_lib.PHASE_HOOK(), None)
    phases, opened = {}, {}
    for ph, is_end, ev in marks:
        if not is_end:
            opened[ph] = ev
        else:
            name = _lib.PHASES[ph]  # summed over the launches of one step
            phases[name] = round(phases.get(name, 0.0) + opened.pop(ph).elapsed_time(ev), 4)
    if mate.mate_last_error() != 0:
        raise RuntimeError("device error word set")
    del d, out_ssd, out_att, ws
    torch.cuda.empty_cache()
    return ms, phases


def time_compose(cfg, steps, warmup, sample_rows=32):
    """mate_compose_fwd on the grid's branch outputs: (tokens, nh*P) and
    (tokens, th*td) rows to the model width. Device time from CUDA events,
    the tensor-core fraction against the burst bf16 peak (a kernel timed on its
    own), and the oracle timed on `sample_rows` rows, scaled to all rows."""
    import torch

    import linear_complexity_video_b200 as mate
    import oracle

    k1, k2, n = cfg.nheads * cfg.headdim, cfg.attn_heads * cfg.attn_dim, workloads.D_MODEL
    host = workloads.generate_compose(cfg.tokens, k1, k2, n, seed=0)
    d = {k: v.cuda() for k, v in host.items()}
    out = torch.empty(cfg.tokens, n, dtype=torch.bfloat16, device="cuda")
    for _ in range(warmup):
        mate.compose(d["y_ma"], d["y_te"], d["w_ma"], d["w_te"], out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        mate.compose(d["y_ma"], d["y_te"], d["w_ma"], d["w_te"], out=out)
    e1.record()
    torch.cuda.synchronize()
    if mate.mate_last_error() != 0:
        raise RuntimeError("device error word set")
    ms = e0.elapsed_time(e1) / steps
    flops = 2.0 * cfg.tokens * n * (k1 + k2)
    nbytes = 2.0 * (cfg.tokens * (k1 + k2) + n * (k1 + k2) + cfg.tokens * n)
    peaks, _ = load_peaks()
    tf = flops / (ms / 1e3) / 1e12
    t0 = time.perf_counter()
    oracle.get().compose(host["y_ma"][:sample_rows], host["y_te"][:sample_rows], host["w_ma"], host["w_te"])
    t_or = (time.perf_counter() - t0) * cfg.tokens / sample_rows
    del d, out
    torch.cuda.empty_cache()
    return {"report": "compose", "workload": cfg.name, "tokens": cfg.tokens, "k_ma": k1, "k_te": k2, "d_model": n,
            "ms": round(ms, 4), "tflops": round(tf, 1), "tensor_peak_burst": float(peaks["bf16_tflops"]),
            "tensor_frac": round(tf / float(peaks["bf16_tflops"]), 4),
            "hbm_frac": round(nbytes / (ms / 1e3) / 1e9 / float(peaks["hbm_gbs"]), 4),
            "mtokens_per_s": round(cfg.tokens / ms / 1e3, 2),
            "oracle_s_scaled": round(t_or, 1), "oracle_sample_rows": sample_rows}


def time_gate_norm(cfg, steps, warmup, sample_rows=256):
    """mate_gate_norm_fwd on the grid's bi-SSD output rows (tokens, nh*P), one norm group
    per row (ngroups = 1): device time from CUDA events, the HBM fraction by its
    algorithmic bytes (y and z read once, out written once), and the oracle timed on
    `sample_rows` rows, scaled to all rows."""
    import torch

    import linear_complexity_video_b200 as mate
    import oracle

    c = cfg.nheads * cfg.headdim
    group = c // cfg.ngroups
    host = workloads.generate_gate_norm(cfg.tokens, c, seed=0)
    d = {k: v.cuda() for k, v in host.items()}
    out = torch.empty(cfg.tokens, c, dtype=torch.bfloat16, device="cuda")
    for _ in range(warmup):
        mate.gate_norm(d["y"], d["z"], d["w"], group, 1e-5, out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        mate.gate_norm(d["y"], d["z"], d["w"], group, 1e-5, out=out)
    e1.record()
    torch.cuda.synchronize()
    if mate.mate_last_error() != 0:
        raise RuntimeError("device error word set")
    ms = e0.elapsed_time(e1) / steps
    nbytes = 3.0 * 2 * cfg.tokens * c + 4.0 * c
    peaks, _ = load_peaks()
    t0 = time.perf_counter()
    oracle.get().gate_norm(host["y"][:sample_rows], host["z"][:sample_rows], host["w"], group, 1e-5)
    t_or = (time.perf_counter() - t0) * cfg.tokens / sample_rows
    del d, out
    torch.cuda.empty_cache()
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"report": "gate_norm", "workload": cfg.name, "tokens": cfg.tokens, "channels": c, "group": group,
            "ms": round(ms, 4), "gbs": round(gbs, 1), "hbm_peak": float(peaks["hbm_gbs"]),
            "hbm_frac": round(gbs / float(peaks["hbm_gbs"]), 4), "mtokens_per_s": round(cfg.tokens / ms / 1e3, 2),
            "oracle_s_scaled": round(t_or, 2), "oracle_sample_rows": sample_rows}


def time_block(cfg, steps, warmup):
    """One MATE token mixer (api.block: front-end, bi-SSD, gated norm, TE-branch q/k/v
    projections, TESA, composition) on the grid with model width 2560: device time from
    CUDA events, the split by phase from the phase hook (the mean over several hooked
    calls), and the dense GEMMs' rate (in_proj, q/k/v, composition) against the burst
    bf16 peak."""
    import torch

    import linear_complexity_video_b200 as mate
    from linear_complexity_video_b200 import _lib

    host = workloads.generate_block(cfg, seed=0)
    d = {k: v.cuda() for k, v in host.items()}
    spec = dict(scan_mode=cfg.modes[0], review_pool=cfg.review, chunk=cfg.chunk, nheads=cfg.nheads,
                headdim=cfg.headdim, ngroups=cfg.ngroups, dstate=cfg.dstate, attn_heads=cfg.attn_heads,
                attn_dim=cfg.attn_dim, Tw=cfg.Tw, Sw=cfg.Sw, shift=cfg.shift)

    def call():
        return mate.block(d["u"], d, **spec)

    for _ in range(warmup):
        out = call()
    torch.cuda.synchronize()
    uuid = str(torch.cuda.get_device_properties(0).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        out = call()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / steps
    marks, stream = [], torch.cuda.current_stream()

    def hook(ph, is_end, strm, user):
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(stream)
        marks.append((ph, is_end, ev))

    hooked = max(3, steps // 2)
    L = mate.load()
    h = _lib.PHASE_HOOK(hook)
    L.mate_set_phase_hook(h, None)
    for _ in range(hooked):
        out = call()
    torch.cuda.synchronize()
    L.mate_set_phase_hook(_lib.PHASE_HOOK(), None)
    if mate.mate_last_error() != 0:
        raise RuntimeError("device error word set")
    phases, opened = {}, {}
    for ph, is_end, ev in marks:
        if not is_end:
            opened[ph] = ev
        else:
            name = _lib.PHASES[ph]
            phases[name] = phases.get(name, 0.0) + opened.pop(ph).elapsed_time(ev) / hooked
    dm = workloads.D_MODEL
    d_inner, te = cfg.nheads * cfg.headdim, cfg.attn_heads * cfg.attn_dim
    dc = d_inner + 2 * cfg.ngroups * cfg.dstate
    gemm = 2.0 * cfg.tokens * dm * ((d_inner + dc + cfg.nheads) + 3 * te + (d_inner + te))
    gemm_ms = phases.get("front_proj", 0.0) + phases.get("compose", 0.0)
    peaks, _ = load_peaks()
    del d, out
    torch.cuda.empty_cache()
    return {"report": "block", "workload": cfg.name, "scan": workloads.MODE_NAMES[cfg.modes[0]], "tokens": cfg.tokens,
            "d_model": dm, "ms": round(ms, 4), "mtokens_per_s": round(cfg.tokens / ms / 1e3, 2),
            "phase_ms": {k: round(v, 4) for k, v in phases.items()},
            "gemm_tflop": round(gemm / 1e12, 3),
            "gemm_tflops": round(gemm / (gemm_ms / 1e3) / 1e12, 1) if gemm_ms else None,
            "gemm_tensor_frac": round(gemm / (gemm_ms / 1e3) / 1e12 / float(peaks["bf16_tflops"]), 4) if gemm_ms else None,
            "gemm_tensor_frac_sustained": round(gemm / (gemm_ms / 1e3) / 1e12 / float(peaks["bf16_tflops_sustained"]), 4)
            if gemm_ms else None, "clocks": clocks}


def time_frontend(cfg, steps, warmup):
    """mate_frontend_fwd on the grid (d_model 2560 to z, x, B, C, dt): device time
    from CUDA events, the split by phase from the phase hook, the in_proj GEMMs
    against the burst bf16 peak and the conv against the HBM peak (its
    algorithmic bytes: the conv channels read once and written once)."""
    import torch

    import linear_complexity_video_b200 as mate
    from linear_complexity_video_b200 import _lib

    host = workloads.generate_frontend(cfg, seed=0)
    d = {k: v.cuda() for k, v in host.items()}
    mode = cfg.modes[0]

    def call():
        return mate.frontend(d["u"], d["w_in"], d["conv_w"], d["conv_b"], d["dt_bias"], mode, cfg.nheads,
                             cfg.headdim, cfg.ngroups, cfg.dstate)

    for _ in range(warmup):
        outs = call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        outs = call()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    marks, stream = [], torch.cuda.current_stream()

    def hook(ph, is_end, strm, user):
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(stream)
        marks.append((ph, is_end, ev))

    # the phase split: the mean over several hooked calls (one call's split varies
    # with the clock the GEMMs start at)
    hooked = max(3, steps // 2)
    L = mate.load()
    h = _lib.PHASE_HOOK(hook)
    L.mate_set_phase_hook(h, None)
    for _ in range(hooked):
        outs = call()
    torch.cuda.synchronize()
    L.mate_set_phase_hook(_lib.PHASE_HOOK(), None)
    if mate.mate_last_error() != 0:
        raise RuntimeError("device error word set")
    phases, opened = {}, {}
    for ph, is_end, ev in marks:
        if not is_end:
            opened[ph] = ev
        else:
            name = _lib.PHASES[ph]
            phases[name] = phases.get(name, 0.0) + opened.pop(ph).elapsed_time(ev) / hooked
    d_inner = cfg.nheads * cfg.headdim
    dc = d_inner + 2 * cfg.ngroups * cfg.dstate
    rows = d_inner + dc + cfg.nheads
    conv_bytes = 2.0 * cfg.tokens * dc * 2
    peaks, _ = load_peaks()
    conv = phases.get("front_conv", 0.0)
    # the in_proj GEMMs timed on their own without the hook (its events add host latency
    # inside each phase): the z and conv-channel GEMMs the front-end makes (99% of its
    # in_proj flops; the 80-row dt GEMM is left out, its width is no multiple of 64)
    u2 = d["u"].view(-1, workloads.D_MODEL)
    parts = [d["w_in"][:d_inner], d["w_in"][d_inner:d_inner + dc]]
    gemm_flops = 2.0 * cfg.tokens * workloads.D_MODEL * (d_inner + dc)
    scratch = [torch.empty(u2.shape[0], w.shape[0], dtype=torch.bfloat16, device="cuda") for w in parts]

    def gemms():
        for w, o in zip(parts, scratch):
            mate.linear(u2, w, out=o)

    for _ in range(warmup):
        gemms()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        gemms()
    e1.record()
    torch.cuda.synchronize()
    proj = e0.elapsed_time(e1) / steps
    del d, outs, scratch
    torch.cuda.empty_cache()
    return {"report": "frontend", "workload": cfg.name, "scan": workloads.MODE_NAMES[mode], "tokens": cfg.tokens,
            "d_model": workloads.D_MODEL, "in_proj_rows": rows, "ms": round(ms, 4),
            "phase_ms": {k: round(v, 4) for k, v in phases.items()},
            "in_proj_zx_ms": round(proj, 4),
            "in_proj_tflops": round(gemm_flops / (proj / 1e3) / 1e12, 1) if proj else None,
            "in_proj_tensor_frac": round(gemm_flops / (proj / 1e3) / 1e12 / float(peaks["bf16_tflops"]), 4)
            if proj else None,
            "conv_hbm_frac": round(conv_bytes / (conv / 1e3) / 1e9 / float(peaks["hbm_gbs"]), 4) if conv else None,
            "mtokens_per_s": round(cfg.tokens / ms / 1e3, 2)}


def run_report(args):
    """Every bf16 grid in every scan order it lists, the headline grid in the
    zigzag comparison order, then the N sweep with a linearity fit. One JSON
    line per measurement, then a summary line."""
    import numpy as np
    import torch

    peaks, _ = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    for name, cfg in workloads.CONFIGS.items():
        if cfg.dtype != "bf16":
            continue
        for mode in cfg.modes:
            ms, phases = time_config(cfg, mode, args.steps, args.warmup)
            per_tok = algorithmic_bytes(cfg)
            path_bytes = (per_tok["bissd"] + per_tok["tesa"]) * cfg.tokens
            print(json.dumps({"report": "config", "workload": name, "scan": workloads.MODE_NAMES[mode],
                              "tokens": cfg.tokens, "ms_per_step": round(ms, 4),
                              "mtokens_per_s": round(cfg.tokens / ms / 1e3, 3),
                              "path_hbm_frac": round(path_bytes / (ms / 1e3) / 1e9 / hbm, 4),
                              "phase_ms": phases}), flush=True)
    # the pages' scan ablation (paper review 5.5 Table 2: Zigzag instead of RMS) at kernel
    # level: the headline grid in its RMS order and in the zigzag comparison order
    cfg = workloads.CONFIGS[workloads.HEADLINE]
    ms_rms, ph_rms = time_config(cfg, cfg.modes[0], args.steps, args.warmup)
    ms_zz, ph_zz = time_config(cfg, workloads.ZZ, args.steps, args.warmup)
    print(json.dumps({"report": "scan_ablation", "workload": cfg.name, "tokens": cfg.tokens,
                      "rms_scan": workloads.MODE_NAMES[cfg.modes[0]], "rms_ms_per_step": round(ms_rms, 4),
                      "zigzag_ms_per_step": round(ms_zz, 4), "zigzag_over_rms": round(ms_zz / ms_rms, 4),
                      "rms_phase_ms": ph_rms, "zigzag_phase_ms": ph_zz}), flush=True)
    # the MATE composition (projections of both branches to the model width, summed) on
    # the headline grid, against the tensor-core roofline; the oracle on a row sample
    print(json.dumps(time_compose(cfg, args.steps, args.warmup)), flush=True)
    print(json.dumps(time_frontend(cfg, args.steps, args.warmup)), flush=True)
    print(json.dumps(time_gate_norm(cfg, args.steps, args.warmup)), flush=True)
    print(json.dumps(time_block(cfg, args.steps, args.warmup)), flush=True)
    Ns, ts = [], []
    for cfg in workloads.sweep_configs():
        ms, phases = time_config(cfg, cfg.modes[0], args.steps, args.warmup)
        per_tok = algorithmic_bytes(cfg)
        path_bytes = (per_tok["bissd"] + per_tok["tesa"]) * cfg.tokens
        Ns.append(cfg.tokens)
        ts.append(ms)
        print(json.dumps({"report": "sweep", "workload": cfg.name, "tokens": cfg.tokens, "ms_per_step": round(ms, 4),
                          "mtokens_per_s": round(cfg.tokens / ms / 1e3, 3),
                          "path_hbm_frac": round(path_bytes / (ms / 1e3) / 1e9 / hbm, 4), "phase_ms": phases}),
              flush=True)
    N = np.array(Ns, dtype=np.float64)
    t = np.array(ts, dtype=np.float64)
    slope, icpt = np.polyfit(N, t, 1)
    pred = slope * N + icpt
    r2 = 1.0 - float(np.sum((t - pred) ** 2) / np.sum((t - t.mean()) ** 2))
    rate = N / t / 1e3
    big = rate[N >= 32768]
    spread = float(np.max(np.abs(big / np.median(big) - 1.0))) if len(big) else None
    print(json.dumps({"report": "linearity", "fit": "t_ms = a + b*N", "a_ms": round(float(icpt), 5),
                      "b_ns_per_token": round(float(slope) * 1e6, 4), "r2": round(r2, 5),
                      "max_rel_dev_mtokens_per_s_N_ge_32k": round(spread, 4) if spread is not None else None}),
          flush=True)


def load_traffic(kernel, cfg):
    """DRAM bytes per launch of `kernel` from profiles/traffic.txt, if a line
    matches the workload and the kernel's source file is unchanged since the
    capture; else None."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    for ln in lines:
        if not ln.strip() or ln.lstrip().startswith("#"):
            continue
        f = ln.split()
        if len(f) < 5 or f[0] != kernel or f[1] != cfg.name:
            continue
        try:
            sha = hashlib.sha1(open(os.path.join(ROOT, f[3]), "rb").read()).hexdigest()
        except OSError:
            return None
        return int(f[2]) if sha == f[4] else None
    return None


def run_reference(args, cfg):
    """The oracle, timed on the host cores, one bounded sample per step."""
    vals = []
    cores = None
    desc = ""
    for _ in range(args.warmup_ref):
        oracle_sample(cfg)
    for _ in range(args.steps_ref):
        v, cores, desc = oracle_sample(cfg)
        vals.append(v)
    value = statistics.median(vals)
    return {
        "impl": "reference",
        "metric": "MATE token-mix Mtokens/s on 1 B200 (bi-SSD+TESA)",
        "value": value,
        "unit": "Mtokens/s",
        "n_gpus": 1,
        "steps": len(vals),
        "warmup": args.warmup_ref,
        "ms_per_step": cfg.tokens / (value * 1e6) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": f"{cfg.name}: grid T={cfg.T} H={cfg.H} W={cfg.W} x batch {cfg.batch}"},
        "cpu_baseline": {"value": value, "unit": "Mtokens/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "Mtokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def spawn_ranks(args) -> int:
    """--gpus N without an outside launcher: start N ranks of this script on
    this node through torch.distributed.run (one process per GPU) and return
    its exit status. The GPU arm needs N visible devices."""
    import socket

    n = args.gpus
    if args.impl == "mate":
        import torch

        have = torch.cuda.device_count()
        if have < n:
            print(f"bench.py: --gpus {n} needs {n} CUDA devices, {have} visible", file=sys.stderr)
            return 2
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def join_ranks(rank: int, world: int) -> int:
    """Reference arm under N ranks: every rank checks in over a CPU (gloo)
    group, then all but rank 0 leave; rank 0 alone times the oracle.
    Returns the number of ranks that checked in."""
    if world <= 1:
        return 1
    import datetime

    import torch.distributed as tdist

    tdist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    seen = [None] * world
    tdist.all_gather_object(seen, rank)
    tdist.destroy_process_group()
    if rank != 0:
        print(f"bench.py rank {rank}/{world}: reference arm runs on rank 0 only", file=sys.stderr, flush=True)
    return len(set(seen))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=workloads.HEADLINE, choices=sorted(workloads.CONFIGS))
    ap.add_argument("--impl", default="mate", choices=["mate", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--chunk", type=int, default=0, help="override the scan chunk length (a tiling choice)")
    ap.add_argument("--report", action="store_true",
                    help="time every bf16 grid in each of its scan orders and the N sweep (one JSON line each)")
    ap.add_argument("--component", choices=["compose", "frontend", "gate_norm", "block"],
                    help="time one component beside the token mix on --config (one JSON line)")
    ap.add_argument("--steps-ref", type=int, default=1)
    ap.add_argument("--warmup-ref", type=int, default=0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = workloads.CONFIGS[args.config]
    if args.chunk:
        cfg = cfg.with_(chunk=args.chunk)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(spawn_ranks(args))
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if world != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}")

    if args.impl == "reference":
        joined = join_ranks(rank, world)
        if rank == 0:
            res = run_reference(args, cfg)
            res["n_gpus"] = world
            if world > 1:
                res["ranks_joined"] = joined
            print(json.dumps(res), flush=True)
        return
    if args.report:
        run_report(args)
        return
    if args.component:
        fn = {"compose": time_compose, "frontend": time_frontend, "gate_norm": time_gate_norm,
              "block": time_block}[args.component]
        print(json.dumps(fn(cfg, args.steps, args.warmup)), flush=True)
        return

    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        res = run_mate(args, cfg, rank, world, dist)
        if rank == 0:
            if not args.no_cpu_baseline and world == 1:
                v, cores, desc = oracle_sample(cfg)
                res["cpu_baseline"] = {"value": v, "unit": "Mtokens/s", "cores": cores, "kind": "oracle",
                                       "sample": desc}
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
