#!/usr/bin/env python
"""Benchmark of the SDM memory pass on B200.

Headline: prefill of the long skewed workload (B=1, H=4, T=262144, N=1048576 = 1024 x 1024,
W=R=64, d_v=256, bf16 inputs, fp32 state) -- one step is one sdm_scan_forward call doing
every step of the pass: M0 broadcast, product-key selection, sparse gated delta write,
sparse read and RMSNorm + gate.  Reported as token*heads/s (whole job), beside the HBM
roofline of the scan kernel, the end-to-end figure through the C ABI with host buffers,
and the CPU oracle timed on the host cores.  A second object reports decode on the
batched-decode workload (64 sequences x 8 heads, N=262144, d_v=128): 256 successive
sdm_decode_step_chained calls over inputs staged on the device beforehand (each step's
selection may overlap the step before), as plain launches and replayed from a CUDA graph.

Multi-GPU: the pass has no exchange step (every (sequence, head) is independent), so each
rank runs its own batch of the same shape (weak scaling), timed between barriers and
reduced as the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sdm|reference]
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import sdm_synth  # noqa: E402

METRIC = "SDM layer tokens*heads/s (prefill & decode) and HBM GB/s as % of B200 peak"
UNIT = "token*heads/s"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------- helpers
def algorithmic_bytes(wl) -> int:
    """Bytes per token-head the pass must move: the W rows read and rewritten and the R
    rows read (fp32 state), both score halves and v.  Gate, alpha/beta, y/o and the
    selection scratch are not counted."""
    s_in = 2 if wl.in_dtype == torch.bfloat16 else 4
    return (2 * wl.W + wl.R) * wl.d_v * 4 + 2 * (wl.S1 + wl.S2) * s_in + wl.d_v * s_in



def measured_traffic(kernel: str, units: float, unit_key: str):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, scaled to `units`
    units (token-heads or (b, h) pairs) per launch; None once the kernel's source no longer
    has the hash the capture was taken with."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[kernel]
        src = open(os.path.join(ROOT, rec["source"]), "rb").read()
    except (OSError, KeyError, ValueError):
        return None
    if hashlib.sha256(src).hexdigest()[:16] != rec["source_sha256_16"]:
        return None
    return rec[unit_key] * units

def scan_kernel_bytes(wl) -> int:
    """Bytes per token-head of the scan engine alone: the state rows only."""
    return (2 * wl.W + wl.R) * wl.d_v * 4


def hbm_peak():
    try:
        with open(PEAKS_PATH) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class Dist:
    """torch.distributed plumbing: barrier and max over ranks (nccl on GPUs, gloo on CPU)."""

    def __init__(self, backend: str | None = None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import torch.distributed as dist
            if backend is None:
                backend = "nccl" if torch.cuda.is_available() else "gloo"
            self.backend = backend
            if backend == "nccl":
                torch.cuda.set_device(self.local_rank)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", self.local_rank)
                                    if backend == "nccl" else None)
            self.pg = dist

    def _dev(self):
        if self.pg is not None and self.backend == "nccl":
            return torch.device("cuda", self.local_rank)
        return torch.device("cpu")

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self._dev())
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def sum(self, x: float) -> float:
        if self.pg is None:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self._dev())
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()
            self.pg = None


def weak_scaling_value(units_per_rank: float, max_seconds: float, world: int) -> float:
    """Whole-job throughput: every rank processed units_per_rank in at most max_seconds."""
    return units_per_rank * world / max_seconds


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.05):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # clocks are reported as unavailable, never guessed
            self.nv = None
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
                r = get(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def report(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        busy = [s for s in self.samples]
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def timed(fn, steps: int, warmup: int, dist: Dist, stream, after_warmup=None):
    """Runs fn warmup times untimed, then times exactly `steps` calls with CUDA events on
    `stream`, bracketed by barrier + synchronize.  Returns max-over-ranks seconds.
    after_warmup() runs between the two (e.g. to start per-kernel timing)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if after_warmup is not None:
        after_warmup()
    dist.barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    return dist.max(a.elapsed_time(b) / 1e3)


# ----------------------------------------------------------------- the CUDA path
def bench_prefill(args, dist: Dist, dev):
    import sparse_memory_linear_b200 as sdm

    wl = sdm_synth.WORKLOADS[args.workload]
    stream = torch.cuda.current_stream(dev)
    g = {k: v.to(dev) for k, v in sdm_synth.make_inputs(wl, device=dev).items()}
    torch.cuda.synchronize()
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=torch.float32, device=dev)
    shape = sdm.shape_of(wl.B, wl.T, wl.H, wl.S1, wl.S2, wl.W, wl.R, wl.d_v,
                         sdm.SDM_BF16 if wl.in_dtype == torch.bfloat16 else sdm.SDM_F32)
    ws = torch.empty(sdm.sdm_workspace_size(shape), dtype=torch.uint8, device=dev)
    y = torch.empty((wl.B, wl.T, wl.H, wl.d_v), dtype=torch.float32, device=dev)
    o = torch.empty_like(y)

    # One step is the pass over the T tokens from the state the last step left (SDM_CONTINUE):
    # selection, scan engine and norm/gate.  The M0 broadcast (a3) is timed on its own.
    def step():
        sdm.sdm_scan_forward(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M, W=wl.W,
                             R=wl.R, S1=wl.S1, init="continue", gate=g["gate"], y=y,
                             o=o, ws=ws, stream=stream)

    marks = {}

    def start_timing():
        marks["launches"] = sdm.sdm_launch_count()

    sdm.sdm_state_init(g["M0"], M)
    with ClockSampler(dev.index) as clk:
        secs = timed(step, args.steps, args.warmup, dist, stream, after_warmup=start_timing)
    launched = sdm.sdm_launch_count() - marks["launches"]
    # one more step with the library's per-launch events for the per-kernel split
    sdm.sdm_profile_enable(True)
    step()
    torch.cuda.synchronize(dev)
    prof = sdm.sdm_profile_read()
    sdm.sdm_profile_enable(False)
    if sdm.sdm_get_device_status() != 0:
        raise RuntimeError("device status word set during the benchmark")
    init_secs = timed(lambda: sdm.sdm_state_init(g["M0"], M), 3, 1, dist, stream)

    th = wl.B * wl.T * wl.H
    value = weak_scaling_value(th * args.steps, secs, dist.world)
    # per-kind device time per step and launches per step (events on the launching stream)
    ms_step = {k: ms for k, (ms, n) in prof.items() if n}
    n_step = {k: n for k, (ms, n) in prof.items() if n}
    scan_kind = "scan_slot" if prof["scan_slot"][1] else "scan_seq"
    peak, peak_kind = hbm_peak()
    # the scan kernel runs once per time chunk (slot engine) or once per step: bytes per
    # launch = the step's algorithmic bytes over its launches, duration = the average launch
    scan_bytes = th * scan_kernel_bytes(wl)
    per_launch_bytes = scan_bytes / n_step[scan_kind]
    per_launch_ms = ms_step[scan_kind] / n_step[scan_kind]
    achieved = per_launch_bytes / (per_launch_ms * 1e-3) / 1e9
    step_ms = secs / args.steps * 1e3
    res = {
        "value": value,
        "ms_per_step": step_ms,
        "clocks": clk.report(),
        "state_init_ms": init_secs / 3 * 1e3,
        "kernels_ms_per_step": ms_step,
        "kernel_launches_per_step": n_step,
        "kernels_share": {k: ms_step[k] / sum(ms_step.values()) for k in ms_step},
        "select_schedule": (
            "serial: the whole selection, then the chunks" if args.select_schedule == "serial"
            else "pipelined (the library's default): with more than one time chunk, chunk "
                 "c+1's selection runs on a low-priority stream beside chunk c's sort and scan, "
                 "so the per-kernel times overlap and add up to more than the step"),
        "gpu_launches": int(launched),
        "roofline": {
            "kernel": f"seq_scan_kernel" if scan_kind == "scan_seq" else "slot_chunk_kernel",
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_kind": f"{peak_kind} (burst copy)",
            "traffic": (measured_traffic("slot_chunk_kernel", th / n_step[scan_kind],
                                         "dram_bytes_per_token_head")
                        if scan_kind == "scan_slot" else None),
            "algorithmic_bytes_per_launch": per_launch_bytes,
            "launch_ms": per_launch_ms,
            "launches_per_step": n_step[scan_kind],
            "bytes_per_token_head": scan_kernel_bytes(wl),
        },
        "whole_step_hbm": {
            "bytes_per_token_head": algorithmic_bytes(wl),
            "GBps": th * algorithmic_bytes(wl) / (step_ms * 1e-3) / 1e9,
        },
    }

    # end to end through the same call with host buffers: inputs copied in from pinned
    # host memory and the layer output copied back, every step
    if not args.no_e2e:
        host = {k: torch.empty_like(g[k], device="cpu").pin_memory().copy_(g[k])
                for k in ("kp", "qp", "v", "alpha", "beta", "gate")}
        o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o_host.numel() * o_host.element_size()

        def step_e2e():
            for k, t in host.items():
                g[k].copy_(t, non_blocking=True)
            step()
            o_host.copy_(o, non_blocking=True)

        secs_e = timed(step_e2e, max(1, min(args.steps, 3)), 1, dist, stream)
        res["e2e"] = {"value": weak_scaling_value(th * max(1, min(args.steps, 3)), secs_e,
                                                  dist.world),
                      "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        del host, o_host
    res["_inputs"] = (wl, g)
    return res


PREFILL_CONFIGS = ("small", "layer1p4b")


def bench_prefill_configs(args, dist: Dist, dev):
    """The other prefill workloads: the AUTO engine's step and every engine's step, each
    timed alone with CUDA events (median of the timed steps) after a write of twice the L2
    size (the small workload's inputs and state fit in L2).  One step is one
    sdm_scan_forward with SDM_CONTINUE, as in the headline."""
    import sparse_memory_linear_b200 as sdm

    stream = torch.cuda.current_stream(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 64 << 20), dtype=torch.uint8, device=dev)
    peak, peak_kind = hbm_peak()
    out = []
    for name in PREFILL_CONFIGS:
        wl = sdm_synth.WORKLOADS[name]
        g = {k: v.to(dev) for k, v in sdm_synth.make_inputs(wl, device=dev).items()}
        M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=torch.float32, device=dev)
        sdm.sdm_state_init(g["M0"], M)
        y = torch.empty((wl.B, wl.T, wl.H, wl.d_v), dtype=torch.float32, device=dev)
        o = torch.empty_like(y)
        ms = {}
        for engine in ("auto", "seq", "slot", "chunk"):
            def step():
                sdm.sdm_scan_forward(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M,
                                     W=wl.W, R=wl.R, S1=wl.S1, init="continue", gate=g["gate"],
                                     y=y, o=o, engine=engine, stream=stream)
            for _ in range(args.warmup):
                step()
            times = []
            for _ in range(max(3, args.steps)):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                step()
                b.record(stream)
                torch.cuda.synchronize(dev)
                times.append(a.elapsed_time(b))
            ms[engine] = dist.max(statistics.median(times))
        sdm.sdm_profile_enable(True)
        sdm.sdm_scan_forward(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M, W=wl.W,
                             R=wl.R, S1=wl.S1, init="continue", gate=g["gate"], y=y, o=o,
                             stream=stream)
        torch.cuda.synchronize(dev)
        prof = sdm.sdm_profile_read()
        sdm.sdm_profile_enable(False)
        if sdm.sdm_get_device_status() != 0:
            raise RuntimeError("device status word set during the benchmark")
        th = wl.B * wl.T * wl.H
        step_s = ms["auto"] * 1e-3
        out.append({
            "workload": wl.name, "shape": wl.note, "metric": METRIC, "unit": UNIT,
            "value": weak_scaling_value(th, step_s, dist.world), "ms_per_step": ms["auto"],
            "engine": "slot" if prof["scan_slot"][1] else "seq",
            "engine_ms_per_step": {"seq": ms["seq"], "slot": ms["slot"], "chunk": ms["chunk"]},
            "whole_step_hbm": {"bytes_per_token_head": algorithmic_bytes(wl),
                               "GBps": th * algorithmic_bytes(wl) / step_s / 1e9,
                               "frac": th * algorithmic_bytes(wl) / step_s / 1e9 / peak,
                               "peak": peak, "peak_kind": peak_kind},
            "kernels_ms_per_step": {k: v for k, (v, n) in prof.items() if n},
            "l2": "flushed before every timed step (a write of twice the L2 size)",
        })
        del g, M, y, o
        torch.cuda.empty_cache()
    return out


def bench_balance(args, dev):
    """Load balance of the slot engine: one step of the prefill workload (with --override
    applied) with the library's per-CTA work counters on (sdm_slot_cta_stats), after W
    warm-up steps.  Reports events, spans and busy time per CTA (min, median, max, mean,
    max/mean); busy time is the mean over a CTA's eight warps."""
    import sparse_memory_linear_b200 as sdm

    wl = sdm_synth.WORKLOADS[args.workload]
    g = {k: v.to(dev) for k, v in sdm_synth.make_inputs(wl, device=dev).items()}
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=torch.float32, device=dev)
    sdm.sdm_state_init(g["M0"], M)

    def step():
        sdm.sdm_scan_forward(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M, W=wl.W,
                             R=wl.R, S1=wl.S1, init="continue", gate=g["gate"], engine="slot")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    sdm.sdm_slot_cta_stats(reset=True)
    sdm.sdm_set_option("slot_cta_stats", 1)
    try:
        step()
    finally:
        sdm.sdm_set_option("slot_cta_stats", 0)
    st = sdm.sdm_slot_cta_stats(reset=True)
    sdm.sdm_profile_enable(True)
    step()
    torch.cuda.synchronize(dev)
    prof = sdm.sdm_profile_read()
    sdm.sdm_profile_enable(False)
    active = st[st[:, 3] > 0]
    ev = active[:, 0] + active[:, 1]

    def q(x):
        x = np.asarray(x, np.float64)
        return {"min": float(x.min()), "p50": float(np.median(x)), "max": float(x.max()),
                "mean": float(x.mean()), "max_over_mean": float(x.max() / max(x.mean(), 1e-9))}

    return {"workload": wl.name, "shape": wl.note, "ctas": int(active.shape[0]),
            "chunk_launches": int(prof["scan_slot"][1]),
            "scan_ms": prof["scan_slot"][0], "events_total": int(ev.sum()),
            "events_in_long_segments": int(active[:, 1].sum()),
            "events_per_cta": q(ev), "short_events_per_cta": q(active[:, 0]),
            "long_events_per_cta": q(active[:, 1]), "spans_per_cta": q(active[:, 2]),
            "busy_us_per_cta": q(active[:, 3] / 8.0 / 1e3)}


def bench_state_rows(args, dist: Dist, dev):
    """State checkpoints of the long skewed layer (M: 4 heads x 2^20 slots x 256 fp32, 4 GB,
    larger than L2): sdm_state_pack and sdm_state_unpack per format, each timed alone with
    CUDA events (median of 5 after 3 warm-ups).  HBM bytes per call: the fp32 rows plus the
    codes plus the per-row scales, each once."""
    import sparse_memory_linear_b200 as sdm

    torch.cuda.empty_cache()  # the parts before may leave tens of GB cached
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = hbm_peak()
    wl = sdm_synth.WORKLOADS[args.workload]
    gen = torch.Generator(device=dev).manual_seed(0x5D3)
    M = torch.randn((wl.B * wl.H * wl.N, wl.d_v), generator=gen, device=dev) * 0.02
    back = torch.empty_like(M)
    rows = M.shape[0]
    out = {"workload": f"{wl.name} state, {rows} rows x {wl.d_v} fp32 ({M.numel() * 4 >> 20} MiB)"}
    for fmt in ("bf16", "e4m3", "int4"):
        codes, scales = sdm.sdm_state_pack(M, fmt)
        code_bytes = codes.numel() * codes.element_size()
        scale_bytes = 0 if scales is None else rows * 4
        io = M.numel() * 4 + code_bytes + scale_bytes
        res = {"code_bytes": code_bytes, "scale_bytes": scale_bytes}
        for name, fn in (("pack", lambda: sdm.sdm_state_pack(M, fmt, codes=codes, scales=scales)),
                         ("unpack", lambda: sdm.sdm_state_unpack(codes, scales, wl.d_v, fmt,
                                                                 out=back))):
            ts = []
            for i in range(8):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                torch.cuda.synchronize(dev)
                if i >= 3:
                    ts.append(a.elapsed_time(b))
            ms = float(np.median(ts))
            gbps = io / (ms * 1e-3) / 1e9
            res[name] = {"ms": ms, "GBps": gbps, "frac": gbps / peak}
        out[fmt] = res
    out["peak"] = peak
    out["peak_kind"] = f"{peak_kind} (burst copy)"
    if sdm.sdm_get_device_status() != 0:
        raise RuntimeError("device status word set during the checkpoint benchmark")
    del M, back
    torch.cuda.empty_cache()
    return out


def bench_undo(args, dist: Dist, dev):
    """The logged prefill (sdm_scan_forward_logged: the step plus its undo log, W rows of
    d_v fp32 per token-head) and the undo (sdm_state_undo) on the prefill workload, each
    timed with CUDA events (median of 3 after 3 warm-ups); the undo restores the state after
    every logged step, so each logged step starts from the same state."""
    import sparse_memory_linear_b200 as sdm

    torch.cuda.empty_cache()  # the parts before may leave tens of GB cached
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = hbm_peak()
    wl = sdm_synth.WORKLOADS[args.workload]
    g = {k: v.to(dev) for k, v in sdm_synth.make_inputs(wl, device=dev).items()}
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=torch.float32, device=dev)
    sdm.sdm_state_init(g["M0"], M)
    shape = sdm.shape_of(wl.B, wl.T, wl.H, wl.S1, wl.S2, wl.W, wl.R, wl.d_v,
                         sdm.SDM_BF16 if wl.in_dtype == torch.bfloat16 else sdm.SDM_F32)
    ws = torch.empty(sdm.sdm_workspace_size(shape), dtype=torch.uint8, device=dev)
    ws_u = torch.empty(sdm.sdm_undo_workspace_size(shape), dtype=torch.uint8, device=dev)
    y = torch.empty((wl.B, wl.T, wl.H, wl.d_v), dtype=torch.float32, device=dev)
    o = torch.empty_like(y)
    sel = torch.empty(wl.B * wl.T * wl.H * (wl.W + wl.R), dtype=torch.int32, device=dev)
    wlog = torch.empty((wl.B, wl.T, wl.H, wl.W, wl.d_v), dtype=torch.float32, device=dev)
    M_start = M.clone()

    def logged():
        sdm.sdm_scan_forward_logged(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M,
                                    W=wl.W, R=wl.R, S1=wl.S1, init="continue", gate=g["gate"],
                                    y=y, o=o, sel_out=sel, ws=ws, wlog=wlog, stream=stream)

    def undo():
        sdm.sdm_state_undo(M, sel, wlog, W=wl.W, S1=wl.S1, ws=ws_u, stream=stream)

    t_log, t_undo = [], []
    for i in range(6):
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(stream)
        logged()
        b.record(stream)
        undo()
        c.record(stream)
        torch.cuda.synchronize(dev)
        if i >= 3:
            t_log.append(a.elapsed_time(b))
            t_undo.append(b.elapsed_time(c))
    restored = bool(torch.equal(M, M_start))
    if sdm.sdm_get_device_status() != 0:
        raise RuntimeError("device status word set during the undo benchmark")
    th = wl.B * wl.T * wl.H
    log_bytes = wlog.numel() * 4
    ms = float(np.median(t_log))
    step_bytes = th * algorithmic_bytes(wl) + log_bytes
    out = {"workload": wl.name, "logged_ms_per_step": ms,
           "logged_value": th / (ms * 1e-3), "unit": UNIT,
           "log_bytes_per_step": log_bytes,
           "logged_whole_step_hbm": {"bytes_per_token_head": step_bytes / th,
                                     "GBps": step_bytes / (ms * 1e-3) / 1e9,
                                     "frac": step_bytes / (ms * 1e-3) / 1e9 / peak},
           "undo_ms": float(np.median(t_undo)),
           "undo_restored_state_bit_for_bit": restored,
           "peak_kind": peak_kind}
    del g, wlog, ws, ws_u, M, M_start, y, o, sel
    torch.cuda.empty_cache()
    return out


def bench_coupled(args, dist: Dist, dev):
    """The coupled delta rule: prefill of the 1.4B-like workload (sequential engine, the one
    that computes it) and 256 chained decode steps of the batched-decode workload, timed as
    the per-slot lines are."""
    import sparse_memory_linear_b200 as sdm

    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = hbm_peak()
    wl = sdm_synth.WORKLOADS["layer1p4b"]
    g = {k: v.to(dev) for k, v in sdm_synth.make_inputs(wl, device=dev).items()}
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=torch.float32, device=dev)
    sdm.sdm_state_init(g["M0"], M)
    y = torch.empty((wl.B, wl.T, wl.H, wl.d_v), dtype=torch.float32, device=dev)
    o = torch.empty_like(y)

    def step():
        sdm.sdm_scan_forward_coupled(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M,
                                     W=wl.W, R=wl.R, S1=wl.S1, init="continue", gate=g["gate"],
                                     y=y, o=o, stream=stream)

    steps = max(3, args.steps)
    secs = timed(step, steps, args.warmup, dist, stream)
    th = wl.B * wl.T * wl.H
    step_s = secs / steps
    pre = {"workload": wl.name, "shape": wl.note, "engine": "seq",
           "value": weak_scaling_value(th, step_s, dist.world), "unit": UNIT,
           "ms_per_step": step_s * 1e3,
           "whole_step_hbm_frac": th * algorithmic_bytes(wl) / step_s / 1e9 / peak}
    del g, M, y, o
    torch.cuda.empty_cache()

    wl = sdm_synth.WORKLOADS[args.decode_workload]
    steps_in = [{k: t.to(dev) for k, t in sdm_synth.make_inputs(wl, device=dev, step=s).items()}
                for s in range(wl.T)]
    M0 = steps_in[0].pop("M0")
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=torch.float32, device=dev)
    sdm.sdm_state_init(M0, M)
    yd = torch.empty((wl.B, wl.H, wl.d_v), dtype=torch.float32, device=dev)
    od = torch.empty_like(yd)

    def run_all():
        for s in steps_in:
            sdm.sdm_decode_step(s["kp"], s["qp"], s["v"], s["alpha"], s["beta"], M, W=wl.W,
                                R=wl.R, S1=wl.S1, gate=s["gate"], y=yd, o=od, stream=stream,
                                chained=True, coupled=True)

    reps = max(1, args.steps // 2)
    secs = timed(run_all, reps, 1, dist, stream)
    per_step = secs / (reps * wl.T)
    dec = {"workload": wl.note, "launch": "sdm_decode_step_coupled_chained",
           "us_per_step": per_step * 1e6, "value": weak_scaling_value(wl.B * wl.H, per_step,
                                                                       dist.world),
           "unit": UNIT, "step_roofline_frac": step_bytes_of(wl) / per_step / 1e9 / peak}
    if sdm.sdm_get_device_status() != 0:
        raise RuntimeError("device status word set during the coupled benchmark")
    del M, steps_in
    torch.cuda.empty_cache()
    return {"rule": "coupled delta (one prediction shared by the written rows)",
            "prefill": pre, "decode": dec, "peak_kind": peak_kind}


def step_bytes_of(wl) -> float:
    """Algorithmic bytes of one decode step of every (sequence, head)."""
    return wl.B * wl.H * algorithmic_bytes(wl)


def per_step_of(secs: float, reps: int, nsteps: int) -> float:
    return secs / (reps * nsteps)


def bench_decode(args, dist: Dist, dev):
    import sparse_memory_linear_b200 as sdm

    wl = sdm_synth.WORKLOADS[args.decode_workload]
    stream = torch.cuda.current_stream(dev)
    nsteps = wl.T
    steps = [{k: t.to(dev) for k, t in sdm_synth.make_inputs(wl, device=dev, step=s).items()}
             for s in range(nsteps)]
    M0 = steps[0].pop("M0")
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=torch.float32, device=dev)
    sdm.sdm_state_init(M0, M)
    y = torch.empty((wl.B, wl.H, wl.d_v), dtype=torch.float32, device=dev)
    o = torch.empty_like(y)

    def run_all():
        for s in steps:
            sdm.sdm_decode_step(s["kp"], s["qp"], s["v"], s["alpha"], s["beta"], M, W=wl.W,
                                R=wl.R, S1=wl.S1, gate=s["gate"], y=y, o=o, stream=stream,
                                chained=True)

    reps = max(1, args.steps // 2)
    # plain launches, timed without the library's per-launch events (these would sit between
    # consecutive steps and serialise them)
    secs = timed(run_all, reps, 1, dist, stream)
    # one more pass with per-launch events for the kernel's own duration
    sdm.sdm_profile_enable(True)
    run_all()
    torch.cuda.synchronize(dev)
    prof = sdm.sdm_profile_read()
    sdm.sdm_profile_enable(False)
    ms_k, n_k = prof["decode"]
    per_step = secs / (reps * nsteps)
    th = wl.B * wl.H
    peak, peak_kind = hbm_peak()
    step_bytes = th * algorithmic_bytes(wl)
    kernel_s = ms_k / n_k * 1e-3
    out = {
        "workload": wl.note, "steps_per_run": nsteps, "runs": reps,
        "launch": "sdm_decode_step_chained (programmatic stream serialisation)",
        # the step's algorithmic bytes over the step time: consecutive steps overlap (the
        # selection of a step runs while the step before it drains), so this is above the
        # per-kernel fraction of `roofline`, whose duration is a launch timed alone
        "step_roofline_frac": step_bytes_of(wl) / per_step_of(secs, reps, nsteps) / 1e9 / hbm_peak()[0],
        "value": weak_scaling_value(th, per_step, dist.world), "unit": UNIT,
        "us_per_step": per_step * 1e6,
        "roofline": {"kernel": "decode_kernel", "bound": "hbm",
                     "achieved": step_bytes / kernel_s / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": step_bytes / kernel_s / 1e9 / peak,
                     "peak_kind": f"{peak_kind} (burst copy)",
                     "algorithmic_bytes_per_launch": step_bytes, "kernel_us": kernel_s * 1e6,
                     "traffic": measured_traffic("decode_kernel", wl.B * wl.H,
                                                 "dram_bytes_per_unit")},
    }
    # the same 256 steps captured once into a CUDA graph and replayed
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            run_all()
        stream.wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for s in steps:
                sdm.sdm_decode_step(s["kp"], s["qp"], s["v"], s["alpha"], s["beta"], M,
                                    W=wl.W, R=wl.R, S1=wl.S1, gate=s["gate"], y=y, o=o,
                                    stream=side, chained=True)
        secs_g = timed(graph.replay, reps, 1, dist, stream)
        out["graph_us_per_step"] = secs_g / (reps * nsteps) * 1e6
        out["graph_value"] = weak_scaling_value(th, secs_g / (reps * nsteps), dist.world)
        del graph
    except Exception as e:  # reported, not hidden
        out["graph_error"] = repr(e)
    if sdm.sdm_get_device_status() != 0:
        raise RuntimeError("device status word set during the decode benchmark")
    del M, steps
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------- the CPU oracle arm
def cpu_units_sample(wl, tokens: int, g=None):
    """Host arrays of the first `tokens` tokens of sequence 0 (every head) of a workload,
    taken from device tensors when given, else drawn on the host."""
    if g is None:
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        sub = wl.replace(B=1, T=tokens)
        d = sdm_synth.make_inputs(sub, device=dev)
    else:
        d = {k: (t[:1, :tokens] if k != "M0" else t) for k, t in g.items()}
    return {k: v.float().cpu().numpy() for k, v in d.items()}


def oracle_sample_time(wl, tokens: int, threads: int, g=None, h=None):
    """The oracle, as it stands, over the first `tokens` tokens of every head of sequence 0
    (all N rows tracked), one head per thread.  `h` (host arrays of at least `tokens`
    tokens, from cpu_units_sample) saves drawing the sample again.  Returns (token-heads,
    seconds, cores)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    if h is None:
        h = cpu_units_sample(wl, tokens, g)
    else:
        h = {k: (v[:, :tokens] if k != "M0" else v) for k, v in h.items()}
    units = [(0, hh) for hh in range(wl.H)]
    cores = max(1, min(threads, len(units)))

    def one(u):
        b, hh = u
        oracle.run_unit(h["kp"], h["qp"], h["v"], h["alpha"], h["beta"], h["M0"], b, hh,
                        S1=wl.S1, W=wl.W, R=wl.R)
        return u

    t0 = time.perf_counter()
    with ThreadPoolExecutor(cores) as ex:
        list(ex.map(one, units))
    secs = time.perf_counter() - t0
    return tokens * len(units), secs, cores


def run_reference(args, dist: Dist):
    """The reference arm: the CPU oracle on the same workload, metric and unit."""
    if dist.rank != 0:
        return None
    wl = sdm_synth.WORKLOADS[args.workload]
    tokens = args.reference_tokens
    cores = max(1, min(os.cpu_count() or 1, wl.H))
    h = cpu_units_sample(wl, tokens)  # drawn once, outside the timed calls
    for _ in range(args.warmup):
        oracle_sample_time(wl, max(16, tokens // 8), cores, h=h)
    done, secs = 0, 0.0
    for _ in range(args.steps):
        n, s, cores = oracle_sample_time(wl, tokens, cores, h=h)
        done += n
        secs += s
    value = done / secs
    sample = (f"first {tokens} tokens of sequence 0, all {wl.H} heads, every step; "
              f"{wl.note}")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator)",
        "config": {"workload": wl.name, "shape": wl.note},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores,
                         "host_cores": os.cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------------- main
def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["sdm", "reference"], default="sdm")
    ap.add_argument("--workload", default="long_skew")
    ap.add_argument("--decode-workload", default="decode")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the prefill lines of the small and 1.4B-like workloads")
    ap.add_argument("--cpu-tokens", type=int, default=8192,
                    help="tokens per head of the CPU-oracle sample")
    ap.add_argument("--reference-tokens", type=int, default=2048)
    ap.add_argument("--select-schedule", choices=["default", "serial", "pipelined"],
                    default="default",
                    help="the slot engine's selection schedule (SDM_OPT_SELECT_SCHEDULE)")
    ap.add_argument("--only", choices=["prefill", "decode", "balance", "rows", "undo"],
                    default=None,
                    help="run one part (profiling of a small case)")
    ap.add_argument("--override", default="",
                    help="workload fields to change, e.g. B=1,T=4096 (prefill workload)")
    ap.add_argument("--decode-override", default="",
                    help="workload fields to change for the decode workload, e.g. B=8")
    args = ap.parse_args(argv)
    for attr, key in (("override", "workload"), ("decode_override", "decode_workload")):
        kv = getattr(args, attr)
        if kv:
            base = sdm_synth.WORKLOADS[getattr(args, key)]
            fields = {k: int(v) for k, v in (x.split("=") for x in kv.split(","))}
            name = f"{base.name}[{kv}]"
            sdm_synth.WORKLOADS[name] = base.replace(name=name, **fields)
            setattr(args, key, name)
    if args.warmup < 3 and args.impl == "sdm":
        ap.error("--warmup must be at least 3")

    dist = Dist()
    try:
        if args.impl == "reference":
            line = run_reference(args, dist)
            if line is not None:
                print(json.dumps(line), flush=True)
            return 0
        if dist.world != args.gpus:
            if dist.world > 1:
                raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={dist.world}")
        dev = torch.device("cuda", dist.local_rank)
        torch.cuda.set_device(dev)
        import sparse_memory_linear_b200 as sdm
        sdm.library()
        sdm.sdm_set_option("select_schedule",
                           {"default": 0, "serial": 1, "pipelined": 2}[args.select_schedule])

        if args.only == "balance":
            out = bench_balance(args, dev)
            if dist.rank == 0:
                print(json.dumps({"balance": out}), flush=True)
            return 0
        if args.only == "undo":
            out = bench_undo(args, dist, dev)
            if dist.rank == 0:
                print(json.dumps({"undo": out}), flush=True)
            return 0
        if args.only == "rows":
            out = bench_state_rows(args, dist, dev)
            if dist.rank == 0:
                print(json.dumps({"state_rows": out}), flush=True)
            return 0
        if args.only == "decode":
            out = bench_decode(args, dist, dev)
            if dist.rank == 0:
                print(json.dumps({"decode": out}), flush=True)
            return 0
        if args.only == "prefill":
            args.no_decode = True
        pre = bench_prefill(args, dist, dev)
        wl, g = pre.pop("_inputs")
        line = {
            "metric": METRIC, "value": pre["value"], "unit": UNIT, "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": pre["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded counter-based generator; bf16 inputs, fp32 state)",
            "config": {"workload": wl.name, "shape": wl.note, "global_batch": wl.B * dist.world,
                       "seq_len": wl.T, "heads": wl.H, "parallelism": f"replicas x{dist.world}",
                       "l2": "inputs larger than L2 (9 GB of inputs, 4 GB state per step)",
                       "step": "sdm_scan_forward with SDM_CONTINUE: select + scan + norm/gate (M0 init timed apart: state_init_ms)"},
            "roofline": pre["roofline"], "whole_step_hbm": pre["whole_step_hbm"],
            "state_init_ms": pre["state_init_ms"],
            "kernels_ms_per_step": pre["kernels_ms_per_step"],
            "kernel_launches_per_step": pre["kernel_launches_per_step"],
            "kernels_share": pre["kernels_share"],
            "gpu_launches": pre["gpu_launches"], "clocks": pre["clocks"],
        }
        if "e2e" in pre:
            line["e2e"] = pre["e2e"]
        if not args.no_cpu_baseline and dist.world == 1 and dist.rank == 0:
            n, s, cores = oracle_sample_time(wl, args.cpu_tokens, os.cpu_count() or 1, g)
            line["cpu_baseline"] = {
                "value": n / s, "unit": UNIT, "cores": cores, "host_cores": os.cpu_count(),
                "kind": "oracle",
                "sample": f"first {args.cpu_tokens} tokens of sequence 0, all {wl.H} heads "
                          f"({n} token-heads, {s:.1f} s wall, one head per thread: the "
                          f"recurrence of a head is sequential, so {cores} of the "
                          f"{os.cpu_count()} host cores have work)"}
        del g
        torch.cuda.empty_cache()
        if not args.no_configs and args.only is None:
            line["prefill_configs"] = bench_prefill_configs(args, dist, dev)
        if not args.no_decode:
            line["decode"] = bench_decode(args, dist, dev)
        if not args.no_configs and args.only is None:
            line["coupled"] = bench_coupled(args, dist, dev)
            line["state_rows"] = bench_state_rows(args, dist, dev)
            line["undo"] = bench_undo(args, dist, dev)
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
        return 0
    finally:
        dist.close()


if __name__ == "__main__":
    sys.exit(main())
