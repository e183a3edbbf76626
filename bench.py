"""Benchmark of the selective-scan hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one forward scan of the Mamba-2.8B mixer-layer shape (batch 4,
L 4096, D 5120, N 16, bf16 activations, fp32 state; also returns h_last) over
inputs already resident in HBM.  The reported metric is achieved HBM
bandwidth over the compulsory bytes (read x, delta, z, B, C, A, D, bias; write
out and h_last), with Gtoken-channel/s and the fraction of the measured HBM
peak alongside.  The recurrent decode step (256 x 5120 x 16 fp32 state,
one bf16 token per sequence) is measured in the same run under "decode".

Multi-GPU (torchrun): every rank scans its own independent copy of the
workload (weak scaling, no data-path collective); the time is the maximum over
ranks and the value the bytes of all ranks over that time.

`--impl reference` times the float64 CPU oracle instead (the reference arm of
this project), on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import platform
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

FWD_CFG = 2
DECODE_CFG = 4
METRIC = "selective-scan fwd: achieved HBM GB/s (% of peak), Gtoken·ch/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor()


def fwd_bytes(cfg):
    c = workloads.CONFIGS[cfg]
    return workloads.compulsory_bytes_fwd(c.batch, c.seqlen, c.dim, c.dstate,
                                          2 if c.dtype == "bf16" else 4, c.has_h0, True)


def step_bytes(cfg):
    c = workloads.CONFIGS[cfg]
    return workloads.compulsory_bytes_step(c.batch, c.dim, c.dstate, 2 if c.dtype == "bf16" else 4)


def fwd_config(world):
    """The workload both arms report: the forward scan of the Mamba-2.8B layer shape."""
    c = workloads.CONFIGS[FWD_CFG]
    return {"workload": f"{c.name} forward scan (Mamba-2.8B mixer layer shape)",
            "batch": c.batch, "seqlen": c.seqlen, "dim": c.dim, "dstate": c.dstate,
            "state_dtype": "f32", "returns_h_last": True,
            "l2": f"inputs {fwd_bytes(FWD_CFG) / 1e6:.0f} MB > L2 126 MB; no flush needed",
            "parallelism": f"{world} independent replica(s)"}


def _source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_38_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def _profiled(kernel_key):
    """The committed ncu summary of a kernel (profiles/traffic.json): DRAM bytes
    per launch and pipe utilisation, if the kernel sources have not changed
    since it was taken (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel_key]
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("source_hash") != _source_hash():
        return None
    return rec


def _pipes(kernel_key):
    rec = _profiled(kernel_key)
    if rec is None:
        return None
    keys = ("fma_pipe_pct", "xu_pipe_pct", "tensor_pipe_pct", "dram_throughput_pct", "issue_active_pct",
            "smem_pipe_pct", "smem_bank_conflicts_ld", "smem_bank_conflicts_st")
    out = {k: rec[k] for k in keys if k in rec}
    out["source"] = "ncu, profiles/traffic.json"
    return out


# ---------------------------------------------------------------------------
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index, period_s=0.005):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: report no clocks
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _max_over_ranks(value, world, device):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_oracle_rate(cfg, target_s=10.0, threads=None):
    """Time the float64 oracle (as it stands) on a bounded channel sample of
    `cfg`; returns (GB/s-equivalent, seconds, channels, threads)."""
    import oracle
    orc = oracle.load()
    c = workloads.CONFIGS[cfg]
    threads = threads or _cores()
    inp = workloads.make_inputs(cfg)
    rng = np.random.default_rng(123)
    nsel = 64
    spent = 0.0
    done = 0
    while True:
        chan = rng.choice(c.channels, nsel, replace=False)
        t0 = time.perf_counter()
        orc.fwd_channels(inp["x"], inp["delta"], inp["delta_bias"], True, inp["A"], inp["B"],
                         inp["C"], inp["D"], inp["z"], inp["h0"], chan, threads=threads)
        dt = time.perf_counter() - t0
        spent += dt
        done += nsel
        if spent >= target_s or done >= c.channels:
            break
        # grow the sample towards the time budget
        nsel = int(min(c.channels - done, max(nsel, nsel * max(1.0, (target_s - spent) / max(dt, 1e-3)))))
        nsel = max(nsel, 1)
    bytes_per_chan = fwd_bytes(cfg) / c.channels
    return bytes_per_chan * done / spent / 1e9, spent, done, threads


def run_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return 0
    import oracle
    orc = oracle.load()
    c = workloads.CONFIGS[FWD_CFG]
    inp = workloads.make_inputs(FWD_CFG)
    threads = _cores()
    rng = np.random.default_rng(7)
    nsel = max(1, min(c.channels, int(os.environ.get("SSM_REF_CHANNELS", "256"))))
    bytes_per_chan = fwd_bytes(FWD_CFG) / c.channels

    def one():
        chan = rng.choice(c.channels, nsel, replace=False)
        t0 = time.perf_counter()
        orc.fwd_channels(inp["x"], inp["delta"], inp["delta_bias"], True, inp["A"], inp["B"],
                         inp["C"], inp["D"], inp["z"], inp["h0"], chan, threads=threads)
        return time.perf_counter() - t0

    for _ in range(args.warmup):
        one()
    times = [one() for _ in range(args.steps)]
    total = sum(times)
    value = bytes_per_chan * nsel * args.steps / total / 1e9
    sample = (f"{nsel} random channels (full L={c.seqlen}) of the {c.name} forward scan per step; "
              f"GB/s counts the compulsory bytes of those channels")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": fwd_config(1),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample, "cpu": _cpu_model()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
def _to_dev(a, device):
    import torch
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def _to_pinned(a):
    import torch
    if a is None:
        return None
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    return t.pin_memory()


def bench_fwd(args, device, world, cfg=FWD_CFG, steps=None, warmup=None):
    """Event-timed forward scans of `cfg` over inputs resident in HBM (all
    configs' inputs exceed the 126 MB L2, so no flush is needed).  One launch =
    the forward call (its S4D and general kernel instances, and for few-group
    shapes the summary pass, the combine and the second pass)."""
    import torch
    import selective_state_space_38_b200 as ssm
    steps = args.steps if steps is None else steps
    warmup = args.warmup if warmup is None else warmup
    c = workloads.CONFIGS[cfg]
    inp = workloads.make_inputs(cfg)
    t = {k: _to_dev(v, device) for k, v in inp.items() if isinstance(v, np.ndarray)}
    out = torch.empty_like(t["x"])
    hl = torch.empty((c.batch, c.dim, c.dstate), dtype=torch.float32, device=device)
    ws = torch.empty(ssm.ssm_scan_fwd_workspace_size(c.batch, c.seqlen, c.dim, device), dtype=torch.uint8,
                     device=device)
    stream = torch.cuda.current_stream(device)

    def launch():
        ssm.ssm_scan_fwd(t["x"], t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"], t["D"],
                         t["z"], t.get("h0"), out=out, h_last=hl, workspace=ws)

    for _ in range(warmup):
        launch()
    torch.cuda.synchronize(device)
    if ssm.ssm_scan_fwd_status(ws, stream) != 0:
        raise RuntimeError("a bounded device wait gave up during the warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    _barrier(world)
    torch.cuda.synchronize(device)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clk:
        start.record(stream)
        for i in range(steps):
            ev[i][0].record(stream)
            launch()
            ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize(device)
    _barrier(world)
    total_ms = start.elapsed_time(end)
    per_launch = [a.elapsed_time(b) for a, b in ev]
    total_ms = _max_over_ranks(total_ms, world, device)
    segs_schedule = ssm.ssm_scan_fwd_workspace_size(c.batch, c.seqlen, c.dim, device) > \
        ssm.ssm_scan_fwd_workspace_size(c.batch, 1, c.dim, device)
    return dict(total_ms=total_ms, launch_ms=statistics.mean(per_launch),
                launch_ms_median=statistics.median(per_launch), clocks=clk.summary(), inputs=inp,
                kernels_per_call=5 if segs_schedule else 2)


def bench_e2e(args, device, world, inp):
    """Same metric through the public API from pinned host buffers: H2D copy of
    the step's inputs, the scan, D2H copy of out and h_last, every step."""
    import torch
    import selective_state_space_38_b200 as ssm
    c = workloads.CONFIGS[FWD_CFG]
    host = {k: _to_pinned(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    dev = {k: torch.empty(v.shape, dtype=v.dtype, device=device) for k, v in host.items()}
    out_h = torch.empty((c.batch, c.dim, c.seqlen), dtype=torch.bfloat16).pin_memory()
    hl_h = torch.empty((c.batch, c.dim, c.dstate), dtype=torch.float32).pin_memory()
    out_d = torch.empty(out_h.shape, dtype=out_h.dtype, device=device)
    hl_d = torch.empty(hl_h.shape, dtype=hl_h.dtype, device=device)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_h.numel() * out_h.element_size() + hl_h.numel() * hl_h.element_size()
    stream = torch.cuda.current_stream(device)

    ws = torch.empty(ssm.ssm_scan_fwd_workspace_size(c.batch, c.seqlen, c.dim, device), dtype=torch.uint8,
                     device=device)

    def one():
        for k, v in host.items():
            dev[k].copy_(v, non_blocking=True)
        ssm.ssm_scan_fwd(dev["x"], dev["delta"], dev["delta_bias"], True, dev["A"], dev["B"],
                         dev["C"], dev["D"], dev["z"], None, out=out_d, h_last=hl_d, workspace=ws)
        out_h.copy_(out_d, non_blocking=True)
        hl_h.copy_(hl_d, non_blocking=True)

    steps = max(1, min(args.steps, 20))
    for _ in range(max(1, min(args.warmup, 3))):
        one()
    torch.cuda.synchronize(device)
    _barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        one()
    b.record(stream)
    torch.cuda.synchronize(device)
    _barrier(world)
    ms = _max_over_ranks(a.elapsed_time(b), world, device) / steps
    return dict(ms=ms, h2d=h2d, d2h=d2h, steps=steps)


def _next_rows_inputs(device):
    """The Mamba-2.8B layer workload on the device, plus the extra inputs of
    the widened rows: width-4 convolution taps, lambda ~ U(0, 1), dout ~ N(0, 1)."""
    import torch
    c = workloads.CONFIGS[FWD_CFG]
    inp = workloads.make_inputs(FWD_CFG)
    t = {k: _to_dev(v, device) for k, v in inp.items() if isinstance(v, np.ndarray)}
    g = torch.Generator(device=device)
    g.manual_seed(22)
    t["conv_w"] = torch.randn((c.dim, 4), generator=g, device=device) * 0.5
    t["conv_bias"] = torch.randn(c.dim, generator=g, device=device) * 0.2
    t["lam"] = torch.rand(t["x"].shape, generator=g, device=device).to(torch.bfloat16)
    t["dout"] = torch.randn(t["x"].shape, generator=g, device=device).to(torch.bfloat16)
    return c, t


def bench_next_rows(args, device, hbm_peak, only=None):
    """Event-timed sub-lines of the widened rows on the Mamba-2.8B layer shape:
    the convolution fused in front of the scan, the exponential-trapezoidal
    scan, and the backward pass.  Bytes are each call's compulsory traffic."""
    import torch
    import selective_state_space_38_b200 as ssm
    c, t = _next_rows_inputs(device)
    tok = c.batch * c.seqlen * c.dim
    bc = 2 * c.batch * c.dstate * c.seqlen
    base = fwd_bytes(FWD_CFG)
    out = torch.empty_like(t["x"])
    hl = torch.empty((c.batch, c.dim, c.dstate), dtype=torch.float32, device=device)
    ws = torch.empty(ssm.ssm_scan_fwd_workspace_size(c.batch, c.seqlen, c.dim, device), dtype=torch.uint8,
                     device=device)
    cs_out = torch.empty((c.batch, c.dim, 3), dtype=torch.bfloat16, device=device)
    dims = ssm.Dims(c.batch, c.seqlen, c.dim, c.dstate, ssm.SSM_BF16)
    nbw = ctypes.c_size_t(0)
    ssm.get_lib().ssm_scan_bwd_workspace_size(ctypes.byref(dims), ctypes.byref(nbw))
    wsb = torch.empty(int(nbw.value), dtype=torch.uint8, device=device)
    rows = {
        "conv_scan_fwd": (lambda: ssm.ssm_conv_scan_fwd(
            t["x"], t["conv_w"], t["conv_bias"], None, t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"],
            t["D"], t["z"], None, out=out, h_last=hl, conv_state_out=cs_out, workspace=ws),
            base + c.dim * 5 * 4 + c.batch * c.dim * 3 * 2, "causal conv (width 4) + silu fused in front of the scan"),
        "trap_scan_fwd": (lambda: ssm.ssm_trap_scan_fwd(
            t["x"], t["delta"], t["delta_bias"], True, t["lam"], t["A"], t["B"], t["C"], t["D"], t["z"], None,
            out=out, h_last=hl, workspace=ws),
            base + tok * 2, "exponential-trapezoidal scan (lambda per token and channel)"),
        "scan_bwd": (lambda: ssm.ssm_scan_bwd(
            t["x"], t["delta"], t["delta_bias"], True, t["A"], t["B"], t["C"], t["D"], t["z"], None, t["dout"],
            None, workspace=wsb),
            tok * 2 * 7 + bc * 2 + bc * 4 + c.dim * c.dstate * 8 + c.dim * 16 + c.batch * c.dim * c.dstate * 4,
            "backward pass: read x, delta, z, dout, B, C; write dx, ddelta, dz, dB, dC, dA, dD, dbias, dh0"),
    }
    # Mamba-2 SSD on a 2.7B-like layer: 4 x 4096, 80 heads of 64, one group of B and C, state 128
    sb, sl, sh, sp_, sg, sn = 4, 4096, 80, 64, 1, 128
    g = torch.Generator(device=device)
    g.manual_seed(23)
    sx = torch.randn((sb, sl, sh, sp_), generator=g, device=device).to(torch.bfloat16)
    sdt = (torch.randn((sb, sl, sh), generator=g, device=device) * 0.1).to(torch.bfloat16)
    sB = torch.randn((sb, sl, sg, sn), generator=g, device=device).to(torch.bfloat16)
    sC = torch.randn((sb, sl, sg, sn), generator=g, device=device).to(torch.bfloat16)
    sA = -(torch.rand(sh, generator=g, device=device) * 15 + 1)
    sbias = torch.full((sh,), -4.0, device=device)
    sD = torch.ones(sh, device=device)
    sy = torch.empty_like(sx)
    shl = torch.empty((sb, sh, sp_, sn), dtype=torch.float32, device=device)
    sws = torch.empty(ssm.ssm_ssd_fwd_workspace_size(sb, sh, device), dtype=torch.uint8, device=device)
    rows["ssd_fwd"] = (lambda: ssm.ssm_ssd_fwd(sx, sdt, sbias, True, sA, sB, sC, sD, None, y=sy, h_last=shl,
                                                workspace=sws),
                       2 * sx.numel() * 2 + sdt.numel() * 2 + 2 * sB.numel() * 2 + sh * 12 + shl.numel() * 4,
                       "Mamba-2 SSD (tensor cores), 2.7B-like layer 4 x 4096, 80 heads x 64, state 128")
    res = {}
    for name, (fn, nbytes, what) in rows.items():
        if only and name != only:
            continue
        try:
            for _ in range(3):
                fn()
            torch.cuda.synchronize(device)
        except ssm.SSMError as exc:  # a refused call is reported in its row, not fatal to the line
            res[name] = {"workload": what, "error": str(exc)}
            continue
        n = 20 if name != "scan_bwd" else 10
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, b in ev:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize(device)
        ms = statistics.mean([a.elapsed_time(b) for a, b in ev])
        gbs = nbytes / (ms * 1e-3) / 1e9
        key = {"ssd_fwd": "ssd_fwd_layer", "scan_bwd": "scan_bwd_cfg2"}.get(name, f"{name}_cfg2")
        res[name] = {"workload": what if name == "ssd_fwd" else f"{c.name}: {what}", "ms": round(ms, 5),
                     "value": round(gbs, 2), "unit": "GB/s",
                     "frac": round(gbs / hbm_peak, 4), "algorithmic_bytes_per_launch": nbytes, "steps": n,
                     "traffic": (_profiled(key) or {}).get("dram_bytes_per_launch"), "pipes": _pipes(key)}
    return res


def _device_tokens(c, n, gen, device):
    """n decode token sets drawn on the device with the decode config's
    distributions (x, z, B, C ~ N(0,1), delta ~ N(0, 0.1^2)), rounded to bf16."""
    import torch

    def draw(shape, scale=1.0):
        return (torch.randn(shape, generator=gen, device=device) * scale).to(torch.bfloat16)
    return dict(x=draw((n, c.batch, c.dim)), delta=draw((n, c.batch, c.dim), 0.1),
                z=draw((n, c.batch, c.dim)), B=draw((n, c.batch, c.dstate)), C=draw((n, c.batch, c.dstate)))


def bench_decode(args, device, flushed_steps=64):
    """The recurrent step on the decode config (256 sequences x 5120 channels x
    16 fp32 states): 1024 consecutive steps, back to back, from the state a
    64-step prefill leaves; the per-step mean is the headline.  Beside it, the
    median of single steps with the L2 flushed before each one (so the 84 MB
    state comes from HBM)."""
    import torch
    import selective_state_space_38_b200 as ssm
    c = workloads.CONFIGS[DECODE_CFG]
    prm = workloads.decode_params(DECODE_CFG)
    p = {k: _to_dev(prm[k], device) for k in ("A", "D", "delta_bias")}
    gen = torch.Generator(device=device)
    gen.manual_seed(4)
    pre = _device_tokens(c, c.prefill_steps, gen, device)
    tok = _device_tokens(c, c.decode_steps, gen, device)
    state = torch.zeros((c.batch, c.dim, c.dstate), dtype=torch.float32, device=device)
    outb = torch.empty((c.batch, c.dim), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def step(src, i):
        ssm.ssm_scan_step(state, src["x"][i], src["delta"][i], p["delta_bias"], True, p["A"], src["B"][i],
                          src["C"][i], p["D"], src["z"][i], out=outb)

    for i in range(c.prefill_steps):
        step(pre, i)
    prefill_state = state.clone()
    for i in range(8):  # warm-up
        step(tok, i)
    state.copy_(prefill_state)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(c.decode_steps):
        step(tok, i)
    b.record(stream)
    torch.cuda.synchronize(device)
    ms_b2b = a.elapsed_time(b) / c.decode_steps

    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    times = []
    for s in range(flushed_steps + 4):
        flush.fill_(float(s))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step(tok, s)
        e1.record(stream)
        times.append((e0, e1))
    torch.cuda.synchronize(device)
    ms_flushed = statistics.median([x.elapsed_time(y) for x, y in times[4:]])
    nb = step_bytes(DECODE_CFG)
    return dict(ms=ms_b2b, gbs=nb / (ms_b2b * 1e-3) / 1e9, bytes=nb, steps=c.decode_steps,
                gtok_ch=c.batch * c.dim / (ms_b2b * 1e-3) / 1e9,
                ms_flushed=ms_flushed, gbs_flushed=nb / (ms_flushed * 1e-3) / 1e9,
                launches=c.prefill_steps + 8 + c.decode_steps + flushed_steps + 4)


def run_gpu(args):
    import torch
    world, rank, local = _dist()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    hbm_peak, peak_kind = _peaks()
    c = workloads.CONFIGS[FWD_CFG]

    if args.only and world > 1:
        raise SystemExit("--only is a single-GPU profiling mode")
    if args.only == "step":
        dec = bench_decode(args, device)
        print(json.dumps({"only": "step", "ms_per_step": round(dec["ms"], 5), "value": round(dec["gbs"], 2),
                          "unit": "GB/s", "ms_per_step_flushed": round(dec["ms_flushed"], 5)}), flush=True)
        return 0
    if args.only in ("conv_scan_fwd", "trap_scan_fwd", "scan_bwd", "ssd_fwd"):
        r = bench_next_rows(args, device, hbm_peak, only=args.only)
        print(json.dumps({"only": args.only, **r[args.only]}), flush=True)
        return 0
    if args.only == "fwd":
        f = bench_fwd(args, device, world, cfg=args.config)
        nb = fwd_bytes(args.config)
        print(json.dumps({"only": "fwd", "config": args.config, "launch_ms_mean": round(f["launch_ms"], 5),
                          "value": round(nb / (f["launch_ms"] * 1e-3) / 1e9, 2), "unit": "GB/s"}),
              flush=True)
        return 0
    f = bench_fwd(args, device, world)
    nb = fwd_bytes(FWD_CFG)
    ms_step = f["total_ms"] / args.steps
    value = world * nb / (ms_step * 1e-3) / 1e9
    achieved = nb / (f["launch_ms"] * 1e-3) / 1e9
    e = bench_e2e(args, device, world, f["inputs"])
    del f["inputs"]
    e2e_gbs = world * nb / (e["ms"] * 1e-3) / 1e9
    dec = bench_decode(args, device) if rank == 0 else None
    launches = f["kernels_per_call"] * args.steps

    subs = {}
    if rank == 0:
        # the other forward configs, one sub-line each (same timing, fewer steps)
        for cfg, steps in ((1, 50), (3, 10)):
            cs = workloads.CONFIGS[cfg]
            g = bench_fwd(args, device, 1, cfg=cfg, steps=steps, warmup=3)
            del g["inputs"]
            nbs = fwd_bytes(cfg)
            gbs = nbs / (g["launch_ms"] * 1e-3) / 1e9
            subs[cs.name] = {"launch_ms_mean": round(g["launch_ms"], 5), "value": round(gbs, 2), "unit": "GB/s",
                             "frac": round(gbs / hbm_peak, 4),
                             "gtok_ch_per_s": round(cs.batch * cs.seqlen * cs.dim / (g["launch_ms"] * 1e-3) / 1e9, 2),
                             "algorithmic_bytes_per_launch": nbs, "steps": steps,
                             "kernels_per_call": g["kernels_per_call"], "clocks": g["clocks"],
                             "pipes": _pipes(f"scan_fwd_cfg{cfg}")}
            launches += g["kernels_per_call"] * (steps + 3)
        launches += dec["launches"]
        nxt = bench_next_rows(args, device, hbm_peak)

    if rank == 0:
        cpu_val, cpu_s, cpu_ch, cores = cpu_oracle_rate(FWD_CFG, target_s=float(
            os.environ.get("SSM_CPU_BASELINE_S", "10")))
        # the oracle on one thread, on the Mamba-130M layer shape (a bounded channel sample)
        one_val, one_s, one_ch, _ = cpu_oracle_rate(1, target_s=float(os.environ.get("SSM_CPU_ONE_S", "3")),
                                                    threads=1)
        tok_ch = c.batch * c.seqlen * c.dim
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": fwd_config(world),
            "pct_of_hbm_peak": round(100.0 * value / world / hbm_peak, 2),
            "pct_of_hbm_spec_8tbs": round(100.0 * value / world / 8000.0, 2),
            "gtok_ch_per_s": round(world * tok_ch / (ms_step * 1e-3) / 1e9, 2),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": hbm_peak,
                         "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                         "peak_kind": peak_kind,
                         "traffic": (_profiled("scan_fwd_cfg2") or {}).get("dram_bytes_per_launch"),
                         "algorithmic_bytes_per_launch": nb,
                         "launch_ms_mean": round(f["launch_ms"], 5),
                         "launch_ms_median": round(f["launch_ms_median"], 5)},
            "pipes": _pipes("scan_fwd_cfg2"),
            "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": e["h2d"],
                    "d2h_bytes_per_step": e["d2h"], "ms_per_step": round(e["ms"], 3),
                    "steps": e["steps"]},
            "cpu_baseline": {"value": round(cpu_val, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "cpu": _cpu_model(),
                             "sample": f"{cpu_ch} channels (full L) of the same workload, "
                                       f"{cpu_s:.1f} s of float64 oracle time",
                             "single_thread": {"value": round(one_val, 4), "unit": "GB/s", "cores": 1,
                                               "workload": workloads.CONFIGS[1].name,
                                               "sample": f"{one_ch} channels (full L), {one_s:.1f} s"}},
            "other_configs": subs,
            "next_rows": nxt,
            "decode": {"workload": workloads.CONFIGS[DECODE_CFG].name,
                       "ms_per_step": round(dec["ms"], 5), "value": round(dec["gbs"], 2),
                       "unit": "GB/s", "pct_of_hbm_peak": round(100 * dec["gbs"] / hbm_peak, 2),
                       "gtok_ch_per_s": round(dec["gtok_ch"], 3), "steps": dec["steps"],
                       "bytes_per_step": dec["bytes"],
                       "l2": "back to back from the 64-step prefill state (the 84 MB state partly stays in L2)",
                       "flushed": {"ms_per_step": round(dec["ms_flushed"], 5),
                                   "value": round(dec["gbs_flushed"], 2),
                                   "pct_of_hbm_peak": round(100 * dec["gbs_flushed"] / hbm_peak, 2),
                                   "l2": "flushed before each step"},
                       "pipes": _pipes("scan_step_cfg4")},
            # kernels of this library launched inside the timed region: per forward call its
            # S4D and general instances (five kernels on the two-pass schedule)
            "gpu_launches": f["kernels_per_call"] * args.steps,
            # and over the whole run (warm-up, end-to-end leg, other configs, decode)
            "gpu_launches_run": launches,
            "clocks": f["clocks"],
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    # profiler runs: only the forward-scan or only the decode-step timing loop
    ap.add_argument("--only", default=None, choices=["fwd", "step", "conv_scan_fwd", "trap_scan_fwd", "scan_bwd",
                                                        "ssd_fwd"])
    ap.add_argument("--config", type=int, default=FWD_CFG, choices=[0, 1, 2, 3],
                    help="forward config of --only fwd")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
