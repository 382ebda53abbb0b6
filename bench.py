"""Benchmark of windowed INT8 delta-rule decode on B200.

`python bench.py --gpus N --steps K --warmup W [--workload NAME] [--impl ours|reference]`

One step = one window of the workload on every head of the batch: W decode
calls through the C ABI (the W-th also reconstructs, re-extracts the
compensators, smooths and requantizes the state), replayed from a CUDA graph.
Prints ONE JSON line (rank 0).  Default workload: GDN, 1024 independent
states x 16 heads, d = 128, W = 64, r = 4 (state + buffers ~1.3 GB, larger
than L2, so no L2 flush is needed between steps).

--impl reference times the CPU oracle (the plain C implementation the parity
tests compare against) on a bounded sample of heads of the same workload.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_recurrent_state_lq_b200 import configs, inputs as gen, lq, runner, traffic  # noqa: E402

METRIC = "state updates/s (batch·head·token) and achieved HBM TB/s vs ~8 TB/s B200 peak"
UNIT = "state updates/s"
DEFAULT_WL = configs.GDN_PREFIX_CACHE.name


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# ---------------------------------------------------------------- clocks

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and throttle reasons of this process's GPU through NVML."""

    def __init__(self, device: int, period: float = 0.05):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(device)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
        except Exception:  # NVML unavailable: report no clocks
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in _REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- distributed

from quantized_recurrent_state_lq_b200 import dist as D  # noqa: E402

dist_setup = D.setup
max_over_ranks = D.max_over_ranks
barrier = D.barrier


# ---------------------------------------------------------------- CPU oracle leg

def oracle_sample_seconds(wl, heads: int, threads: int, seed_offset: int = 0):
    """Time the oracle on `heads` heads of the workload for one window (W tokens
    and the flush).  Initial states: a short oracle prefill plus the workload's
    outliers (the decode's CPU work does not depend on the values)."""
    import numpy as np
    from oracle import oracle as O
    sw = wl.with_(B=max(1, heads // wl.H + (heads % wl.H > 0)), seed=wl.seed + seed_offset)
    oc = O.Cfg(dk=wl.dk, dv=wl.dv, gate=wl.gate, W=wl.W, r=wl.r, K=wl.K, smoothing=wl.smoothing, P=wl.P,
               bf16_buffer=wl.buffer_bf16, bits=wl.bits)
    pre = gen.token_inputs(sw, 16, stream="prefill")
    S0 = O.prefill(O.Cfg(dk=wl.dk, dv=wl.dv, gate=wl.gate, quantize=0), O.per_head_inputs(pre, wl.H),
                   nthreads=threads).astype(np.float32).reshape(sw.B, wl.H, wl.dk, wl.dv)
    S0 = gen.apply_outliers(torch.from_numpy(S0), sw).numpy().reshape(-1, wl.dk, wl.dv)[:heads]
    tok = O.per_head_inputs(gen.token_inputs(sw, wl.W), wl.H)
    tok = {k: np.ascontiguousarray(v[:, :heads]) for k, v in tok.items()}
    rows = None
    if wl.P:
        rows = np.tile(np.arange(wl.P, dtype=np.int32) * (wl.dk // wl.P), (heads, 1))
    t0 = time.perf_counter()
    O.run(oc, tok, S0=S0, hp_rows=rows, flush_last=True, nthreads=threads)
    dt = time.perf_counter() - t0
    return dt


def cpu_baseline(wl, target_s: float = 12.0, target_1t_s: float = 6.0):
    """The oracle on all host cores (OpenMP across heads), and beside it on one
    thread, each on a bounded sample of the workload's heads."""
    threads = os.cpu_count() or 1
    probe = 32
    dt = oracle_sample_seconds(wl, probe, threads)
    heads = int(max(probe, min(100000, probe * target_s / max(dt, 1e-3))))
    dt = oracle_sample_seconds(wl, heads, threads, seed_offset=1)
    value = heads * wl.W / dt
    probe1 = 4
    d1 = oracle_sample_seconds(wl, probe1, 1)
    heads1 = int(max(probe1, min(4096, probe1 * target_1t_s / max(d1, 1e-3))))
    d1 = oracle_sample_seconds(wl, heads1, 1, seed_offset=2)
    return {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{heads} heads of {wl.name} x one window ({wl.W} tokens + flush), "
                      f"includes the oracle's initial quantization; {dt:.1f} s",
            "single_thread": {"value": heads1 * wl.W / d1, "unit": UNIT, "cores": 1, "kind": "oracle",
                              "sample": f"{heads1} heads x one window on one thread; {d1:.1f} s"}}


def run_reference(args, wl, world, rank, pg):
    if rank != 0:
        return 0
    threads = os.cpu_count() or 1
    probe = 16
    dt = oracle_sample_seconds(wl, probe, threads)
    heads = int(max(probe, min(100000, probe * 2.5 / max(dt, 1e-3))))   # ~2.5 s per step
    for _ in range(args.warmup):
        oracle_sample_seconds(wl, heads, threads)
    times = [oracle_sample_seconds(wl, heads, threads, seed_offset=1 + k) for k in range(args.steps)]
    t = sum(times)
    value = heads * wl.W * args.steps / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": wl.name, "sample_heads": heads},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"{heads} heads x one window of {wl.W} tokens per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU leg

def _code_only(text: str) -> str:
    """C / C++ source without comments, trailing blanks and empty lines (the
    sources carry no comment markers inside string literals)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_sources_sha(names) -> str:
    """sha256 prefix of the listed csrc files' code (in the order given,
    comments left out): the sources the profiled kernel is built from."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_recurrent_state_lq_b200", "csrc")
    try:
        for f in names:
            h.update(_code_only(open(os.path.join(csrc, f)).read()).encode())
    except OSError:
        return "missing"
    return h.hexdigest()[:16] if names else "none"


def profile_traffic(wl):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current sources of that kernel (the files
    listed under `sources:`); else None."""
    path = os.path.join(ROOT, "profiles", "decode_window_traffic.txt")
    try:
        kv = dict(line.split(":", 1) for line in open(path) if ":" in line)
    except OSError:
        return None
    if kv.get("sources_sha256", "").strip() != kernel_sources_sha(kv.get("sources", "").split()):
        return None
    if kv.get("workload", "").strip() != wl.name:
        return None
    if wl.bits != 8 or wl.buffer_bf16:   # the capture is of the INT8 state with the FP32 buffer
        return None
    try:
        return float(kv["dram_bytes_per_launch_full"])
    except (KeyError, ValueError):
        return None


def time_graph_steps(r: runner.WindowRunner, K: int, start: int, stream) -> float:
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for k in range(K):
        r.replay(start + k)
    ev1.record(stream)
    ev1.synchronize()
    return ev0.elapsed_time(ev1) / 1e3


def kernel_times(r: runner.WindowRunner, windows: int, stream):
    """Mean device time of the buffering decode launches and of the flushing
    launch, each bracketed by CUDA events on the launching stream."""
    W = r.W
    evs = []
    for w in range(windows):
        for t in range(W):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            r.step_call(w * W + t)
            b.record(stream)
            evs.append((t, a, b))
    torch.cuda.synchronize()
    buf = [a.elapsed_time(b) / 1e3 for t, a, b in evs if t < W - 1]
    fl = [a.elapsed_time(b) / 1e3 for t, a, b in evs if t == W - 1]
    return (statistics.mean(buf) if buf else None), statistics.mean(fl)


def e2e_measure(r: runner.WindowRunner, steps: int, stream):
    """Whole windows through the C ABI with HOST inputs and outputs: every
    window's inputs are copied from pinned host memory to the device and its
    outputs back, all inside the timed region.  The copies are pipelined with
    the decode: window k+1's inputs go up on a copy stream into the other of
    two input slots while window k runs, and window k's outputs come down on a
    third stream while window k+1 runs (events order every reuse of a slot)."""
    W = r.W
    keys = ["q", "k", "v", "beta", "alpha"]
    host_in = {k: torch.empty_like(r.tok[k][:W], device="cpu").pin_memory() for k in keys}
    for k in keys:
        host_in[k].copy_(r.tok[k][:W])
    host_out = [torch.empty_like(r.out[:W], device="cpu").pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, used, out_ready, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]
    slot_tok = lambda sl: {k: r.tok[k][sl * W:(sl + 1) * W] for k in keys}

    def upload(sl):
        with torch.cuda.stream(up):
            dst = slot_tok(sl)
            for key in keys:
                dst[key].copy_(host_in[key], non_blocking=True)
            in_ready[sl].record(up)

    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    up.wait_event(ev0)
    upload(0)
    for k in range(steps):
        sl = k % 2
        if k + 1 < steps:
            if k >= 1:
                up.wait_event(used[1 - sl])     # window k-1 is done reading that slot
            upload(1 - sl)
        stream.wait_event(in_ready[sl])
        if k >= 2:
            stream.wait_event(out_free[sl])     # window k-2's outputs are down
        r.replay(sl)
        used[sl].record(stream)
        out_ready[sl].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(out_ready[sl])
            host_out[sl].copy_(r.out[sl * W:(sl + 1) * W], non_blocking=True)
            out_free[sl].record(down)
    stream.wait_stream(down)
    stream.wait_stream(up)
    ev1.record(stream)
    ev1.synchronize()
    dt = ev0.elapsed_time(ev1) / 1e3
    return dt, h2d, d2h


def mode_throughput(wl, S0, mode: str, windows: int, stream):
    """Throughput of a reference mode on the same inputs (FP32 state or
    per-step INT8), timed over whole graph-replayed windows."""
    r = runner.WindowRunner(wl, S0, mode=mode, tokens=wl.W * min(2, wl.T // wl.W))
    r.capture()
    for k in range(2):
        r.replay(k)
    torch.cuda.synchronize()
    dt = time_graph_steps(r, windows, 0, stream)
    v = wl.heads * wl.W * windows / dt
    del r
    torch.cuda.empty_cache()
    return v


def variant(wv, S0, stream, peak_gbs: float, note: str, windows: int = 3, static=None, hp_rows=None) -> dict:
    """Another configuration of the window step on the same inputs: whole-window
    throughput by graph replay, and the buffering launch's achieved
    algorithmic bandwidth."""
    r = runner.WindowRunner(wv, S0, tokens=wv.W * min(2, wv.T // wv.W), static=static, hp_rows=hp_rows)
    r.capture()
    for k in range(2):
        r.replay(k)
    torch.cuda.synchronize()
    dt = time_graph_steps(r, windows, 0, stream)
    t_buf, t_flush = kernel_times(r, 1, stream)
    rc = lq.lq_get_status(r.st)
    if rc != lq.LQ_OK:
        raise lq.LqError(rc, f"variant status ({note})")
    launch_bytes = traffic.nonflush_launch_bytes(wv) * wv.heads
    del r
    torch.cuda.empty_cache()
    step_bytes = traffic.window_bytes(wv) * wv.heads
    return {"value": wv.heads * wv.W * windows / dt, "unit": UNIT, "ms_per_step": 1e3 * dt / windows,
            "decode_buffering_mean_s": t_buf, "decode_flushing_mean_s": t_flush,
            "buffering_roofline_frac": launch_bytes / t_buf / 1e9 / peak_gbs,
            "algorithmic_bytes_per_step": step_bytes,
            "hbm": {"achieved_tbs": step_bytes * windows / dt / 1e12, "frac_of_8tbs": step_bytes * windows / dt / 8e12,
                    "frac_of_measured": step_bytes * windows / dt / 1e9 / peak_gbs},
            "state_bits_per_value": traffic.bits_per_value(wv), "note": note}


def workload_line(wl, stream, peak_gbs: float, windows: int = 6) -> dict:
    """Another benchmark workload at its full size (its own initial state from
    the GPU prefill, BF16 rows from the DAMP calibration where it has them):
    the same whole-window measurement, with the clocks sampled over it."""
    rows = runner.damp_rows(wl) if wl.P else None
    S0, _ = runner.initial_state(wl)
    dev = torch.cuda.current_device()
    with ClockSampler(dev) as clk:
        out = variant(wl, S0, stream, peak_gbs, f"workload {wl.name}", windows=windows, hp_rows=rows)
    out["clocks"] = clk.summary()
    out["config"] = {"workload": wl.name, "gate": wl.gate, "B": wl.B, "H": wl.H, "Hk": wl.Hk, "dk": wl.dk,
                     "dv": wl.dv, "W": wl.W, "r": wl.r, "P": wl.P}
    del S0
    torch.cuda.empty_cache()
    return out


# FP32 arithmetic peak of the B200 used for ALU-bound kernels: 148 SMs x 128
# FP32 lanes x 2 flops per FMA x the 1965 MHz maximum SM clock.
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def prefill_line(wl, stream, chunks: int = 8, tokens: int = 256) -> dict:
    """The chunked prefill (lq_prefill) of the workload's heads over its
    prefill length: `chunks` calls of `tokens` tokens each from one seeded
    draw of `tokens` tokens (the kernel's work does not depend on the values),
    the state carried in place; beside it the token-by-token FP32-state kernel
    on 64 tokens.  CUDA events on the launching stream."""
    cfg = lq.Config(B=wl.B, H=wl.H, Hk=wl.Hk, dk=wl.dk, dv=wl.dv, gate=wl.gate, mode="fp32", r=0)
    tok = gen.token_inputs(wl, tokens, stream="prefill", device="cuda")
    S = torch.zeros((wl.B, wl.H, wl.dk, wl.dv), device="cuda")
    run = lambda: lq.lq_prefill(cfg, tok["q"], tok["k"], tok["v"], tok["beta"], tok["alpha"], S0=S, S_out=S)
    for _ in range(2):
        run()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(chunks):
        run()
    ev1.record(stream)
    ev1.synchronize()
    dt = ev0.elapsed_time(ev1) / 1e3
    T = chunks * tokens
    if not bool(torch.isfinite(S).all()):
        raise lq.LqError(lq.LQ_ERR_NONFINITE, "prefill")
    # the recurrent FP32-state kernel on `tokens` tokens
    st = lq.lq_state_init(cfg, S)
    o = torch.empty((wl.B, wl.H, wl.dv), device="cuda")
    step = lambda t: lq.lq_decode_step(st, tok["q"][t], tok["k"][t], tok["v"][t], tok["beta"][t],
                                       tok["alpha"][t], o)
    for t in range(4):
        step(t)
    torch.cuda.synchronize()
    nrec = min(tokens, 64)
    ev0.record(stream)
    for t in range(nrec):
        step(t)
    ev1.record(stream)
    ev1.synchronize()
    dtr = ev0.elapsed_time(ev1) / 1e3 * (T / nrec)
    lq.lq_state_destroy(st)
    flops = traffic.prefill_flops(wl, T) * wl.heads
    achieved = flops / dt / 1e12
    peaks, src = measured_peaks()
    # FP32-accurate products as three TF32 passes: the TF32 peak (the measured
    # bf16 peak x the nominal 1.1 / 2.25 ratio) / 3
    peak = peaks["bf16_tflops"] * 1.1 / 2.25 / 3
    del tok, S
    torch.cuda.empty_cache()
    return {"tokens": T, "heads": wl.heads, "chunk": traffic.PREFILL_CHUNK, "seconds": dt,
            "value": wl.heads * T / dt, "unit": "state updates/s",
            "recurrent_fp32_seconds": dtr, "speedup_vs_recurrent": dtr / dt,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None,
                         "kernel": ("prefill_umma_kernel (chunked WY form; the state in tensor memory, "
                                    "products as tcgen05.mma TF32 x3, inputs by TMA tensor copies)"
                                    if wl.dk == 128 and wl.dv == 128 else
                                    "prefill_tc_kernel (chunked WY form; products as mma.sync TF32 x3)"),
                         "peak_source": f"{src} bf16 burst x 1.1/2.25 (TF32) / 3 passes",
                         "fp32_alu_frac": achieved / FP32_PEAK_TFLOPS},
            "note": f"{chunks} calls of one {tokens}-token draw; recurrent time from {nrec} tokens x {T // nrec}"}


def state_dtype(wl) -> str:
    return "int8" if wl.bits == 8 else f"int{wl.bits} (bit-packed)"


def run_ours(args, wl, world, rank, pg):
    dev = torch.cuda.current_device()
    stream = torch.cuda.current_stream()
    peaks, peak_src = measured_peaks()
    rows = runner.damp_rows(wl) if wl.P else None
    S0, _ = runner.initial_state(wl)
    r = runner.WindowRunner(wl, S0, hp_rows=rows)
    r.capture()
    for k in range(args.warmup):
        r.replay(k)
    torch.cuda.synchronize()
    barrier(pg)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        dt = time_graph_steps(r, args.steps, args.warmup, stream)
    torch.cuda.synchronize()
    barrier(pg)
    dt_max = max_over_ranks(dt, pg)
    rc = lq.lq_get_status(r.st)
    if rc != lq.LQ_OK:
        raise lq.LqError(rc, "decode status")

    value = D.weak_scaling_value(wl.heads * wl.W * args.steps, world, dt_max)
    step_bytes = traffic.window_bytes(wl) * wl.heads
    t_buf, t_flush = kernel_times(r, 2, stream)
    launch_bytes = traffic.nonflush_launch_bytes(wl) * wl.heads
    achieved = launch_bytes / t_buf / 1e9
    tr = profile_traffic(wl)
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": tr,
            "kernel": "decode_kernel (buffering launches, n = 0..W-2)",
            "algorithmic_bytes_per_launch": launch_bytes, "mean_launch_s": t_buf,
            "peak_source": f"{peak_src} hbm_gbs (copy kernel)"}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "state_dtype": state_dtype(wl), "data": "synthetic",
            "config": {"workload": wl.name, "gate": wl.gate, "prefill": wl.prefill, "B": wl.B, "H": wl.H, "Hk": wl.Hk, "dk": wl.dk,
                       "dv": wl.dv, "W": wl.W, "r": wl.r, "K": wl.K, "P": wl.P, "step": "one window per head",
                       "l2": "state + buffers + inputs larger than L2 (no flush needed)",
                       "parallelism": f"dp{world} (independent heads, no collective)"},
            "hbm": {"achieved_tbs": step_bytes * args.steps / dt / 1e12,
                    "frac_of_8tbs": step_bytes * args.steps / dt / 8e12,
                    "frac_of_measured": step_bytes * args.steps / dt / 1e9 / peaks["hbm_gbs"],
                    "algorithmic_bytes_per_step": step_bytes},
            "kernels": {"decode_buffering_mean_s": t_buf, "decode_flushing_mean_s": t_flush},
            "roofline": roof, "gpu_launches": wl.W * args.steps, "clocks": clk.summary(),
            "state_bits_per_value": traffic.bits_per_value(wl)}

    e2e_steps = max(1, min(args.steps, 5))
    dte, h2d, d2h = e2e_measure(r, e2e_steps, stream)
    dte = max_over_ranks(dte, pg)
    line["e2e"] = {"value": wl.heads * wl.W * e2e_steps * world / dte, "unit": UNIT,
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del r
    torch.cuda.empty_cache()

    if not args.no_modes and wl.P == 0 and not wl.buffer_bf16 and wl.bits == 8:
        modes = {"window_int8": value / world}
        modes["fp32_state"] = mode_throughput(wl, S0, "fp32", 4, stream)
        modes["per_step_int8"] = mode_throughput(wl, S0, "step", 2, stream)
        nv = wl.with_(r=0, smoothing=0)
        modes["naive_per_step_int8"] = mode_throughput(nv, S0, "step", 2, stream)
        modes["window_vs_fp32_speedup"] = modes["window_int8"] / modes["fp32_state"]
        line["modes_per_gpu"] = modes
        line["buffer_bf16_per_gpu"] = variant(wl.with_(buffer_bf16=1), S0, stream, peaks["hbm_gbs"],
                                              "option: buffered token updates stored as bf16(k/Gamma), bf16(u)")
        line["low_bit_states_per_gpu"] = {
            f"int{b}": variant(wl.with_(bits=b), S0, stream, peaks["hbm_gbs"],
                               f"{b}-bit window-start state (codes in +-{(1 << (b - 1)) - 1}, bit-packed)")
            for b in (6, 4)}
        line["static_scales_per_gpu"] = {
            f"int{b}": variant(wl.with_(smoothing=2, bits=b), S0, stream, peaks["hbm_gbs"],
                               f"{b}-bit state, fixed key-row / value-column scales fitted offline on 8 "
                               "calibration prefills (not timed)",
                               static=runner.static_scales(wl.with_(bits=b)))
            for b in (8, 4)}

    if not args.no_modes:
        line["prefill_per_gpu"] = prefill_line(wl, stream)
        # the other two large workloads of the benchmark set, whole windows
        for other in (configs.KDA_B256, configs.GDN_DAMP):
            if other.name != wl.name:
                line[other.name.split("_h")[0] + "_per_gpu"] = workload_line(other, stream, peaks["hbm_gbs"])

    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WL, choices=sorted(configs.BY_NAME))
    ap.add_argument("--no-modes", action="store_true", help="skip the FP32 / per-step INT8 context lines")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling runs)")
    ap.add_argument("--prefill", type=int, default=None, help="override the prefill length (profiling runs)")
    ap.add_argument("--buffer-bf16", action="store_true",
                    help="run the traffic-lean option (buffered token updates in BF16) as the main line")
    ap.add_argument("--bits", type=int, choices=[8, 6, 4], default=8,
                    help="code width of the quantized state for the main line (6, 4: bit-packed)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the chunked prefill of the workload's heads (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    wl = configs.BY_NAME[args.workload]
    if args.batch is not None:
        wl = wl.with_(B=args.batch)
    if args.prefill is not None:
        wl = wl.with_(prefill=args.prefill)
    if args.buffer_bf16:
        wl = wl.with_(buffer_bf16=1)
    if args.bits != 8:
        wl = wl.with_(bits=args.bits)
    world, rank, local, pg = dist_setup()
    try:
        if args.impl == "reference":
            rc = run_reference(args, wl, world, rank, pg)
        elif args.prefill_only:
            line = {"workload": wl.name, "B": wl.B, "H": wl.H,
                    "prefill_per_gpu": prefill_line(wl, torch.cuda.current_stream())}
            if rank == 0:
                print(json.dumps(line), flush=True)
            rc = 0
        else:
            rc = run_ours(args, wl, world, rank, pg)
    finally:
        D.teardown(pg)
    return rc


if __name__ == "__main__":
    sys.exit(main())
