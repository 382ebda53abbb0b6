"""Workload driver on one GPU: builds the initial states, optionally calibrates
the DAMP rows, and runs windowed decode steps through the C ABI.

Every numerical step runs in liblq.so kernels: the prefill that produces the
initial state uses the chunked prefill (lq_prefill; or, on request, the
FP32-state decode kernel token by token), the initial quantization uses
lq_state_init, the DAMP choice uses lq_damp_select.  torch provides device
memory, the seeded input draws (inputs.py), streams and CUDA graphs.
"""
from __future__ import annotations

import torch

from . import inputs as gen
from . import lq
from .configs import Workload


def gpu_prefill(wl: Workload, *, tokens: int | None = None, batch: int | None = None, stream: str = "prefill",
                chunk: int = 64, device="cuda", capture_heads=None, keep_inputs: bool = False,
                method: str = "chunked"):
    """FP32 recurrence from zero over `tokens` generator tokens on the GPU:
    `method` "chunked" runs lq_prefill on each generator chunk, "recurrent"
    the FP32-state decode kernel one token at a time.

    Returns the state [batch, H, dk, dv] (float32, no outliers yet) and, if
    capture_heads lists (b, h) pairs, those heads' inputs on the host in the
    generator's [T, B', Hk|H, ...] layout restricted to the listed batch rows.
    """
    T = wl.prefill if tokens is None else tokens
    B = wl.B if batch is None else batch
    cfg = lq.Config(B=B, H=wl.H, Hk=wl.Hk, dk=wl.dk, dv=wl.dv, gate=wl.gate, mode="fp32", r=0, n_hp_rows=0)
    S0 = torch.zeros((B, wl.H, wl.dk, wl.dv), device=device)
    st = lq.lq_state_init(cfg, S0) if method != "chunked" else None
    o = torch.empty((B, wl.H, wl.dv), device=device)
    captured = []
    bsel = None
    if capture_heads:
        bsel = torch.tensor(sorted({b for b, _ in capture_heads}), device=device)
    S = torch.zeros_like(S0)
    for c in range((T + chunk - 1) // chunk):
        n = min(chunk, T - c * chunk)
        tok = gen.token_inputs(wl, n, stream=stream, chunk=c, batch=B, device=device)
        if method == "chunked":
            lq.lq_prefill(cfg, tok["q"], tok["k"], tok["v"], tok["beta"], tok["alpha"], S0=S, S_out=S)
        else:
            for t in range(n):
                lq.lq_decode_step(st, tok["q"][t], tok["k"][t], tok["v"][t], tok["beta"][t], tok["alpha"][t], o)
        if bsel is not None:
            captured.append({k: v.index_select(1, bsel).cpu() for k, v in tok.items()})
    if st is not None:
        lq.lq_state_export_fp32(st, S)
        rc = lq.lq_get_status(st)
        if rc != lq.LQ_OK:
            raise lq.LqError(rc, "prefill")
        lq.lq_state_destroy(st)
    elif not bool(torch.isfinite(S).all()):
        raise lq.LqError(lq.LQ_ERR_NONFINITE, "prefill")
    if bsel is None:
        return S, None
    cap = {k: torch.cat([c[k] for c in captured], dim=0) for k in captured[0]}
    return S, cap


def initial_state(wl: Workload, **kw):
    S, cap = gpu_prefill(wl, **kw)
    return gen.apply_outliers(S, wl), cap


def damp_rows(wl: Workload, device="cuda") -> torch.Tensor:
    """Offline DAMP calibration on the GPU: calibration prefills (lq_prefill),
    the workload's outliers, then lq_damp_select.  Returns rows [H, P] (host)."""
    n, T = wl.calib_prefills, wl.calib_tokens
    states, _ = gpu_prefill(wl, tokens=T, batch=n, stream="calib", device=device)
    states = gen.apply_outliers(states, wl)
    gates = []
    for c in range((T + 63) // 64):
        tok = gen.token_inputs(wl, min(64, T - c * 64), stream="calib", chunk=c, batch=n, device=device)
        gates.append(tok["alpha"].reshape(-1, wl.H, wl.dk if wl.gate == "kda" else 1))
    gates = torch.cat(gates).contiguous()
    cfg = lq.Config(B=1, H=wl.H, Hk=wl.H, dk=wl.dk, dv=wl.dv, gate=wl.gate, r=wl.r,
                    power_iters=wl.K, n_hp_rows=wl.P, smoothing=wl.smoothing)
    energy = torch.zeros((wl.H, wl.dk), dtype=torch.float64, device=device)
    rows = torch.zeros((wl.H, wl.P), dtype=torch.int32, device=device)
    lq.lq_damp_select(cfg, states.contiguous(), gates, energy, rows)
    return rows.cpu()


def static_scales(wl: Workload, n: int = 8, tokens: int | None = None, device="cuda"):
    """Offline fit of fixed key-row / value-column scales (smoothing 2) on the
    GPU: n calibration prefills of the workload's prefill length (calibration
    draws, the workload's outliers), rows weighted by their decay persistence
    (lq_fit_static_scales forms it from the calibration decays: per key channel
    for KDA, one value per head for GDN).  Returns (m [H, dk], s [H, dv]) on
    the device."""
    T = wl.prefill if tokens is None else tokens
    states, _ = gpu_prefill(wl, tokens=T, batch=n, stream="calib", device=device)
    states = gen.apply_outliers(states, wl).contiguous()
    tok = gen.token_inputs(wl, min(T, 256), stream="calib", batch=n, device=device)
    gates = tok["alpha"].reshape(-1, wl.H, wl.dk if wl.gate == "kda" else 1).contiguous()
    cfg = lq.Config(B=1, H=wl.H, Hk=wl.H, dk=wl.dk, dv=wl.dv, gate=wl.gate, r=wl.r, power_iters=wl.K,
                    state_bits=wl.bits, smoothing=2)
    return lq.lq_fit_static_scales(cfg, states, gates=gates)


class WindowRunner:
    """Holds a decode state, the decode inputs of T tokens and one CUDA graph
    per window of W tokens (the W-th call also flushes)."""

    def __init__(self, wl: Workload, S0: torch.Tensor, *, mode: str = "window", hp_rows=None,
                 tokens: int | None = None, device="cuda", static=None, phases=None):
        self.wl = wl
        self.cfg = lq.Config.from_workload(wl, mode=mode)
        self.W = wl.W          # tokens per graph; in step mode every call also requantizes
        self.T = wl.T if tokens is None else tokens
        self.hp_rows = hp_rows
        if static is not None:   # fixed scales (smoothing 2): (m [H, dk], s [H, dv])
            self.st = lq.lq_state_init(self.cfg, S0.contiguous(), static_m=static[0], static_s=static[1])
        else:
            self.st = lq.lq_state_init(self.cfg, S0.contiguous(), hp_rows=hp_rows)
        # staggered windows: batch entry b ends its windows at the steps where
        # (step + phases[b]) mod W = W - 1 (lq_state_set_phases)
        self.phases = phases
        if phases is not None:
            lq.lq_state_set_phases(self.st, phases)
        self.tok = gen.token_inputs(wl, self.T, device=device)
        self.out = torch.empty((self.T, wl.B, wl.H, wl.dv), device=device)
        self.graphs = {}

    @property
    def n_windows(self) -> int:
        return self.T // self.W

    def step_call(self, t: int):
        tk = self.tok
        lq.lq_decode_step(self.st, tk["q"][t], tk["k"][t], tk["v"][t], tk["beta"][t], tk["alpha"][t], self.out[t])

    def run_window_eager(self, w: int):
        for t in range(w * self.W, (w + 1) * self.W):
            self.step_call(t)

    def capture(self):
        """One graph per window slot; replays must start at a window boundary.
        The warm-up runs window 0 eagerly: with phases it holds every entry's
        shorter first window, and the graphs then hold full windows only."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run_window_eager(0)          # warm the launch path before capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        for w in range(self.n_windows):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.run_window_eager(w)
            self.graphs[w] = g
        torch.cuda.synchronize()

    def replay(self, w: int):
        self.graphs[w % self.n_windows].replay()
