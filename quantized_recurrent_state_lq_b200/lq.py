"""Thin Python binding of liblq.so (include/lq_state.h), same names as the C ABI.

Argument marshalling only: torch tensors are checked for device, dtype, shape
and contiguity and passed as raw device pointers together with torch's current
CUDA stream.  Every computation happens in the CUDA library; if liblq.so is
missing this module raises on import of the library instead of falling back.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblq.so")

LQ_OK = 0
LQ_ERR_INVALID_ARG = -1
LQ_ERR_SHAPE = -2
LQ_ERR_WORKSPACE = -3
LQ_ERR_WINDOW_FULL = -4
LQ_ERR_CUDA = -5
LQ_ERR_NONFINITE = -6
LQ_ERR_UNSUPPORTED = -7
LQ_ERR_TIMEOUT = -8

LQ_GATE_SCALAR, LQ_GATE_CHANNEL = 0, 1
LQ_MODE_FP32, LQ_MODE_INT8_STEP, LQ_MODE_INT8_WINDOW = 0, 1, 2

EXPORTED = ["lq_workspace_bytes", "lq_config_check", "lq_state_init", "lq_decode_step",
            "lq_window_flush", "lq_state_buffered", "lq_state_export_fp32",
            "lq_state_export_view", "lq_state_import_view", "lq_quantize_state",
            "lq_dequantize_state", "lq_quantize_state_static", "lq_damp_select", "lq_get_status",
            "lq_state_destroy", "lq_strerror", "lq_selftest_division", "lq_prefill",
            "lq_state_init_static", "lq_fit_static_scales", "lq_selftest_wait", "lq_state_set_phases"]


class LqError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


class lq_config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("B", "H", "Hk", "dk", "dv", "gate", "mode", "W", "r",
                                          "power_iters", "n_hp_rows", "smoothing", "fused_flush",
                                          "buffer_bf16", "state_bits")]


class lq_qstate_view(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("bf16_rows", C.c_void_p), ("m", C.c_void_p),
                ("s", C.c_void_p), ("comp_k", C.c_void_p), ("comp_v", C.c_void_p)]


_lib = None


def lib():
    """Load liblq.so (building it in-tree first if it is missing or stale)."""
    global _lib
    if _lib is None:
        from . import build as _build
        if not os.path.exists(LIB_PATH) or _build._stale():
            _build.build()
        L = C.CDLL(LIB_PATH)
        vp, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
        cfgp = C.POINTER(lq_config)
        viewp = C.POINTER(lq_qstate_view)
        sig = {
            "lq_workspace_bytes": (sz, [cfgp]),
            "lq_config_check": (C.c_int, [cfgp]),
            "lq_state_init": (C.c_int, [C.POINTER(vp), cfgp, vp, sz, vp, vp, vp]),
            "lq_decode_step": (C.c_int, [vp, vp, vp, vp, vp, vp, vp, vp]),
            "lq_window_flush": (C.c_int, [vp, vp]),
            "lq_state_buffered": (C.c_int, [vp]),
            "lq_state_export_fp32": (C.c_int, [vp, vp, vp]),
            "lq_state_export_view": (C.c_int, [vp, viewp, vp]),
            "lq_state_import_view": (C.c_int, [vp, viewp, vp]),
            "lq_quantize_state": (C.c_int, [cfgp, vp, vp, viewp, vp]),
            "lq_dequantize_state": (C.c_int, [cfgp, viewp, vp, vp, vp]),
            "lq_quantize_state_static": (C.c_int, [cfgp, vp, vp, viewp, vp]),
            "lq_damp_select": (C.c_int, [cfgp, i32, vp, i32, vp, vp, vp, vp]),
            "lq_get_status": (C.c_int, [vp, vp]),
            "lq_state_destroy": (None, [vp]),
            "lq_strerror": (C.c_char_p, [C.c_int]),
            "lq_selftest_division": (C.c_int, [vp, vp, vp, vp, vp, i32, vp]),
            "lq_prefill": (C.c_int, [cfgp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
            "lq_state_init_static": (C.c_int, [C.POINTER(vp), cfgp, vp, sz, vp, vp, vp, vp]),
            "lq_fit_static_scales": (C.c_int, [cfgp, i32, vp, i32, vp, vp, vp, vp]),
            "lq_selftest_wait": (C.c_int, [vp, C.c_int64, vp]),
            "lq_state_set_phases": (C.c_int, [vp, vp, vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().lq_strerror(code).decode()


def _chk(rc: int, what: str):
    if rc != LQ_OK:
        raise LqError(rc, what)


@dataclass
class Config:
    B: int
    H: int
    Hk: int
    dk: int
    dv: int
    gate: str = "gdn"            # "gdn" | "kda"
    mode: str = "window"         # "fp32" | "step" | "window"
    W: int = 32
    r: int = 4
    power_iters: int = 8
    n_hp_rows: int = 0
    smoothing: int = 1
    fused_flush: int = 1
    buffer_bf16: int = 0         # 1: buffered token updates kept in BF16 (window mode)
    state_bits: int = 8          # code width of the quantized state: 8, 6 or 4 (bit-packed)

    def c(self) -> lq_config:
        gate = {"gdn": LQ_GATE_SCALAR, "kda": LQ_GATE_CHANNEL}[self.gate]
        mode = {"fp32": LQ_MODE_FP32, "step": LQ_MODE_INT8_STEP, "window": LQ_MODE_INT8_WINDOW}[self.mode]
        return lq_config(self.B, self.H, self.Hk, self.dk, self.dv, gate, mode, self.W, self.r,
                         self.power_iters, self.n_hp_rows, self.smoothing, self.fused_flush,
                         self.buffer_bf16, self.state_bits)

    @property
    def heads(self) -> int:
        return self.B * self.H

    @property
    def ga(self) -> int:
        return self.dk if self.gate == "kda" else 1

    @staticmethod
    def from_workload(wl, mode: str = "window", **kw) -> "Config":
        base = dict(B=wl.B, H=wl.H, Hk=wl.Hk, dk=wl.dk, dv=wl.dv, gate=wl.gate, mode=mode,
                    W=(1 if mode == "step" else wl.W), r=wl.r, power_iters=wl.K,
                    n_hp_rows=(wl.P if mode != "fp32" else 0), smoothing=wl.smoothing,
                    buffer_bf16=(wl.buffer_bf16 if mode == "window" else 0),
                    state_bits=(wl.bits if mode != "fp32" else 8))
        base.update(kw)
        return Config(**base)


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dev(t: torch.Tensor, name: str, shape=None, dtype=torch.float32) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _host_rows(cfg: Config, hp_rows):
    if cfg.n_hp_rows == 0:
        return None, None
    arr = torch.as_tensor(hp_rows, dtype=torch.int32).cpu().contiguous()
    if tuple(arr.shape) != (cfg.H, cfg.n_hp_rows):
        raise ValueError(f"hp_rows must be [H, P] = {(cfg.H, cfg.n_hp_rows)}")
    return arr, C.c_void_p(arr.data_ptr())


def view_shapes(cfg: Config) -> dict:
    B, H, dk, dv, P, r = cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.n_hp_rows, cfg.r
    return {"codes": ((B, H, dk - P, dv), torch.int8), "bf16_rows": ((B, H, P, dv), torch.int16),
            "m": ((B, H, dk), torch.float32), "s": ((B, H, dv), torch.float32),
            "comp_k": ((B, H, r, dk), torch.float32), "comp_v": ((B, H, r, dv), torch.float32)}


def alloc_view(cfg: Config, device="cuda") -> dict:
    return {k: torch.zeros(shape, dtype=dt, device=device) for k, (shape, dt) in view_shapes(cfg).items()}


def _view_struct(cfg: Config, view: dict) -> lq_qstate_view:
    ptr = {}
    for k, (shape, dt) in view_shapes(cfg).items():
        t = view[k]
        ptr[k] = _dev(t, k, shape, dt) if t.numel() else None
    return lq_qstate_view(ptr["codes"], ptr["bf16_rows"], ptr["m"], ptr["s"], ptr["comp_k"], ptr["comp_v"])


def lq_config_check(cfg: Config) -> int:
    return lib().lq_config_check(C.byref(cfg.c()))


def lq_workspace_bytes(cfg: Config) -> int:
    return lib().lq_workspace_bytes(C.byref(cfg.c()))


class LqState:
    """Owns the opaque handle and keeps the workspace tensor alive."""

    def __init__(self, cfg: Config, handle: int, workspace: torch.Tensor, rows):
        self.cfg = cfg
        self.handle = C.c_void_p(handle)
        self.workspace = workspace
        self._rows = rows

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value and _lib is not None:
            _lib.lq_state_destroy(h)
            self.handle = C.c_void_p(0)


def lq_state_init(cfg: Config, S0: torch.Tensor, hp_rows=None, workspace: torch.Tensor | None = None,
                  stream=None, static_m: torch.Tensor | None = None,
                  static_s: torch.Tensor | None = None) -> LqState:
    """lq_state_init, or lq_state_init_static when the scales are given
    (cfg.smoothing = 2: static_m [H, dk], static_s [H, dv])."""
    nbytes = lq_workspace_bytes(cfg)
    if nbytes == 0:
        _chk(lq_config_check(cfg), "lq_config_check")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=S0.device)
    p_s0 = _dev(S0, "S0", (cfg.B, cfg.H, cfg.dk, cfg.dv))
    h = C.c_void_p()
    ws = (C.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size())
    if static_m is not None or static_s is not None:
        pm = _dev(static_m, "static_m", (cfg.H, cfg.dk))
        ps = _dev(static_s, "static_s", (cfg.H, cfg.dv))
        _chk(lib().lq_state_init_static(C.byref(h), C.byref(cfg.c()), *ws, C.c_void_p(p_s0), C.c_void_p(pm),
                                        C.c_void_p(ps), C.c_void_p(_stream(stream))), "lq_state_init_static")
        return LqState(cfg, h.value, workspace, None)
    rows, p_rows = _host_rows(cfg, hp_rows)
    _chk(lib().lq_state_init(C.byref(h), C.byref(cfg.c()), *ws, C.c_void_p(p_s0), p_rows,
                             C.c_void_p(_stream(stream))), "lq_state_init")
    return LqState(cfg, h.value, workspace, rows)


def lq_fit_static_scales(cfg: Config, states: torch.Tensor, gates: torch.Tensor | None = None,
                         stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Static scales (smoothing 2) of every head from calibration states
    [n, H, dk, dv]; gates [n_samples, H, 1 | dk] (the calibration decays that
    weight the rows by their persistence) or None (unweighted).  Returns
    (m [H, dk], s [H, dv])."""
    n = states.shape[0]
    p_st = _dev(states, "states", (n, cfg.H, cfg.dk, cfg.dv))
    ng, p_g = 0, None
    if gates is not None:
        ng = gates.shape[0]
        p_g = _dev(gates, "gates", (ng, cfg.H, cfg.dk if cfg.gate == "kda" else 1))
    m = torch.empty((cfg.H, cfg.dk), device=states.device)
    s = torch.empty((cfg.H, cfg.dv), device=states.device)
    _chk(lib().lq_fit_static_scales(C.byref(cfg.c()), C.c_int32(n), C.c_void_p(p_st), C.c_int32(ng),
                                    C.c_void_p(p_g), C.c_void_p(m.data_ptr()), C.c_void_p(s.data_ptr()),
                                    C.c_void_p(_stream(stream))), "lq_fit_static_scales")
    return m, s


def lq_decode_step(st: LqState, q, k, v, beta, alpha, o, stream=None):
    c = st.cfg
    args = [_dev(q, "q", (c.B, c.Hk, c.dk)), _dev(k, "k", (c.B, c.Hk, c.dk)),
            _dev(v, "v", (c.B, c.H, c.dv)), _dev(beta, "beta", (c.B, c.H)),
            _dev(alpha, "alpha", (c.B, c.H) if c.gate == "gdn" else (c.B, c.H, c.dk)),
            _dev(o, "o", (c.B, c.H, c.dv))]
    _chk(lib().lq_decode_step(st.handle, *[C.c_void_p(a) for a in args], C.c_void_p(_stream(stream))),
         "lq_decode_step")


def lq_state_set_phases(st: LqState, phases, stream=None):
    """Staggered windows: phases [B] (ints in [0, W)), or None to remove them."""
    if phases is None:
        _chk(lib().lq_state_set_phases(st.handle, None, C.c_void_p(_stream(stream))), "lq_state_set_phases")
        return
    vals = [int(x) for x in phases]
    if len(vals) != st.cfg.B:
        raise ValueError(f"phases: {len(vals)} values for B = {st.cfg.B}")
    arr = (C.c_int32 * len(vals))(*vals)
    _chk(lib().lq_state_set_phases(st.handle, C.cast(arr, C.c_void_p), C.c_void_p(_stream(stream))),
         "lq_state_set_phases")


def lq_window_flush(st: LqState, stream=None):
    _chk(lib().lq_window_flush(st.handle, C.c_void_p(_stream(stream))), "lq_window_flush")


def lq_state_buffered(st: LqState) -> int:
    return lib().lq_state_buffered(st.handle)


def lq_state_export_fp32(st: LqState, S: torch.Tensor, stream=None):
    c = st.cfg
    _chk(lib().lq_state_export_fp32(st.handle, C.c_void_p(_dev(S, "S", (c.B, c.H, c.dk, c.dv))),
                                    C.c_void_p(_stream(stream))), "lq_state_export_fp32")


def lq_state_export_view(st: LqState, view: dict, stream=None):
    v = _view_struct(st.cfg, view)
    _chk(lib().lq_state_export_view(st.handle, C.byref(v), C.c_void_p(_stream(stream))), "lq_state_export_view")


def lq_state_import_view(st: LqState, view: dict, stream=None):
    v = _view_struct(st.cfg, view)
    _chk(lib().lq_state_import_view(st.handle, C.byref(v), C.c_void_p(_stream(stream))), "lq_state_import_view")


def lq_quantize_state(cfg: Config, S: torch.Tensor, view: dict, hp_rows=None, stream=None):
    p = _dev(S, "S", (cfg.B, cfg.H, cfg.dk, cfg.dv))
    rows, p_rows = _host_rows(cfg, hp_rows)
    v = _view_struct(cfg, view)
    _chk(lib().lq_quantize_state(C.byref(cfg.c()), C.c_void_p(p), p_rows, C.byref(v),
                                 C.c_void_p(_stream(stream))), "lq_quantize_state")


LQ_STATIC_ROWS_MAX = 8192
LQ_MAX_WINDOW = 4096


def lq_quantize_state_static(cfg: Config, S: torch.Tensor, view: dict, hp_rows=None, stream=None):
    """lq_quantize_state for callers that must not let the library allocate
    device memory: the BF16 row list goes to a fixed array inside liblq.so
    (at most LQ_STATIC_ROWS_MAX = H * n_hp_rows entries) instead of a per-call
    temporary.  Calls that overlap on the GPU share that array and race."""
    p = _dev(S, "S", (cfg.B, cfg.H, cfg.dk, cfg.dv))
    rows, p_rows = _host_rows(cfg, hp_rows)
    v = _view_struct(cfg, view)
    _chk(lib().lq_quantize_state_static(C.byref(cfg.c()), C.c_void_p(p), p_rows, C.byref(v),
                                        C.c_void_p(_stream(stream))), "lq_quantize_state_static")


LQ_PREFILL_CHUNK = 16


def lq_prefill(cfg: Config, q, k, v, beta, alpha, S0=None, S_out=None, o=None, stream=None) -> torch.Tensor:
    """Chunked prefill of T tokens (inputs [T, ...] stacks of decode-step
    inputs) from S0 (None: zero state) into S_out (allocated when None; may be
    S0); o [T,B,H,dv] receives the outputs when given.  Returns S_out."""
    T = q.shape[0]
    B, H, Hk, dk, dv = cfg.B, cfg.H, cfg.Hk, cfg.dk, cfg.dv
    shapes = {"q": (T, B, Hk, dk), "k": (T, B, Hk, dk), "v": (T, B, H, dv), "beta": (T, B, H),
              "alpha": (T, B, H, dk) if cfg.gate == "kda" else (T, B, H)}
    ptr = {n: _dev(t, n, shapes[n]) for n, t in (("q", q), ("k", k), ("v", v), ("beta", beta), ("alpha", alpha))}
    if S_out is None:
        S_out = torch.empty((B, H, dk, dv), device=q.device)
    p_out = _dev(S_out, "S_out", (B, H, dk, dv))
    p_s0 = _dev(S0, "S0", (B, H, dk, dv)) if S0 is not None else None
    p_o = _dev(o, "o", (T, B, H, dv)) if o is not None else None
    _chk(lib().lq_prefill(C.byref(cfg.c()), C.c_int32(T), C.c_void_p(ptr["q"]), C.c_void_p(ptr["k"]),
                          C.c_void_p(ptr["v"]), C.c_void_p(ptr["beta"]), C.c_void_p(ptr["alpha"]),
                          C.c_void_p(p_s0), C.c_void_p(p_out), C.c_void_p(p_o), C.c_void_p(_stream(stream))),
         "lq_prefill")
    return S_out


def lq_selftest_division(a: torch.Tensor, b: torch.Tensor, stream=None):
    """Run the codec's division routine and IEEE division on the same device
    operands (float32, same even length; pairs b[2j] == b[2j+1] for the
    two-lane variant).  Returns (fast, pair, ieee)."""
    n = a.numel()
    pa = _dev(a, "a", (n,))
    pb = _dev(b, "b", (n,))
    fast, pair, ieee = (torch.empty_like(a) for _ in range(3))
    _chk(lib().lq_selftest_division(C.c_void_p(pa), C.c_void_p(pb), C.c_void_p(fast.data_ptr()),
                                    C.c_void_p(pair.data_ptr()), C.c_void_p(ieee.data_ptr()), n,
                                    C.c_void_p(_stream(stream))), "lq_selftest_division")
    return fast, pair, ieee


def lq_dequantize_state(cfg: Config, view: dict, S: torch.Tensor, hp_rows=None, stream=None):
    p = _dev(S, "S", (cfg.B, cfg.H, cfg.dk, cfg.dv))
    rows, p_rows = _host_rows(cfg, hp_rows)
    v = _view_struct(cfg, view)
    _chk(lib().lq_dequantize_state(C.byref(cfg.c()), C.byref(v), p_rows, C.c_void_p(p),
                                   C.c_void_p(_stream(stream))), "lq_dequantize_state")


def lq_damp_select(cfg: Config, states: torch.Tensor, gates: torch.Tensor, energy: torch.Tensor,
                   rows: torch.Tensor, stream=None):
    n = states.shape[0]
    ps = _dev(states, "states", (n, cfg.H, cfg.dk, cfg.dv))
    ng = gates.shape[0]
    pg = _dev(gates, "gates", (ng, cfg.H, cfg.ga))
    pe = _dev(energy, "energy", (cfg.H, cfg.dk), torch.float64)
    pr = _dev(rows, "rows", (cfg.H, cfg.n_hp_rows), torch.int32)
    _chk(lib().lq_damp_select(C.byref(cfg.c()), n, C.c_void_p(ps), ng, C.c_void_p(pg), C.c_void_p(pe),
                              C.c_void_p(pr), C.c_void_p(_stream(stream))), "lq_damp_select")


def lq_selftest_wait(st: LqState, limit_ns: int = 1_000_000, stream=None):
    """Make one bounded device wait run out on purpose (failure-detection self-test)."""
    _chk(lib().lq_selftest_wait(st.handle, C.c_int64(limit_ns), C.c_void_p(_stream(stream))),
         "lq_selftest_wait")


def lq_get_status(st: LqState, stream=None) -> int:
    return lib().lq_get_status(st.handle, C.c_void_p(_stream(stream)))


def lq_state_destroy(st: LqState):
    if st.handle.value:
        lib().lq_state_destroy(st.handle)
        st.handle = C.c_void_p(0)
