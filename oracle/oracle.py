"""Python face of the CPU oracle (test infrastructure only).

Only the test suite, the package's smoke check and the benchmark's CPU-baseline
leg may import this module.  It compiles `lq_oracle.c` with gcc (double
arithmetic, -ffp-contract=off, OpenMP across heads) and marshals numpy arrays
into it.  Nothing here is used by, or uses, the CUDA library.

Every function follows the C file's definitions; see the header of
`lq_oracle.c` for the sources on the pages and for the readings taken where
they are silent.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lq_oracle.c")
_LIB = os.path.join(_HERE, "liblq_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle if the shared object is missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Cfg(C.Structure):
    _fields_ = [(n, C.c_int) for n in
                ("dk", "dv", "gate", "W", "r", "K", "smoothing", "P", "quantize", "bf16_buffer",
                 "bits")] + [("static_m", C.c_void_p), ("static_s", C.c_void_p)]


class _Views(C.Structure):
    _fields_ = [("codes", C.POINTER(C.c_int8)), ("m", C.POINTER(C.c_float)),
                ("s", C.POINTER(C.c_float)), ("c", C.POINTER(C.c_float)),
                ("w", C.POINTER(C.c_float)), ("hp", C.POINTER(C.c_uint16))]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.lqo_bf16_rne.restype = C.c_uint16
        _lib.lqo_bf16_rne.argtypes = [C.c_float]
        _lib.lqo_bf16_to_float.restype = C.c_float
        _lib.lqo_bf16_to_float.argtypes = [C.c_uint16]
    return _lib


@dataclass
class Cfg:
    """Per-head method parameters (the oracle's own copy of the config)."""
    dk: int
    dv: int
    gate: str = "gdn"      # "gdn" | "kda"
    W: int = 16
    r: int = 2
    K: int = 8
    smoothing: int = 1
    P: int = 0
    quantize: int = 1
    bf16_buffer: int = 0   # 1: buffered updates kept in BF16 (lqo_step_bf16)
    bits: int = 8          # code width of the quantized state: 8, 6 or 4
    static_m: object = None   # smoothing 2: fitted key-row scales [dk] ([nh, dk] for run)
    static_s: object = None   # and value-column scales [dv] ([nh, dv] for run)

    def c(self) -> _Cfg:
        sm = ss = None
        if self.smoothing == 2 and self.static_m is not None:
            self._sm = _f32(self.static_m)
            self._ss = _f32(self.static_s)
            sm, ss = self._sm.ctypes.data, self._ss.ctypes.data
        return _Cfg(self.dk, self.dv, 1 if self.gate == "kda" else 0, self.W,
                    self.r, self.K, self.smoothing, self.P, self.quantize, self.bf16_buffer,
                    self.bits, sm, ss)

    @property
    def ga(self) -> int:
        return self.dk if self.gate == "kda" else 1


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(C.POINTER(t))


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def empty_views(cfg: Cfg, nh: int) -> dict:
    return {"codes": np.zeros((nh, cfg.dk, cfg.dv), np.int8),
            "m": np.zeros((nh, cfg.dk), np.float32),
            "s": np.zeros((nh, cfg.dv), np.float32),
            "c": np.zeros((nh, max(cfg.r, 1), cfg.dk), np.float32)[:, : cfg.r].copy(),
            "w": np.zeros((nh, max(cfg.r, 1), cfg.dv), np.float32)[:, : cfg.r].copy(),
            "hp": np.zeros((nh, max(cfg.P, 1), cfg.dv), np.uint16)}


def _views_struct(v: dict) -> _Views:
    for key in ("codes", "m", "s", "c", "w", "hp"):
        assert v[key].flags["C_CONTIGUOUS"], key
    return _Views(_p(v["codes"], C.c_int8), _p(v["m"], C.c_float), _p(v["s"], C.c_float),
                  _p(v["c"], C.c_float) if v["c"].size else None,
                  _p(v["w"], C.c_float) if v["w"].size else None,
                  _p(v["hp"], C.c_uint16))


def _one_view(v: dict, h: int) -> dict:
    return {k: v[k][h] for k in v}


def step(cfg: Cfg, S: np.ndarray, q, k, v, beta: float, alpha) -> tuple[np.ndarray, np.ndarray]:
    """One recurrence token on a single head; returns (new S, o) in float64."""
    S = np.ascontiguousarray(np.array(S, dtype=np.float64))
    o = np.zeros(cfg.dv, np.float64)
    a = _f32(np.atleast_1d(alpha))
    lib().lqo_step(C.byref(cfg.c()), _p(S, C.c_double), _p(_f32(q), C.c_float),
                   _p(_f32(k), C.c_float), _p(_f32(v), C.c_float), C.c_float(beta),
                   _p(a, C.c_float), _p(o, C.c_double))
    return S, o


def quantize(cfg: Cfg, S, hp_rows=None, want_ratio: bool = False) -> dict:
    """Q on one head: float32 state [dk, dv] -> view dict (plus 'ratio' = x/s)."""
    S = _f32(S)
    v = _one_view(empty_views(cfg, 1), 0)
    v = {k: np.ascontiguousarray(a) for k, a in v.items()}
    hr = _i32(hp_rows if hp_rows is not None else np.zeros(1, np.int32))
    ratio = np.zeros((cfg.dk, cfg.dv), np.float64) if want_ratio else None
    st = _views_struct(v)
    vv = C.cast(C.pointer(st), C.c_void_p)
    lib().lqo_quantize(C.byref(cfg.c()), _p(hr, C.c_int), _p(S, C.c_float), vv,
                       _p(ratio, C.c_double) if want_ratio else None)
    if want_ratio:
        v["ratio"] = ratio
    return v


def dequantize(cfg: Cfg, view: dict, hp_rows=None) -> np.ndarray:
    """Window-start state Deq(C, m, s) + sum_j c_j w_j^T of one head (float64)."""
    v = {k: np.ascontiguousarray(view[k]) for k in ("codes", "m", "s", "c", "w", "hp")}
    hr = _i32(hp_rows if hp_rows is not None else np.zeros(1, np.int32))
    S = np.zeros((cfg.dk, cfg.dv), np.float64)
    st = _views_struct(v)
    lib().lqo_dequantize(C.byref(cfg.c()), _p(hr, C.c_int), C.cast(C.pointer(st), C.c_void_p),
                         _p(S, C.c_double))
    return S


def run(cfg: Cfg, inputs: dict, *, S0=None, view=None, hp_rows=None,
        flush_last: bool = False, nthreads: int | None = None, phase=None) -> dict:
    """Decode T tokens of nh independent heads.

    phase [nh] (optional): staggered windows, head h's first window holding
    W - phase[h] tokens (lqo_run).

    inputs: q, k [T, nh, dk]; v [T, nh, dv]; beta [T, nh]; alpha [T, nh] or
    [T, nh, dk] (already one entry per value head).  Give S0 [nh, dk, dv] or a
    starting `view` (dict of head-major arrays).  Returns o [T, nh, dv], view,
    S (state after the run), S_pre (state before the last flush), n.
    """
    q = _f32(inputs["q"]); k = _f32(inputs["k"]); v = _f32(inputs["v"])
    beta = _f32(inputs["beta"]); alpha = _f32(inputs["alpha"])
    T, nh = q.shape[0], q.shape[1]
    if alpha.ndim == 2:
        alpha = alpha[..., None]
    assert alpha.shape[-1] == cfg.ga
    views = empty_views(cfg, nh)
    from_view = 0
    if view is not None:
        for key in views:
            if key in view:
                views[key][...] = np.asarray(view[key]).reshape(views[key].shape)
        from_view = 1
    S0a = _f32(S0 if S0 is not None else np.zeros((nh, cfg.dk, cfg.dv), np.float32))
    hr = _i32(hp_rows if hp_rows is not None else np.zeros((nh, max(cfg.P, 1)), np.int32))
    o = np.zeros((T, nh, cfg.dv), np.float64)
    S = np.zeros((nh, cfg.dk, cfg.dv), np.float64)
    S_pre = np.zeros((nh, cfg.dk, cfg.dv), np.float64)
    n = np.zeros(nh, np.int32)
    st = _views_struct(views)
    lib().lqo_run(C.byref(cfg.c()), C.c_int(nh), _p(hr, C.c_int), C.c_int(from_view),
                  _p(S0a, C.c_float), C.cast(C.pointer(st), C.c_void_p), C.c_int(T),
                  _p(q, C.c_float), _p(k, C.c_float), _p(v, C.c_float),
                  _p(beta, C.c_float), _p(alpha, C.c_float), _p(o, C.c_double),
                  _p(S, C.c_double), _p(S_pre, C.c_double), _p(n, C.c_int),
                  C.c_int(1 if flush_last else 0), C.c_int(nthreads or os.cpu_count() or 1),
                  _p(_i32(phase), C.c_int) if phase is not None else None)
    if cfg.r == 0:
        views["c"] = views["c"][:, :0]
        views["w"] = views["w"][:, :0]
    return {"o": o, "view": views, "S": S, "S_pre": S_pre, "n": n}


def prefill(cfg: Cfg, inputs: dict, S0=None, nthreads: int | None = None) -> np.ndarray:
    """Plain FP recurrence from S0 (zeros by default); returns the state, float64."""
    c2 = Cfg(**{**cfg.__dict__, "quantize": 0})
    return run(c2, inputs, S0=S0, nthreads=nthreads)["S"]


FIT_ROUNDS = 3


def fit_static(cfg: Cfg, states, weight=None) -> dict:
    """Static key-row / value-column scales of one head fitted on calibration
    states [n, dk, dv] (lqo_fit_static).  Returns m [dk], s [dv] and the
    objective after the start and after every round."""
    st = _f32(states)
    m = np.zeros(cfg.dk, np.float32)
    s = np.zeros(cfg.dv, np.float32)
    obj = np.zeros(FIT_ROUNDS + 1, np.float64)
    w = None if weight is None else np.ascontiguousarray(np.asarray(weight, np.float64))
    lib().lqo_fit_static(C.byref(cfg.c()), C.c_int(st.shape[0]), _p(st, C.c_float),
                         _p(w, C.c_double) if w is not None else None, _p(m, C.c_float),
                         _p(s, C.c_float), _p(obj, C.c_double))
    return {"m": m, "s": s, "obj": obj}


def fit_objective(cfg: Cfg, states, m, s, weight=None) -> float:
    """The fit's weighted error of scales m [dk], s [dv] on states [n, dk, dv]."""
    st = _f32(states)
    w = None if weight is None else np.ascontiguousarray(np.asarray(weight, np.float64))
    fn = lib().lqo_fit_objective
    fn.restype = C.c_double
    return fn(C.byref(cfg.c()), C.c_int(st.shape[0]), _p(st, C.c_float),
              _p(w, C.c_double) if w is not None else None, _p(_f32(m), C.c_float), _p(_f32(s), C.c_float))


def damp_energy(cfg: Cfg, states) -> np.ndarray:
    """Quantization-error energy per key row, summed over states [n, dk, dv]."""
    st = _f32(states)
    E = np.zeros(cfg.dk, np.float64)
    lib().lqo_damp_energy(C.byref(cfg.c()), C.c_int(st.shape[0]), _p(st, C.c_float),
                          _p(E, C.c_double))
    return E


def damp_score(E, gates) -> np.ndarray:
    """DAMP risk score per key row: E [dk] (calibration error energy) times
    1 / (1 - mean decay); gates [n, ga] are the calibration decays of the head
    (ga = dk per channel for KDA, 1 for GDN) (lqo_damp_score)."""
    e = np.ascontiguousarray(np.asarray(E, dtype=np.float64))
    g = _f32(gates)
    if g.ndim == 1:
        g = g[:, None]
    out = np.zeros(e.shape[0], np.float64)
    lib().lqo_damp_score(C.c_int(e.shape[0]), C.c_int(g.shape[1]), C.c_int(g.shape[0]), _p(g, C.c_float),
                         _p(e, C.c_double), _p(out, C.c_double))
    return out


def damp_select(score, P: int) -> np.ndarray:
    """Top-P rows by score (ties to the lower index), in increasing row order."""
    sc = np.ascontiguousarray(np.asarray(score, dtype=np.float64))
    rows = np.zeros(P, np.int32)
    lib().lqo_damp_select(C.c_int(sc.shape[0]), C.c_int(P), _p(sc, C.c_double), _p(rows, C.c_int))
    return rows


def bf16_rne(x: float) -> int:
    return int(lib().lqo_bf16_rne(C.c_float(x)))


def bf16_to_float(h: int) -> float:
    return float(lib().lqo_bf16_to_float(C.c_uint16(h)))


def per_head_inputs(tok: dict, H: int, heads=None) -> dict:
    """Generator tensors [T, B, Hk|H, ...] -> oracle layout [T, nh, ...].

    q/k of value head h come from q/k head floor(h*Hk/H).  `heads` selects a
    list of (b, h) pairs; by default all of them in (b, h) order.
    """
    import torch
    q, k, v = tok["q"], tok["k"], tok["v"]
    beta, alpha = tok["beta"], tok["alpha"]
    T, B, Hk = q.shape[0], q.shape[1], q.shape[2]
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    bi = torch.tensor([b for b, _ in heads], dtype=torch.long)
    hi = torch.tensor([h for _, h in heads], dtype=torch.long)
    gi = (hi * Hk) // H

    def sel(x, hidx):
        return x[:, bi.to(x.device), hidx.to(x.device)].cpu().numpy()

    return {"q": sel(q, gi), "k": sel(k, gi), "v": sel(v, hi), "beta": sel(beta, hi),
            "alpha": sel(alpha, hi)}
