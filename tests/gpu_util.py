"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and the
oracle on the same seeded inputs, map between the two layouts, compare.

Directions of data flow: inputs come from the seeded generator (or from the
oracle, e.g. an oracle window-start state imported into the GPU state to
teacher-force a window); nothing computed by the CUDA path is ever fed to the
oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_recurrent_state_lq_b200 import configs, inputs as gen, lq

f32 = np.float32


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def ocfg(cfg: lq.Config, quantize: int = 1) -> O.Cfg:
    return O.Cfg(dk=cfg.dk, dv=cfg.dv, gate=cfg.gate, W=cfg.W, r=cfg.r, K=cfg.power_iters,
                 smoothing=cfg.smoothing, P=cfg.n_hp_rows, quantize=quantize,
                 bf16_buffer=cfg.buffer_bf16 if (quantize and cfg.mode == "window") else 0,
                 bits=cfg.state_bits if quantize else 8)


def head_rows(cfg: lq.Config, hp_rows):
    """[H, P] row lists -> per (b, h) head [B*H, P] for the oracle."""
    if cfg.n_hp_rows == 0:
        return None
    hr = np.asarray(hp_rows, np.int32)
    return np.ascontiguousarray(np.tile(hr, (cfg.B, 1)))


def gpu_view_to_oracle(cfg: lq.Config, view: dict, hp_rows) -> dict:
    """GPU view (compact INT8 rows) -> oracle view (full [dk, dv] codes, zero on BF16 rows)."""
    B, H, dk, dv, P = cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.n_hp_rows
    nh = B * H
    codes_c = view["codes"].cpu().numpy().reshape(nh, dk - P, dv)
    codes = np.zeros((nh, dk, dv), np.int8)
    for b in range(B):
        for h in range(H):
            keep = np.setdiff1d(np.arange(dk), np.asarray(hp_rows[h])) if P else np.arange(dk)
            codes[b * H + h, keep] = codes_c[b * H + h]
    out = {"codes": codes,
           "m": view["m"].cpu().numpy().reshape(nh, dk).copy(),
           "s": view["s"].cpu().numpy().reshape(nh, dv).copy(),
           "c": view["comp_k"].cpu().numpy().reshape(nh, cfg.r, dk).copy(),
           "w": view["comp_v"].cpu().numpy().reshape(nh, cfg.r, dv).copy(),
           "hp": np.zeros((nh, max(P, 1), dv), np.uint16)}
    if P:
        out["hp"] = view["bf16_rows"].cpu().numpy().view(np.uint16).reshape(nh, P, dv).copy()
    return out


def oracle_view_to_gpu(cfg: lq.Config, ov: dict, hp_rows, device="cuda") -> dict:
    B, H, dk, dv, P = cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.n_hp_rows
    nh = B * H
    codes = np.zeros((nh, dk - P, dv), np.int8)
    for b in range(B):
        for h in range(H):
            keep = np.setdiff1d(np.arange(dk), np.asarray(hp_rows[h])) if P else np.arange(dk)
            codes[b * H + h] = ov["codes"][b * H + h][keep]
    v = lq.alloc_view(cfg, device)
    v["codes"].copy_(torch.from_numpy(codes.reshape(B, H, dk - P, dv)))
    v["m"].copy_(torch.from_numpy(np.asarray(ov["m"], f32).reshape(B, H, dk)))
    v["s"].copy_(torch.from_numpy(np.asarray(ov["s"], f32).reshape(B, H, dv)))
    if cfg.r:
        v["comp_k"].copy_(torch.from_numpy(np.asarray(ov["c"], f32).reshape(B, H, cfg.r, dk)))
        v["comp_v"].copy_(torch.from_numpy(np.asarray(ov["w"], f32).reshape(B, H, cfg.r, dv)))
    if P:
        hp = np.asarray(ov["hp"], np.uint16)[:, :P].reshape(B, H, P, dv).view(np.int16)
        v["bf16_rows"].copy_(torch.from_numpy(hp.copy()))
    return v


def rel_inf_rows(a: np.ndarray, ref: np.ndarray, axis=-1) -> np.ndarray:
    """||a - ref||_inf / ||ref||_inf along `axis` (one value per vector)."""
    num = np.abs(np.asarray(a, np.float64) - ref).max(axis=axis)
    den = np.abs(ref).max(axis=axis)
    return num / np.maximum(den, 1e-30)


# Codes bar where both sides quantize the SAME float32 state (lq_quantize_state,
# lq_state_init): bit-exact except 1 LSB on at most 0.01% of the entries.
CODE_FLIP_FRAC = 1e-4
# Codes after a window flush: the GPU quantizes its own FP32 end-of-window
# state, which differs from the oracle's double-precision one by ~1e-7
# relative (FP32 buffered updates and reconstruction).  A code can then differ
# wherever the oracle's x/s lies within that perturbation of a rounding
# boundary -- after the unconverged power iteration amplifies it by up to
# 1/(1 - sigma_{j+1}/sigma_j) (measured ~10) and the 127-level scale:
# 2 * 127 * 1e-7 * 10 * (cancellation of compensators, ~10) ~ 3e-4.  Bar:
# 1 LSB on at most 0.1% of the entries.
FLUSH_FLIP_FRAC = 1e-3


def compare_codes(gpu: np.ndarray, orc: np.ndarray, ratio: np.ndarray | None, tie_eps: float = 1e-3):
    """Compare INT8 codes.  Returns a dict: n (mismatches), total, max_diff (in
    LSB) and at_tie (mismatches whose oracle value x/s lies within tie_eps of a
    rounding tie -- the expected cause; the rest come from the FP32 residual
    differing from the oracle's double one where compensators cancel most of a
    row)."""
    d = gpu.astype(np.int32) - orc.astype(np.int32)
    mism = d != 0
    out = {"n": int(mism.sum()), "total": int(gpu.size), "max_diff": int(np.abs(d).max()) if d.size else 0,
           "at_tie": 0}
    if out["n"] and ratio is not None:
        frac = np.abs(ratio - np.trunc(ratio))
        out["at_tie"] = int((np.abs(frac - 0.5) < tie_eps)[mism].sum())
    return out


def assert_flush_params(cfg: lq.Config, got: dict, want: dict, S_pre: np.ndarray, hp_rows, label: str = "",
                        rel: float = 1e-3, guard: float = 1e-2):
    """m, s, BF16 rows and the compensators of a flush, judged by the
    window-start state they produce.  With the oracle's codes on both sides
    (flips are counted on their own), Deq(C; m, s, BF16 rows) + sum_j c_j w_j^T
    from the GPU's parameters must match the oracle's within `rel` of
    max|S_pre| per head -- the FP32-state bar.  Per-element m, s are only guarded against gross error
    (`guard` relative): an FP32 power iteration on a state whose leading
    singular values dwarf the residual moves a residual column's amax by far
    more, relatively, than it moves the state.  `got`/`want` are oracle-layout
    views [nh, ...]; hp_rows are per-head row lists or None."""
    oc = ocfg(cfg)
    nh = S_pre.shape[0]
    np.testing.assert_allclose(got["m"], want["m"], rtol=guard)
    np.testing.assert_allclose(got["s"], want["s"], rtol=guard, atol=1e-30)
    worst = 0.0
    for h in range(nh):
        hr = None if hp_rows is None else hp_rows[h]
        base = {"codes": want["codes"][h]}
        mine = dict(base, hp=got["hp"][h], m=got["m"][h], s=got["s"][h], c=got["c"][h], w=got["w"][h])
        ref = dict(base, hp=want["hp"][h], m=want["m"][h], s=want["s"][h], c=want["c"][h], w=want["w"][h])
        dg = O.dequantize(oc, mine, hp_rows=hr)
        dr = O.dequantize(oc, ref, hp_rows=hr)
        e = float(np.abs(dg - dr).max() / max(np.abs(S_pre[h]).max(), 1e-30))
        worst = max(worst, e)
    assert worst <= rel, f"{label}: window-start state from m, s, comps off by {worst:.2e} (bar {rel:.0e})"
    return worst


def assert_code_bar(stats: dict, label: str = "", frac: float = CODE_FLIP_FRAC):
    assert stats["max_diff"] <= 1, f"{label}: a code differs by {stats['max_diff']} LSB"
    assert stats["n"] <= frac * stats["total"] + 1, \
        f"{label}: {stats['n']}/{stats['total']} codes differ (bar {frac:.0e})"


def oracle_ratios(cfg: lq.Config, S_heads: np.ndarray, hp_rows_heads, head_cfg=None) -> np.ndarray:
    """x/s behind every oracle code, for float32 states S_heads [nh, dk, dv]
    (head_cfg(h): the oracle config of head h, for per-head fixed scales)."""
    oc = ocfg(cfg)
    out = np.zeros(S_heads.shape, np.float64)
    for h in range(S_heads.shape[0]):
        rows = None if hp_rows_heads is None else hp_rows_heads[h]
        c = oc if head_cfg is None else head_cfg(h)
        out[h] = O.quantize(c, S_heads[h].astype(f32), hp_rows=rows, want_ratio=True)["ratio"]
    return out


def prefill_state(wl: configs.Workload, tokens: int, heads=None) -> np.ndarray:
    """Oracle prefill from zero over `tokens` generator tokens, then the
    workload's outliers; returns float32 [B, H, dk, dv] (or the listed heads)."""
    pre = gen.token_inputs(wl, tokens, stream="prefill")
    oc = O.Cfg(dk=wl.dk, dv=wl.dv, gate=wl.gate, quantize=0)
    S = O.prefill(oc, O.per_head_inputs(pre, wl.H)).astype(f32).reshape(wl.B, wl.H, wl.dk, wl.dv)
    return gen.apply_outliers(torch.from_numpy(S), wl).numpy()


def step_args(tok: dict, t: int):
    return (tok["q"][t], tok["k"][t], tok["v"][t], tok["beta"][t], tok["alpha"][t])
