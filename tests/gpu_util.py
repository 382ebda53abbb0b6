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


# Codes bar: bit-exact except 1 LSB on at most 0.01% of the entries, and every
# differing code at a rounding tie -- within the band that the bounded
# difference of the two sides' inputs to that code's rounding can move its
# quotient x/s (check_quantized).
CODE_FLIP_FRAC = 1e-4
FLUSH_FLIP_FRAC = CODE_FLIP_FRAC
# Inputs accumulated over many more tokens than the benchmark windows (W = 32,
# 64): windows of 200 and more tokens and the 2048-token prefill state.  The
# two sides' FP32-vs-double state difference grows with the accumulation
# (~4e-6 of max|S| at W = 200 against ~5e-7 at W <= 64), and the share of
# codes within that difference of a rounding tie with it: the oracle's own
# quantizer applied to the GPU's exported pre-flush FP32 state of W = 200
# windows already differs from its quantization of its double state on
# ~1e-4 of the codes.  Bar there: 2e-4, every flip still asserted at a tie.
LONG_ACCUMULATION_FLIP_FRAC = 2e-4

U32 = 2.0 ** -24   # unit roundoff of float32


# Rounding errors of float32 sums are judged with the probabilistic bound of
# Higham and Mary ("A new approach to probabilistic rounding error analysis",
# SIAM J. Sci. Comput. 41(5), 2019): with independent, mean-zero rounding
# errors, a sum over a path of n roundings is within
#     gamma_p(n) = exp(lam sqrt(n) u + n u^2 / (1 - u)) - 1  ~  lam sqrt(n) u
# of its magnitude sum except with probability below 2 exp(-lam^2 (1-u)^2 / 2)
# (about 1e-14 at lam = 8); the worst-case bound n u / (1 - n u) is orders of
# magnitude wider than what float32 sums show in practice.
LAMBDA = 8.0


def gamma(n: int) -> float:
    """Probabilistic relative-error bound of a float32 sum along n roundings."""
    return float(np.expm1(LAMBDA * np.sqrt(n) * U32 + n * U32 * U32 / (1.0 - U32)))


def _bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).bfloat16().float().numpy()


def _bf16_risk(x32: np.ndarray, dx: np.ndarray) -> np.ndarray:
    """Elements whose BF16 rounding may differ for an input within dx of x32
    (a rounding boundary -- half a BF16 step from a representable value -- is
    closer than dx); returns one BF16 step at those elements, else 0."""
    r = _bf16_round(x32).astype(np.float64)
    ax = np.maximum(np.abs(r), 1e-38)
    step = 2.0 ** (np.floor(np.log2(ax)) - 7)          # spacing of BF16 values at |r|
    dist = np.abs(0.5 * step - np.abs(x32.astype(np.float64) - r))
    return np.where(dist <= dx + 2 * U32 * np.abs(x32), 2 * step, 0.0)


def _gate_chain(a: np.ndarray, g: np.ndarray) -> np.ndarray:
    """The BF16 buffer's decay chain (float32): the product, taken 64 binades
    up when it falls below 2^-64, restarted at 1 below 2^-128."""
    a = np.asarray(a, np.float32)
    p = (a * g).astype(np.float32)
    p2 = ((a * np.float32(2.0 ** 64)).astype(np.float32) * g).astype(np.float32)
    low = (p >= 0) & (p < np.float32(2.0 ** -64))
    return np.where(low, np.where(p2 >= np.float32(2.0 ** -64), p2, np.float32(1.0)), p).astype(np.float32)


def window_state_bound(oc: O.Cfg, view: dict, tok: dict, hp_rows=None, risk_cols: bool = False):
    """Per-element bound on |S_gpu - S| for the state at the end of one window
    of n = len(tok["k"]) tokens of one head, started from the quantized view
    `view` (oracle layout), S being the exact recurrence from that view.

    The kernels keep S_t = Gamma_t [Deq + sum_j c_j w_j^T + sum_e ktil_e u_e^T]
    and form each step's y = S'^T k as float32 sums of the terms' products,
    then u = beta (v - y); the window end rebuilds the state as a float32 sum
    of the same terms (three-pass TF32 products, float32 accumulation).  With
    M the element-wise sum of |terms| (decayed like the state), a step's
    rounding is
        |r_y,c| <= gamma(N_y) sum_i |k_i| M'_ic,   rho_c = beta r_y,c + 2 u |u_c|,
    and the error of the state that the GPU's u's define evolves as
        dS_new = (I - beta k k^T) D dS + k rho^T,
    a contraction of the inherited part (beta in (0, 1), D <= 1), so the
    2-norm of each column's error grows by at most |k| |rho_c| a step.  At the
    window end, |dS_ic| <= e_ic + gamma(N_S) M_ic + u |S_ic|.  N counts the roundings on the longest summation path (dot products
    over d_k, the r + n entries, the decay products and the divisions of
    ktil, the TF32 split of each product).  With the BF16 buffer both sides
    round k / Gamma and u to the same BF16 values, so a u differs only where
    its FP32 value lies within the error of y of a BF16 rounding boundary,
    and then by at most one BF16 step; the update's key Gamma bf16(k/Gamma)
    differs slightly from k, so the map grows norms by at most
    1 + beta |kg - k| |k| a step.  With risk_cols, also returns the value
    columns in which some token's BF16 u may round the other way."""
    dk, dv, r = oc.dk, oc.dv, oc.r
    k = np.asarray(tok["k"], np.float64)
    v = np.asarray(tok["v"], np.float64)
    beta = np.asarray(tok["beta"], np.float64).reshape(-1)
    alpha = np.asarray(tok["alpha"], np.float32)
    n = k.shape[0]
    cw = np.zeros((dk, dv))
    cwa = np.zeros((dk, dv))
    for j in range(r):
        o = np.outer(np.asarray(view["c"][j], np.float64), np.asarray(view["w"][j], np.float64))
        cw += o
        cwa += np.abs(o)
    S = O.dequantize(oc, view, hp_rows=hp_rows)
    M = np.abs(S - cw) + cwa
    Ec = np.zeros(dv)
    e = np.zeros((dk, dv))
    E = r + n
    n_y = dk + 2 * E + 2 * n + 40
    n_s = E + 2 * n + 40
    gam32 = np.ones(dk if oc.gate == "kda" else 1, np.float32)
    risk = np.zeros(dv, bool)
    for t in range(n):
        a = alpha[t].reshape(-1).astype(np.float64)
        d = a[:, None] if oc.gate == "kda" else a[0]
        S *= d
        M *= d
        Ec *= a.max()
        e *= d
        kn = float(np.linalg.norm(k[t]))
        y = S.T @ k[t]
        ry = gamma(n_y) * (M.T @ np.abs(k[t]))
        if oc.bf16_buffer:
            gam32 = _gate_chain(alpha[t].reshape(-1), gam32)
            uf = (beta[t] * (v[t] - y)).astype(np.float32)
            rho = _bf16_risk(uf, beta[t] * (ry + Ec * kn) + 2 * U32 * np.abs(uf))
            risk |= rho > 0
            u = _bf16_round(uf).astype(np.float64)
            g = np.broadcast_to(gam32, (dk,)).astype(np.float32)
            kt = g.astype(np.float64) * _bf16_round((k[t].astype(np.float32) / g).astype(np.float32))
            Ec *= 1.0 + beta[t] * float(np.linalg.norm(kt - k[t])) * kn
        else:
            u = beta[t] * (v[t] - y)
            rho = beta[t] * ry + 2 * U32 * np.abs(u)
            kt = k[t]
        e = np.sqrt(e ** 2 + np.outer(kt, beta[t] * kn * Ec + rho) ** 2)
        S += np.outer(kt, u)
        M += np.outer(np.abs(kt), np.abs(u))
        Ec = np.sqrt(Ec ** 2 + (float(np.linalg.norm(kt)) * rho) ** 2)
    bound = e + gamma(n_s) * M + U32 * np.abs(S)
    return (bound, risk) if risk_cols else bound


def check_quantized(oc: O.Cfg, got: dict, want: dict, ratio: np.ndarray, S_ref: np.ndarray, dS, hp_rows=None,
                    label: str = "", risk_cols=None) -> dict:
    """One head's quantized view from the GPU (`got`, oracle layout) against
    the oracle's (`want`) for the state S_ref the oracle quantized, when the
    GPU's input state is within dS (element-wise bound, or 0) of S_ref.

    Bounds, first order in the differences, from the method's steps:
      residual   |dR| <= dS + sum_j |c_j w_j^T (GPU) - c_j w_j^T (oracle)|
                         + (r + 2) u (|S_ref| + sum_j |c_j w_j^T|)
      row scale  |dm_i| <= RMS_c |dR_ic| + 3 u m_i        (RMS is 1-Lipschitz)
      x = R / m  |dx| <= |dR| / m + |x| |dm| / m + 2 u |x|
      col scale  |ds_c| <= max_i |dx_ic| / qmax + 2 u s_c  (max is 1-Lipschitz)
      quotient   |dq| <= |dx| / s + |q| |ds| / s + 3 u |q|
    (fixed scales, smoothing 2: m and s equal; smoothing 0: m = 1).  Asserts
    m and s within their bounds and every GPU code among the roundings of
    [q - |dq|, q + |dq|] (q the oracle's quotient).  Where that bound is
    below half an LSB and outside degenerate columns, a code differs by at
    most 1 LSB, and only at a rounding tie (q within |dq| of a half-integer);
    a bound of half an LSB or more leaves the code undetermined (a tie is
    always within reach).  A column is degenerate when the oracle's
    whole residual column is no larger than its bound |dR| -- the noise left
    when the compensators take a state of rank <= r whole: its codes are not
    determined by the state's FP32 value, and only the range applies.
    risk_cols: value columns whose buffered BF16 u may round either way (the
    buffer's own rounding tie); their flips are counted apart.
    Returns n (differing determined codes outside risk columns), n_risk,
    n_undetermined (differing codes in degenerate columns or with a bound of
    half an LSB or more), total and the largest band a counted flip used."""
    dk, dv, r = oc.dk, oc.dv, oc.r
    qmax = (1 << ((oc.bits or 8) - 1)) - 1
    P = oc.P
    int8_rows = np.ones(dk, bool)
    if P:
        int8_rows[np.asarray(hp_rows)] = False
    cwo = np.zeros((dk, dv))
    cwa = np.zeros((dk, dv))
    dcw = np.zeros((dk, dv))
    for j in range(r):
        o = np.outer(np.asarray(want["c"][j], np.float64), np.asarray(want["w"][j], np.float64))
        g = np.outer(np.asarray(got["c"][j], np.float64), np.asarray(got["w"][j], np.float64))
        cwo += o
        cwa += np.abs(o)
        dcw += np.abs(g - o)
    dR = dS + dcw + (r + 2) * U32 * (np.abs(S_ref) + cwa)
    mo = np.asarray(want["m"], np.float64)
    mg = np.asarray(got["m"], np.float64)
    so = np.asarray(want["s"], np.float64)
    sg = np.asarray(got["s"], np.float64)
    dm = np.abs(mg - mo)
    if oc.smoothing == 1:
        bm = np.sqrt((dR ** 2).mean(axis=1)) + 3 * U32 * mo
        bad = int8_rows & (dm > bm)
        assert not bad.any(), f"{label}: row scale m off by {dm[bad].max():.3e} > bound {bm[bad].max():.3e}"
    else:
        assert (dm[int8_rows] == 0).all(), f"{label}: fixed row scales changed"
    R_ref = S_ref - cwo
    x = R_ref / mo[:, None]
    dx = dR / mo[:, None] + np.abs(x) * (dm / mo)[:, None] + 2 * U32 * np.abs(x)
    ds = np.abs(sg - so)
    if oc.smoothing == 2:
        assert (ds == 0).all(), f"{label}: fixed column scales changed"
    else:
        bs = dx[int8_rows].max(axis=0) / qmax + 2 * U32 * so
        bad = ds > bs
        assert not bad.any(), f"{label}: column scale s off by {ds[bad].max():.3e} > bound {bs[bad].max():.3e}"
    sden = np.where(so > 0, so, np.inf)
    q = np.asarray(ratio, np.float64)
    band = dx / sden[None, :] + np.abs(q) * (ds / sden)[None, :] + 3 * U32 * np.abs(q)
    # a zero column scale on the oracle's side: its codes are 0; the GPU's
    # are undetermined if its residual column can be nonzero
    zc = so == 0
    band[:, zc] = np.where(dR[:, zc] > 0, np.inf, 0.0)
    cg = np.asarray(got["codes"]).astype(np.int32)
    co = np.asarray(want["codes"]).astype(np.int32)
    d = cg - co
    # every rounding of a quotient in [q - band, q + band], clamped to the range
    lo = np.clip(np.ceil(q - band - 0.5), -qmax, qmax)
    hi = np.clip(np.floor(q + band + 0.5), -qmax, qmax)
    valid = np.isfinite(band)
    out_of_range = int8_rows[:, None] & valid & ((cg < lo) | (cg > hi))
    assert not out_of_range.any(), (f"{label}: {int(out_of_range.sum())} codes outside the roundings their "
                                    f"bounded quotient allows (largest |diff| {np.abs(d[out_of_range]).max()} LSB)")
    rows_i8 = np.where(int8_rows)[0]
    degenerate = np.abs(R_ref[rows_i8]).max(axis=0) <= dR[rows_i8].max(axis=0)
    # a quotient whose bound reaches half an LSB or more always has a rounding
    # tie within reach: its code is not determined to 1 LSB by the FP32
    # arithmetic (a residual element left by the compensators' cancellation of
    # a state element thousands of times larger)
    determined = int8_rows[:, None] & ~degenerate[None, :] & (band < 0.5)
    flips = (d != 0) & determined
    assert np.abs(d[determined]).max(initial=0) <= 1, f"{label}: a determined code differs by more than 1 LSB"
    tie = np.abs(np.abs(q - np.trunc(q)) - 0.5)
    off = flips & (tie > band)
    assert not off.any(), (f"{label}: {int(off.sum())} differing codes away from a rounding tie "
                           f"(distance {tie[off].min():.3e} > band {band[off].max():.3e})")
    used = float((tie[flips] / np.maximum(band[flips], 1e-300)).max()) if flips.any() else 0.0
    risky = np.zeros(dv, bool) if risk_cols is None else np.asarray(risk_cols, bool)
    n_risk = int((flips & risky[None, :]).sum())
    return {"n": int((flips & ~risky[None, :]).sum()), "n_risk": n_risk,
            "n_undetermined": int(((d != 0) & int8_rows[:, None] & ~determined).sum()),
            "total": int(int8_rows.sum()) * dv, "band_used": used,
            "band_median": float(np.median(band[int8_rows]))}


def assert_flush_params(cfg: lq.Config, got: dict, want: dict, S_pre: np.ndarray, hp_rows, label: str = "",
                        rel: float = 1e-3):
    """The window-start state the GPU's flushed parameters produce: with the
    oracle's codes on both sides (code flips are judged by check_quantized),
    Deq(C; m, s, BF16 rows) + sum_j c_j w_j^T from the GPU's parameters must
    match the oracle's within `rel` of max|S_pre| per head -- the FP32-state
    bar.  `got`/`want` are oracle-layout views [nh, ...]; hp_rows are per-head
    row lists or None."""
    oc = ocfg(cfg)
    nh = S_pre.shape[0]
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
    assert stats.get("max_diff", 0) <= 1, f"{label}: a code differs by {stats['max_diff']} LSB"
    assert stats["n"] <= frac * stats["total"] + 1, \
        f"{label}: {stats['n']}/{stats['total']} codes differ (bar {frac:.0e})"


def head_view(v: dict, h: int) -> dict:
    return {k: v[k][h] for k in ("codes", "m", "s", "c", "w", "hp")}


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
