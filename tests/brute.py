"""Brute-force numpy twins used to pin the oracle on tiny heads.

These are written from the mathematics, independently of `oracle/lq_oracle.c`:
the recurrence as literal matrix products in the pages' own (d_v x d_k) form,
the power iteration by its closed form (R^T R)^K w0, and codes by exhaustive
search over all 255 levels.  They are slow and only meant for d <= 16.
"""
from __future__ import annotations

import numpy as np

f32 = np.float32


def step_pages_form(Sp: np.ndarray, q, k, v, beta, alpha, gate: str):
    """One token in the LinQuant page's Table 3 form, S_pages is (d_v x d_k).

    GDN: S_t = a S_{t-1} (I - b k k^T) + b v k^T
    KDA: S_t = S_{t-1} diag(a) (I - b k k^T) + b v k^T
    Output o = S_t q.
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    dk = k.shape[0]
    P = np.eye(dk) - beta * np.outer(k, k)
    if gate == "gdn":
        Sn = float(np.asarray(alpha).reshape(-1)[0]) * Sp @ P + beta * np.outer(v, k)
    else:
        Sn = Sp @ np.diag(np.asarray(alpha, np.float64)) @ P + beta * np.outer(v, k)
    return Sn, Sn @ q


def power_closed_form(R: np.ndarray, K: int) -> np.ndarray:
    """w_K = (R^T R)^K w0 / |.|, w0 = 1/sqrt(d_v) -- the iterate of K power steps."""
    dv = R.shape[1]
    w0 = np.full(dv, 1.0 / np.sqrt(dv))
    G = R.T @ R
    g = np.linalg.norm(G)
    if g > 0:
        G = G / g          # rescaling does not change the direction
    x = np.linalg.matrix_power(G, K) @ w0
    return x / np.linalg.norm(x)


def codes_exhaustive(x: np.ndarray, s: np.ndarray, qmax: int = 127) -> np.ndarray:
    """argmin over k in [-qmax, qmax] of |x/s - k|, ties to the even k."""
    levels = np.arange(-qmax, qmax + 1, dtype=np.float64)
    out = np.zeros(x.shape, np.int64)
    for i in range(x.shape[0]):
        for c in range(x.shape[1]):
            if s[c] == 0:
                continue
            t = float(x[i, c]) / float(s[c])
            d = np.abs(t - levels)
            best = np.flatnonzero(d == d.min())
            if best.size > 1:
                best = best[(levels[best].astype(np.int64) % 2) == 0]
            out[i, c] = int(levels[best[0]])
    return out


def quantize(S: np.ndarray, r: int, K: int, smoothing: bool = True, qmax: int = 127):
    """Brute-force quantizer Q on one head (no BF16 rows), codes in [-qmax, qmax].

    Float rounding happens where the method stores a float: compensator
    vectors, the residual handed to the codec, m and s, and x = R/m.
    """
    R = np.asarray(S, np.float32).astype(np.float64)
    cs, ws = [], []
    for _ in range(r):
        w = power_closed_form(R, K).astype(f32)
        c = (R @ w.astype(np.float64)).astype(f32)
        cs.append(c); ws.append(w)
        R = R - np.outer(c.astype(np.float64), w.astype(np.float64))
    R32 = R.astype(f32)
    if smoothing:
        m = np.sqrt((R32.astype(np.float64) ** 2).mean(axis=1)).astype(f32)
        m[m == 0] = 1
    else:
        m = np.ones(R.shape[0], f32)
    x = (R32 / m[:, None]).astype(f32)
    a = np.abs(x).max(axis=0).astype(f32)
    s = (a / f32(qmax)).astype(f32)
    codes = codes_exhaustive(x, s, qmax)
    dk, dv = R.shape
    return {"codes": codes, "m": m, "s": s, "c": np.array(cs, f32).reshape(r, dk),
            "w": np.array(ws, f32).reshape(r, dv), "R32": R32, "x": x}


def dequantize(view) -> np.ndarray:
    deq = ((view["codes"].astype(f32) * view["s"][None, :]).astype(f32) * view["m"][:, None]).astype(f32)
    S = deq.astype(np.float64)
    for c, w in zip(view["c"], view["w"]):
        S = S + np.outer(c.astype(np.float64), w.astype(np.float64))
    return S


def run_windowed(S0, toks, W: int, r: int, K: int, gate: str, smoothing=True, quantize_on=True,
                 qmax: int = 127, first: int | None = None):
    """Whole windowed decode of one head with literal matrices.

    toks: list of (q, k, v, beta, alpha).  first: length of the first window
    (W by default).  Returns (outputs, last view).
    """
    view = None
    if quantize_on:
        view = quantize(S0, r, K, smoothing, qmax)
        S = dequantize(view)
    else:
        S = np.asarray(S0, np.float64)
    Sp = S.T.copy()
    outs = []
    n = 0
    length = W if first is None else first
    for (q, k, v, beta, alpha) in toks:
        Sp, o = step_pages_form(Sp, q, k, v, beta, alpha, gate)
        outs.append(o)
        n += 1
        if quantize_on and n == length:
            view = quantize(Sp.T.astype(f32), r, K, smoothing, qmax)
            Sp = dequantize(view).T.copy()
            n = 0
            length = W
    return np.array(outs), view


ROWGRID = [0.5, 0.625, 0.75, 0.875, 1.0, 1.25, 1.5, 1.75, 2.0]
COLGRID = [1.0 - j / 16.0 for j in range(12)]


def _fit_err(R, m, s, qmax):
    """(R - Deq)^2 in double for one float32 entry under scales m, s."""
    dq = f32(0)
    if s != 0:
        x = f32(R) / f32(m)
        rq = np.float32(np.rint(f32(x) / f32(s)))
        rq = f32(min(max(rq, -qmax), qmax))
        dq = f32(f32(rq * f32(s)) * f32(m))
    d = float(R) - float(dq)
    return d * d


def fit_static(R, weight, qmax, rounds=3):
    """Coordinate descent for static scales on residuals R [n, dk, dv]
    (float32), written out loop by loop: start from the rows' RMS and the
    columns' amax / qmax; per round the columns (s0 x COLGRID), then the rows
    (m0 x ROWGRID), first best candidate kept."""
    n, dk, dv = R.shape
    w = np.ones(dk) if weight is None else np.asarray(weight, np.float64)
    m0 = np.zeros(dk, f32)
    for i in range(dk):
        ss = 0.0
        for t in range(n):
            for c in range(dv):
                ss += float(R[t, i, c]) * float(R[t, i, c])
        mi = f32(np.sqrt(ss / (n * dv)))
        m0[i] = mi if mi != 0 else f32(1)
    m = m0.copy()
    s0 = np.zeros(dv, f32)
    for c in range(dv):
        a = f32(0)
        for t in range(n):
            for i in range(dk):
                a = max(a, f32(abs(f32(R[t, i, c]) / m[i])))
        s0[c] = f32(a / f32(qmax))
    s = s0.copy()
    for _ in range(rounds):
        for c in range(dv):
            best, sb = np.inf, s[c]
            for g in COLGRID:
                sc = f32(s0[c] * f32(g))
                e = 0.0
                for t in range(n):
                    for i in range(dk):
                        e += w[i] * _fit_err(R[t, i, c], m[i], sc, qmax)
                if e < best:
                    best, sb = e, sc
            s[c] = sb
        for i in range(dk):
            best, mb = np.inf, m[i]
            for g in ROWGRID:
                mi = f32(m0[i] * f32(g))
                e = 0.0
                for t in range(n):
                    for c in range(dv):
                        e += _fit_err(R[t, i, c], mi, s[c], qmax)
                if e < best:
                    best, mb = e, mi
            m[i] = mb
    return m, s
