"""Algorithmic HBM bytes of the decode path -- what the method must move, not
what a kernel happens to move -- used for the roofline figures.

Per head and token of a window (n tokens already buffered, 0 <= n < W):
  IO      q, k read once per q/k head (shared by H/Hk value heads), v and o,
          beta, the gate (1 or dk floats)
  state   codes (dk-P)*dv*bits/8 (INT8, or packed 6 / 4 bits), BF16 rows 2*P*dv,
          m and s (dk+dv)*4,
          r compensators r*(dk+dv)*4, the n buffered entries n*(dk+dv)*4
          (n*(dk+dv)*2 with the BF16 buffer)
  append  one entry (dk+dv)*4 (or *2) and Gamma written (read too when n > 0)
At the window end the new state is written once: codes, BF16 rows, m, s and
the compensators.
"""
from __future__ import annotations

from .configs import Workload


def io_bytes(wl: Workload) -> float:
    G = wl.H // wl.Hk
    gate = wl.dk if wl.gate == "kda" else 1
    return 2 * wl.dk * 4 / G + 2 * wl.dv * 4 + 4 + gate * 4


def state_bytes(wl: Workload, P: int | None = None) -> int:
    P = wl.P if P is None else P
    return ((wl.dk - P) * wl.dv * wl.bits // 8 + 2 * P * wl.dv + 4 * (wl.dk + wl.dv)
            + 4 * wl.r * (wl.dk + wl.dv))


def gamma_bytes(wl: Workload, n: int) -> int:
    g = wl.dk if wl.gate == "kda" else 1
    return 4 * g * (2 if n > 0 else 1)


def token_entry_bytes(wl: Workload) -> int:
    """One buffered token (ktil, u): FP32, or BF16 with the traffic-lean buffer."""
    return (2 if wl.buffer_bf16 else 4) * (wl.dk + wl.dv)


def decode_launch_bytes(wl: Workload, n: int, flush: bool = False) -> float:
    """Bytes per head of the decode launch that buffers token n+1 of a window."""
    e = token_entry_bytes(wl)
    b = io_bytes(wl) + state_bytes(wl) + n * e
    if flush:
        b += state_bytes(wl)           # the new window-start state is written once
    else:
        b += e + gamma_bytes(wl, n)    # append the entry, keep Gamma
    return b


def window_bytes(wl: Workload) -> float:
    """Bytes per head for one whole window (W decode tokens, the last one flushing)."""
    return sum(decode_launch_bytes(wl, n, flush=(n == wl.W - 1)) for n in range(wl.W))


def nonflush_launch_bytes(wl: Workload) -> float:
    """Mean bytes per head of the W-1 launches that only buffer (n = 0 .. W-2)."""
    if wl.W < 2:
        return 0.0
    return sum(decode_launch_bytes(wl, n) for n in range(wl.W - 1)) / (wl.W - 1)


def fp32_step_bytes(wl: Workload) -> float:
    return io_bytes(wl) + 8 * wl.dk * wl.dv


def step_int8_bytes(wl: Workload) -> float:
    return io_bytes(wl) + 2 * state_bytes(wl)


def bits_per_value(wl: Workload) -> dict:
    """Effective bits per state value of the window-start state (the DAMP
    abstract reports its state-storage saving; it gives no definition, so both
    readings are reported): `payload` counts the codes and the BF16 rows only,
    (bits (dk-P) + 16 P) / dk; `total` adds the FP32 smoothing and column scales
    and the r compensators, 32 (dk + dv) (1 + r) / (dk dv).  The transient
    window buffer is excluded (it is the method's FP32 update stream)."""
    payload = (wl.bits * (wl.dk - wl.P) + 16 * wl.P) / wl.dk
    total = payload + 32 * (wl.dk + wl.dv) * (1 + wl.r) / (wl.dk * wl.dv)
    return {"payload": payload, "total": total, "fp32_reference": 32.0}


PREFILL_CHUNK = 16


def prefill_flops(wl: Workload, T: int) -> float:
    """Floating-point operations per head of the chunked prefill over T tokens
    (chunks of 16; counted as the kernel evaluates them, an FMA as 2):
      S^T (Gamma k), S^T (Gamma q), the state update      3 x 2 C dk dv + dk dv
      decayed keys / queries / update keys                3 C dk (+ 3 C dk exp2 for KDA)
      pair matrices A, P (i <= t)                         C(C+1)/2 x dk x (4, KDA 6 + 1 exp2)
      forward substitution, outputs                       C(C-1)/2 dv 2 + C(C+1)/2 dv 2 + 3 C dv
    exp2 counted as one operation."""
    C = PREFILL_CHUNK
    n = (T + C - 1) // C
    dk, dv = wl.dk, wl.dv
    kda = wl.gate == "kda"
    pairs = C * (C + 1) // 2
    per = (3 * 2 * C * dk * dv + dk * dv
           + 3 * C * dk * (2 if kda else 1)
           + pairs * dk * (7 if kda else 4)
           + (C * (C - 1) // 2) * dv * 2 + pairs * dv * 2 + 3 * C * dv)
    return float(n * per)
