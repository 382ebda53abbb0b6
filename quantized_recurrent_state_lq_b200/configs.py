"""Synthetic decode workloads for the windowed INT8 recurrent-state path.

Five workloads, named by what they are and their sizes.  They stand in for the
decode-time state traffic of the models the LeapQuant project page evaluates
("LeapQuant: Efficient Linear Attention with Accurate Recurrent State
Quantization", accuracy table and kernel-speedup paragraph): no dataset items,
no trained weights, only seeded synthetic tensors with the stated shapes and
distributions.

Field meanings
--------------
gate        "gdn" (one scalar decay per head, Gated DeltaNet) or "kda" (one
            decay per key channel, Kimi Delta Attention); update rules from the
            LinQuant page, appendix Table 3 (state-update rules).
B, H, Hk    batch, value heads, query/key heads (GQA when Hk < H; value head h
            reads q/k head floor(h*Hk/H)).
dk, dv      key and value head sizes; the state S is dk x dv (key rows, value
            columns).
prefill     tokens of FP32 recurrence that produce the initial state.
T           decode tokens; W window length; r compensator tokens;
K           power-iteration steps per compensator; P DAMP rows kept in BF16.
n_out_rows  outlier key rows and value columns injected after the prefill;
out_lo/hi   their multiplicative factors, uniform in [out_lo, out_hi].
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    gate: str
    B: int
    H: int
    Hk: int
    dk: int
    dv: int
    prefill: int
    T: int
    W: int
    r: int
    K: int = 8
    smoothing: int = 1
    P: int = 0
    n_out_rows: int = 3
    n_out_cols: int = 3
    out_lo: float = 10.0
    out_hi: float = 50.0
    seed: int = 0
    calib_prefills: int = 0
    calib_tokens: int = 0
    buffer_bf16: int = 0         # 1: the traffic-lean BF16 window buffer (an option, not a config)
    bits: int = 8                # code width of the quantized state: 8, or the packed 6 / 4 bits

    @property
    def heads(self) -> int:
        return self.B * self.H

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# Tiny GDN case the oracle finishes in seconds (d=64, two heads).
TINY_GDN = Workload(
    name="gdn_tiny_b1_h2_d64_w16_r2", gate="gdn", B=1, H=2, Hk=2, dk=64, dv=64,
    prefill=512, T=256, W=16, r=2, n_out_rows=4, n_out_cols=4, out_lo=20.0,
    out_hi=20.0, seed=0)

# GDN at serving shape with grouped q/k heads.
GDN_SERVING = Workload(
    name="gdn_b64_h32_hk16_d128_w32_r4", gate="gdn", B=64, H=32, Hk=16, dk=128,
    dv=128, prefill=2048, T=1024, W=32, r=4, seed=1)

# KDA with per-key-channel decay.
KDA_B256 = Workload(
    name="kda_b256_h32_d128_w32_r4", gate="kda", B=256, H=32, Hk=32, dk=128,
    dv=128, prefill=2048, T=512, W=32, r=4, seed=2)

# Prefix-cache scale GDN, 1024 independent states.
GDN_PREFIX_CACHE = Workload(
    name="gdn_b1024_h16_d128_w64_r4", gate="gdn", B=1024, H=16, Hk=16, dk=128,
    dv=128, prefill=2048, T=128, W=64, r=4, seed=3)

# DAMP-style mixed precision: 16 BF16 key rows per head, the rest INT8.
GDN_DAMP = Workload(
    name="gdn_damp_b256_h32_d128_p16_w32_r2", gate="gdn", B=256, H=32, Hk=32,
    dk=128, dv=128, prefill=2048, T=1024, W=32, r=2, P=16, seed=4,
    calib_prefills=64, calib_tokens=1024)

WORKLOADS = [TINY_GDN, GDN_SERVING, KDA_B256, GDN_PREFIX_CACHE, GDN_DAMP]
BY_NAME = {w.name: w for w in WORKLOADS}
