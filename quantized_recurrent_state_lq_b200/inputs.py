"""Seeded synthetic inputs for the decode path.

This module draws random numbers and shapes them into the input distributions
of the synthetic workloads; it contains none of the recurrence or quantizer
arithmetic.  It is the only code that both the CUDA path and the CPU oracle
consume.  Everything is plain torch on whatever device the caller names, so
that a GPU run can draw its inputs in HBM and a test can copy a few heads of
the very same tensors to the host.

Distributions (one token, one head):
  q, k ~ N(0, 1) then L2-normalised; v ~ N(0, 1);
  beta = sigmoid(N(0, 1));
  GDN gate alpha = exp(-softplus(N(-4, 1)))           (about 0.98);
  KDA gate a_c  = exp(-softplus(N(mu_c, 0.5))), mu_c ~ U(-6, -1) fixed per
  head and key channel.
Outliers after the prefill: per head a fixed set of key rows and value columns
(chosen without replacement), each multiplied by a factor drawn uniformly in
[out_lo, out_hi]; the same positions for every batch entry.
"""
from __future__ import annotations

import torch

from .configs import Workload

# Stream tags keep the draws for different purposes independent.
_STREAM_DECODE = 1
_STREAM_PREFILL = 2
_STREAM_OUTLIER = 3
_STREAM_KDA_MU = 4
_STREAM_CALIB = 5
_STREAM_MATRIX = 6


def generator(seed: int, stream: int, chunk: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    # A plain mixing of the three integers into one 63-bit seed.
    s = (seed * 1_000_003 + stream) * 1_000_033 + chunk
    g.manual_seed(s & ((1 << 63) - 1))
    return g


def kda_mu(wl: Workload, device="cpu") -> torch.Tensor:
    """Per-head, per-key-channel mean of the KDA gate pre-activation, [H, dk]."""
    g = generator(wl.seed, _STREAM_KDA_MU, 0, device)
    u = torch.rand((wl.H, wl.dk), generator=g, device=device, dtype=torch.float32)
    return -6.0 + 5.0 * u


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def token_inputs(wl: Workload, T: int, *, stream: str = "decode", chunk: int = 0,
                 batch: int | None = None, device="cpu") -> dict:
    """Inputs for T consecutive tokens of all heads.

    Returns float32 tensors
      q, k   [T, B, Hk, dk]
      v      [T, B, H, dv]
      beta   [T, B, H]
      alpha  [T, B, H] (gdn) or [T, B, H, dk] (kda)
    `stream` selects decode / prefill / calibration draws; `chunk` lets a long
    sequence be drawn piecewise (chunk c covers its own T tokens).
    """
    tag = {"decode": _STREAM_DECODE, "prefill": _STREAM_PREFILL,
           "calib": _STREAM_CALIB}[stream]
    B = wl.B if batch is None else batch
    g = generator(wl.seed, tag, chunk, device)
    f32 = torch.float32
    q = _l2n(torch.randn((T, B, wl.Hk, wl.dk), generator=g, device=device, dtype=f32))
    k = _l2n(torch.randn((T, B, wl.Hk, wl.dk), generator=g, device=device, dtype=f32))
    v = torch.randn((T, B, wl.H, wl.dv), generator=g, device=device, dtype=f32)
    beta = torch.sigmoid(torch.randn((T, B, wl.H), generator=g, device=device, dtype=f32))
    if wl.gate == "gdn":
        pre = torch.randn((T, B, wl.H), generator=g, device=device, dtype=f32) - 4.0
    else:
        mu = kda_mu(wl, device)
        pre = torch.randn((T, B, wl.H, wl.dk), generator=g, device=device, dtype=f32) * 0.5 + mu
    alpha = torch.exp(-torch.nn.functional.softplus(pre))
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
            "beta": beta.contiguous(), "alpha": alpha.contiguous()}


def strong_decays(shape, mu: float, seed: int, device="cpu") -> torch.Tensor:
    """Decays exp(-softplus(N(mu, 0.5))) of the given shape (per key channel
    for KDA): mu = -1 is the strongest end of the KDA workload's range."""
    g = torch.Generator().manual_seed(seed)
    z = torch.randn(tuple(shape), generator=g, dtype=torch.float32) * 0.5 + mu
    return torch.exp(-torch.nn.functional.softplus(z)).to(device)


def with_vanishing_decays(alpha: torch.Tensor, seed: int, n: int = 6) -> torch.Tensor:
    """A copy of decays alpha [T, B, H] or [T, B, H, dk] with n seeded tokens'
    decays set to 1e-30 (even tokens) or exactly 0 (odd): one key channel of
    them for KDA, and for KDA every channel of the middle token at 1e-30."""
    a = alpha.clone()
    T = a.shape[0]
    g = torch.Generator().manual_seed(seed)
    for t in torch.randperm(T, generator=g)[:n].tolist():
        val = 0.0 if t % 2 else 1e-30
        if a.dim() == 4:
            a[t, ..., int(torch.randint(a.shape[-1], (1,), generator=g))] = val
        else:
            a[t] = val
    if a.dim() == 4:
        a[T // 2] = 1e-30
    return a


def outlier_spec(wl: Workload) -> dict:
    """Outlier key rows / value columns per head and their factors (CPU tensors).

    rows [H, n_out_rows] int64, row_f [H, n_out_rows] float32,
    cols [H, n_out_cols] int64, col_f [H, n_out_cols] float32.
    """
    g = generator(wl.seed, _STREAM_OUTLIER, 0, "cpu")
    rows, cols, rf, cf = [], [], [], []
    for _ in range(wl.H):
        rows.append(torch.randperm(wl.dk, generator=g)[: wl.n_out_rows])
        cols.append(torch.randperm(wl.dv, generator=g)[: wl.n_out_cols])
        rf.append(wl.out_lo + (wl.out_hi - wl.out_lo) *
                  torch.rand(wl.n_out_rows, generator=g, dtype=torch.float32))
        cf.append(wl.out_lo + (wl.out_hi - wl.out_lo) *
                  torch.rand(wl.n_out_cols, generator=g, dtype=torch.float32))
    return {"rows": torch.stack(rows), "cols": torch.stack(cols),
            "row_f": torch.stack(rf), "col_f": torch.stack(cf)}


def outlier_scale(wl: Workload, device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """Row and column multipliers [H, dk], [H, dv] (1 outside the outliers).

    The initial state of head h is S0[b, h] * row[h][:, None] * col[h][None, :]
    applied to the prefill state; that multiply is workload synthesis.
    """
    sp = outlier_spec(wl)
    row = torch.ones((wl.H, wl.dk), dtype=torch.float32)
    col = torch.ones((wl.H, wl.dv), dtype=torch.float32)
    for h in range(wl.H):
        row[h, sp["rows"][h]] = sp["row_f"][h]
        col[h, sp["cols"][h]] = sp["col_f"][h]
    return row.to(device), col.to(device)


def apply_outliers(S: torch.Tensor, wl: Workload) -> torch.Tensor:
    """S [B, H, dk, dv] -> S with the workload's outlier rows/columns scaled."""
    row, col = outlier_scale(wl, S.device)
    return (S * row[None, :, :, None] * col[None, :, None, :]).contiguous()


def random_state(n: int, dk: int, dv: int, *, seed: int = 0, rank: int = 4,
                 n_out: int = 3, out_factor: float = 20.0, device="cpu") -> torch.Tensor:
    """Structured random states [n, dk, dv] for codec tests.

    A low-rank part plus isotropic noise, with a few outlier rows and columns
    scaled by `out_factor` -- the shapes of recurrent states after a prefill,
    drawn directly without running any recurrence.
    """
    g = generator(seed, _STREAM_MATRIX, 0, device)
    f32 = torch.float32
    a = torch.randn((n, dk, rank), generator=g, device=device, dtype=f32)
    b = torch.randn((n, rank, dv), generator=g, device=device, dtype=f32)
    S = a @ b / rank + 0.3 * torch.randn((n, dk, dv), generator=g, device=device, dtype=f32)
    for i in range(n):
        rr = torch.randperm(dk, generator=g, device=device)[:n_out]
        cc = torch.randperm(dv, generator=g, device=device)[:n_out]
        S[i, rr, :] *= out_factor
        S[i, :, cc] *= out_factor
    return S.contiguous()


def expand_qk(x: torch.Tensor, H: int) -> torch.Tensor:
    """[..., Hk, d] -> [..., H, d] by the GQA map h -> floor(h*Hk/H)."""
    Hk = x.shape[-2]
    idx = (torch.arange(H, device=x.device) * Hk) // H
    return x.index_select(-2, idx)
