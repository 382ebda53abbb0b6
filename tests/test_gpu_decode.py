"""GPU decode parity through the C ABI against the oracle on the same seeded
inputs: FP32-state mode, windowed INT8 (teacher-forced per window: each window
starts from the oracle's window-start view, imported into the GPU state),
per-step INT8, naive INT8, DAMP rows, partial windows and error paths."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_recurrent_state_lq_b200 import configs, inputs as gen, lq
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

OUT_REL = 1e-3     # outputs: max relative error per output vector (b, h, t)
STATE_REL = 1e-3   # FP32 state: max relative error per head


def _workload(gate, B, H, Hk, dk, dv, W, r, seed, P=0, bf16=0, bits=8):
    return configs.TINY_GDN.with_(gate=gate, B=B, H=H, Hk=Hk, dk=dk, dv=dv, W=W, r=r, seed=seed, P=P,
                                  n_out_rows=3, n_out_cols=3, out_lo=10.0, out_hi=50.0, buffer_bf16=bf16,
                                  bits=bits)


def _rows_for(wl):
    if not wl.P:
        return None
    g = torch.Generator().manual_seed(wl.seed + 77)
    return torch.stack([torch.sort(torch.randperm(wl.dk, generator=g)[:wl.P]).values
                        for _ in range(wl.H)]).int().numpy()


@pytest.mark.parametrize("gate,B,H,Hk,dk,dv", [("gdn", 2, 4, 2, 128, 128), ("kda", 1, 3, 3, 64, 128),
                                               ("gdn", 1, 2, 2, 64, 64), ("kda", 2, 2, 1, 128, 64)])
def test_fp32_mode_matches_oracle(gate, B, H, Hk, dk, dv):
    U.require_gpu()
    wl = _workload(gate, B, H, Hk, dk, dv, 8, 0, seed=21)
    T = 96
    S0 = U.prefill_state(wl, 64)
    tok = gen.token_inputs(wl, T, device="cuda")
    cfg = lq.Config.from_workload(wl, mode="fp32")
    st = lq.lq_state_init(cfg, torch.from_numpy(S0).cuda())
    outs = torch.empty((T, B, H, dv), device="cuda")
    for t in range(T):
        lq.lq_decode_step(st, *U.step_args(tok, t), outs[t])
    S = torch.empty((B, H, dk, dv), device="cuda")
    lq.lq_state_export_fp32(st, S)
    assert lq.lq_get_status(st) == lq.LQ_OK
    ref = O.run(U.ocfg(cfg, quantize=0), O.per_head_inputs(tok, H), S0=S0.reshape(-1, dk, dv))
    got = outs.cpu().numpy().reshape(T, B * H, dv)
    err = U.rel_inf_rows(got, ref["o"])
    print(f"fp32 mode {gate} d{dk}x{dv}: max out rel err {err.max():.2e}")
    assert err.max() < OUT_REL
    serr = U.rel_inf_rows(S.cpu().numpy().reshape(B * H, -1), ref["S"].reshape(B * H, -1))
    assert serr.max() < STATE_REL


def _teacher_forced(wl, T, fused, mode="window", smoothing=1, label="", static=None, alpha=None, phase=0):
    flip_frac = U.LONG_ACCUMULATION_FLIP_FRAC if wl.W >= 200 else U.FLUSH_FLIP_FRAC
    """Run T tokens window by window; each window starts from the oracle's view.
    static = (m [H, dk], s [H, dv]) numpy arrays: fixed scales (smoothing 2).
    alpha(tok): replaces the generator's decays (a device tensor of their shape).
    phase: every batch entry's window phase (staggered windows, one phase for
    all so that the windows still start together): the first window holds
    W - phase tokens."""
    if static is not None:
        smoothing = 2
    cfg = lq.Config.from_workload(wl, mode=mode, fused_flush=int(fused), smoothing=smoothing)
    if mode == "step":
        cfg.W = 1
    rows = _rows_for(wl)
    hr = U.head_rows(cfg, rows)
    nh = wl.B * wl.H
    S0 = U.prefill_state(wl, 64)
    tok = gen.token_inputs(wl, T, device="cuda")
    if alpha is not None:
        tok["alpha"] = alpha(tok).contiguous()
    ph = O.per_head_inputs(tok, wl.H)
    oc = U.ocfg(cfg)
    if static is None:
        st = lq.lq_state_init(cfg, torch.from_numpy(S0).cuda(), hp_rows=rows)
        head_cfg = lambda h: oc
    else:
        sm, ss = (np.ascontiguousarray(x, np.float32) for x in static)
        st = lq.lq_state_init(cfg, torch.from_numpy(S0).cuda(), static_m=torch.from_numpy(sm).cuda(),
                              static_s=torch.from_numpy(ss).cuda())
        oc.static_m = np.tile(sm, (wl.B, 1))        # per oracle head (b, h)
        oc.static_s = np.tile(ss, (wl.B, 1))
        head_cfg = lambda h: dataclasses.replace(oc, static_m=oc.static_m[h], static_s=oc.static_s[h])
    # window-start view of the oracle
    ov = O.empty_views(oc, nh)
    for h in range(nh):
        q = O.quantize(head_cfg(h), S0.reshape(nh, wl.dk, wl.dv)[h], hp_rows=None if hr is None else hr[h])
        for k in ov:
            ov[k][h][...] = np.asarray(q[k]).reshape(ov[k][h].shape)
    W = cfg.W
    if phase:
        lq.lq_state_set_phases(st, [phase] * wl.B)
    stats = {"out": 0.0, "state": 0.0, "flips": 0, "codes": 0, "band_used": 0.0, "bound_used": 0.0,
             "flips_bf16_tie": 0, "undetermined": 0}
    o = torch.empty((wl.B, wl.H, wl.dv), device="cuda")
    t0 = 0
    while t0 < T:
        Lw = W - phase if t0 == 0 else W   # this window's length
        flips0 = stats["flips"]
        n = min(Lw, T - t0)
        sl = {k: v[t0:t0 + n] for k, v in ph.items()}
        ref = O.run(oc, sl, view=ov, hp_rows=hr, flush_last=(n == Lw),   # oc: all heads' fixed scales
                    phase=[phase] * nh if t0 == 0 else None)
        lq.lq_state_import_view(st, U.oracle_view_to_gpu(cfg, ov, rows))
        S_g = None
        for t in range(n):
            last = t == n - 1
            if last and n == Lw and not fused and mode == "window":
                lq.lq_decode_step(st, *U.step_args(tok, t0 + t), o)
                S = torch.empty((wl.B, wl.H, wl.dk, wl.dv), device="cuda")
                lq.lq_state_export_fp32(st, S)
                S_g = S.cpu().numpy().reshape(nh, wl.dk, wl.dv).astype(np.float64)
                e = U.rel_inf_rows(S_g.reshape(nh, -1), ref["S_pre"].reshape(nh, -1))
                stats["state"] = max(stats["state"], float(e.max()))
                lq.lq_window_flush(st)
            else:
                lq.lq_decode_step(st, *U.step_args(tok, t0 + t), o)
            e = U.rel_inf_rows(o.cpu().numpy().reshape(nh, wl.dv), ref["o"][t])
            stats["out"] = max(stats["out"], float(e.max()))
        assert lq.lq_state_buffered(st) == (0 if n == Lw else n)
        if n == Lw:
            gv = lq.alloc_view(cfg)
            lq.lq_state_export_view(st, gv)
            got = U.gpu_view_to_oracle(cfg, gv, rows)
            ratio = U.oracle_ratios(cfg, ref["S_pre"].astype(np.float32), hr, head_cfg=head_cfg)
            for h in range(nh):
                hrh = None if hr is None else hr[h]
                # the GPU's pre-flush FP32 state: measured (separate flush) or
                # bounded from the arithmetic that forms it (flush fused into
                # the W-th step); the measured difference must obey the bound
                bound, risk = U.window_state_bound(head_cfg(h), U.head_view(ov, h),
                                                   {k: v[:, h] for k, v in sl.items()}, hp_rows=hrh, risk_cols=True)
                if S_g is not None:
                    dS = np.abs(S_g[h] - ref["S_pre"][h])
                    used = float((dS / bound).max())
                    assert used <= 1.0, f"{label}: head {h}: pre-flush state error above its bound ({used:.2f})"
                    stats["bound_used"] = max(stats["bound_used"], used)
                else:
                    dS = bound
                c = U.check_quantized(head_cfg(h), U.head_view(got, h), U.head_view(ref["view"], h), ratio[h],
                                      ref["S_pre"][h], dS, hp_rows=hrh, label=f"{label} window {t0 // W} head {h}",
                                      risk_cols=risk)
                if risk.any():
                    # a buffered u at a BF16 rounding tie moves its column of
                    # the state by a BF16 step, and through the compensators
                    # every column: the window's flips are that tie's
                    c = dict(c, n=0, n_risk=c["n"] + c["n_risk"])
                stats["flips"] += c["n"]
                stats["flips_bf16_tie"] += c["n_risk"]
                stats["undetermined"] += c["n_undetermined"]
                stats["codes"] += c["total"]
                stats["band_used"] = max(stats["band_used"], c["band_used"])
            U.assert_flush_params(cfg, got, ref["view"], ref["S_pre"], hr, label, rel=STATE_REL)
            scale = np.abs(ref["S_pre"]).max(axis=(1, 2))
            for j in range(cfg.r):
                pg = np.einsum("hi,hc->hic", got["c"][:, j], got["w"][:, j])
                pw = np.einsum("hi,hc->hic", ref["view"]["c"][:, j], ref["view"]["w"][:, j])
                assert (np.abs(pg - pw).max(axis=(1, 2)) <= STATE_REL * scale).all()
            if cfg.n_hp_rows:
                # BF16 rows enter the window-start state check above; per
                # element: one bf16 ulp (a rounding tie), or -- for elements
                # far below the head's largest -- within the state bar of it
                hpg = got["hp"][:, :cfg.n_hp_rows]
                hpw = ref["view"]["hp"][:, :cfg.n_hp_rows]
                ulps = np.abs(hpg.view(np.int16).astype(np.int32) - hpw.view(np.int16).astype(np.int32))
                f = lambda x: (x.astype(np.uint32) << 16).view(np.float32)
                dv = np.abs(f(hpg) - f(hpw))
                assert ((ulps <= 1) | (dv <= STATE_REL * scale[:, None, None])).all()
        if n == Lw:
            print(f"{label}: window at token {t0} ({n} tokens): {stats['flips'] - flips0} flips")
        ov = ref["view"]
        t0 += n
    assert lq.lq_get_status(st) == lq.LQ_OK
    print(f"{label}: out {stats['out']:.2e} state {stats['state']:.2e} (bound used {stats['bound_used']:.2f}) "
          f"flips {stats['flips']}/{stats['codes']} (band used {stats['band_used']:.2f}; "
          f"{stats['flips_bf16_tie']} in BF16-tie columns, {stats['undetermined']} undetermined)")
    assert stats["out"] < OUT_REL
    assert stats["state"] < STATE_REL
    U.assert_code_bar({"n": stats["flips"], "total": stats["codes"]}, label, flip_frac)
    return stats


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("gate,B,H,Hk,dk,dv,W,r", [
    ("gdn", 1, 2, 2, 64, 64, 16, 2),        # the tiny workload's shape
    ("gdn", 2, 4, 2, 128, 128, 8, 4),       # GQA, d = 128
    ("kda", 2, 3, 3, 128, 128, 8, 4),
    ("kda", 1, 3, 3, 64, 128, 5, 2),        # dk != dv, odd window
    ("gdn", 2, 2, 2, 128, 64, 6, 3),
    ("gdn", 1, 2, 2, 128, 128, 64, 4),      # 85 KB staged: above the 48 KB default
    ("kda", 1, 2, 2, 128, 128, 200, 4),     # 26 entry chunks per flush, a ragged last one
])
def test_windowed_teacher_forced(fused, gate, B, H, Hk, dk, dv, W, r):
    U.require_gpu()
    wl = _workload(gate, B, H, Hk, dk, dv, W, r, seed=31 + W)
    T = 3 * W + W // 2   # three windows and a ragged tail
    _teacher_forced(wl, T, fused, label=f"window {gate} d{dk}x{dv} W{W} r{r} fused{int(fused)}")


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("gate,H,W,bf16,mu", [
    ("kda", 2, 512, 0, -1.0),     # strong channels: Gamma passes 2^-64 every ~110 tokens
    ("kda", 2, 4096, 0, -1.0),    # the longest window: 2^-1900 by its end
    ("kda", 2, 320, 1, -1.0),     # BF16 buffer: keys rounded against the guarded chain
    ("gdn", 2, 4096, 0, None),    # the benchmark's GDN decays: Gamma ~2^-180 by the end
    ("gdn", 2, 320, 1, -1.0),     # BF16 buffer, whole-entry loads: re-based every ~140 tokens
])
def test_long_windows_strong_decays(fused, gate, H, W, bf16, mu):
    """Decay products far below the FP32 range within a window (the decay
    guard of the buffering and flush kernels): outputs and the flushed state
    against the oracle, which decays its double state directly."""
    U.require_gpu()
    wl = _workload(gate, 1, H, H, 128, 128, W, 4, seed=81 + W + bf16, bf16=bf16)
    T = W + 3
    dec = None if mu is None else (lambda tok: gen.strong_decays(tok["alpha"].shape, mu, 7, device="cuda"))
    st = _teacher_forced(wl, T, fused, alpha=dec,
                         label=f"long window {gate} W{W} bf16{bf16} fused{int(fused)}")
    assert st["out"] < OUT_REL


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("gate,bf16", [("gdn", 0), ("kda", 0), ("kda", 1), ("gdn", 1)])
def test_vanishing_decays(fused, gate, bf16):
    """Decays of 1e-30 and exactly 0 inside a window: the channel (or head)
    restarts, nothing overflows, outputs and flushes match the oracle."""
    U.require_gpu()
    wl = _workload(gate, 2, 2, 2, 128, 128, 16, 4, seed=91 + bf16, bf16=bf16)
    _teacher_forced(wl, 2 * 16 + 5, fused, alpha=lambda tok: gen.with_vanishing_decays(tok["alpha"], 5),
                    label=f"vanishing decays {gate} bf16{bf16} fused{int(fused)}")


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("gate,B,H,Hk,dk,dv,W,r", [
    ("gdn", 2, 2, 2, 128, 128, 64, 4),      # the benchmark's shape: one-pass tensor-core chunks
    ("kda", 2, 3, 3, 128, 128, 32, 4),
    ("gdn", 1, 2, 2, 64, 64, 16, 2),        # d = 64: the tile reads the BF16 entries directly
    ("kda", 1, 3, 3, 128, 64, 5, 3),
])
def test_windowed_bf16_buffer_teacher_forced(fused, gate, B, H, Hk, dk, dv, W, r):
    """The traffic-lean buffer: tokens' updates kept as bf16(k/Gamma), bf16(u);
    the oracle's BF16-buffer mode takes the same rounding decisions in FP32."""
    U.require_gpu()
    wl = _workload(gate, B, H, Hk, dk, dv, W, r, seed=61 + W, bf16=1)
    T = 2 * W + W // 2 + 1
    _teacher_forced(wl, T, fused, label=f"bf16 buffer {gate} d{dk}x{dv} W{W} r{r} fused{int(fused)}")


@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("gate,B,H,Hk,dk,dv,W,r,bf16", [
    ("gdn", 2, 4, 2, 128, 128, 8, 4, 0),    # GQA, d = 128: two packed k-pairs per column
    ("kda", 2, 3, 3, 128, 128, 32, 4, 0),
    ("gdn", 1, 2, 2, 64, 64, 16, 2, 0),     # d = 64: one k-pair, a single pair-plane chunk
    ("kda", 1, 3, 3, 64, 128, 5, 2, 0),     # odd window
    ("gdn", 2, 2, 2, 128, 64, 6, 3, 0),
    ("gdn", 2, 2, 2, 128, 128, 16, 4, 1),   # with the BF16 window buffer
])
def test_windowed_low_bit_teacher_forced(bits, fused, gate, B, H, Hk, dk, dv, W, r, bf16):
    """6- and 4-bit states (codes in +-31 / +-7, bit-packed in the workspace):
    the same teacher-forced bars as INT8 -- outputs and pre-flush state within
    1e-3 of the oracle's low-bit mode, codes exact but for rounding ties."""
    U.require_gpu()
    wl = _workload(gate, B, H, Hk, dk, dv, W, r, seed=71 + W + bits, bf16=bf16, bits=bits)
    T = 2 * W + W // 2 + 1
    _teacher_forced(wl, T, fused, label=f"{bits}-bit {gate} d{dk}x{dv} W{W} r{r} bf16{bf16} fused{int(fused)}")


@pytest.mark.parametrize("bits", [4, 6])
def test_per_step_low_bit_mode(bits):
    U.require_gpu()
    wl = _workload("gdn", 2, 2, 2, 128, 128, 1, 4, seed=45 + bits, bits=bits)
    _teacher_forced(wl, 10, True, mode="step", label=f"per-step {bits}-bit")


def test_damp_rows_teacher_forced():
    U.require_gpu()
    wl = _workload("gdn", 2, 3, 3, 128, 128, 8, 2, seed=41, P=16)
    _teacher_forced(wl, 2 * 8 + 3, True, label="damp P16")


def test_per_step_int8_mode():
    U.require_gpu()
    wl = _workload("kda", 1, 3, 3, 128, 128, 1, 4, seed=43)
    _teacher_forced(wl, 12, True, mode="step", label="per-step int8")


def test_naive_int8_mode():
    U.require_gpu()
    wl = _workload("gdn", 2, 2, 2, 128, 128, 1, 0, seed=44)
    _teacher_forced(wl, 12, True, mode="step", smoothing=0, label="naive int8")


def test_free_running_tiny_workload():
    """The tiny GDN workload end to end (no teacher forcing): the GPU and the
    oracle each run the whole decode from the same initial state."""
    U.require_gpu()
    wl = configs.TINY_GDN
    S0 = U.prefill_state(wl, wl.prefill)
    tok = gen.token_inputs(wl, wl.T, device="cuda")
    cfg = lq.Config.from_workload(wl)
    st = lq.lq_state_init(cfg, torch.from_numpy(S0).cuda())
    outs = torch.empty((wl.T, wl.B, wl.H, wl.dv), device="cuda")
    for t in range(wl.T):
        lq.lq_decode_step(st, *U.step_args(tok, t), outs[t])
    ref = O.run(U.ocfg(cfg), O.per_head_inputs(tok, wl.H), S0=S0.reshape(-1, wl.dk, wl.dv))
    fp = O.run(U.ocfg(cfg, quantize=0), O.per_head_inputs(tok, wl.H), S0=S0.reshape(-1, wl.dk, wl.dv))
    got = outs.cpu().numpy().reshape(wl.T, -1, wl.dv)
    err = U.rel_inf_rows(got, ref["o"])
    q_err = U.rel_inf_rows(ref["o"], fp["o"])
    g_err = U.rel_inf_rows(got, fp["o"])
    print(f"free-running tiny: GPU vs oracle max {err.max():.2e} mean {err.mean():.2e}; "
          f"vs FP recurrence: GPU mean {g_err.mean():.2e}, oracle mean {q_err.mean():.2e}")
    # A code flip at a rounding tie is a valid alternative result that then
    # propagates, so the two runs drift apart; both must still be equally close
    # to the unquantized recurrence (the method's own error).
    assert g_err.mean() <= 1.25 * q_err.mean()
    assert g_err.max() <= 2.0 * q_err.max()
    assert lq.lq_get_status(st) == lq.LQ_OK


def _check_flush_vs_oracle(cfg, st, S_g, ref, ov_start, toks, label):
    """The GPU state's view after a flush against the oracle's (`ref` from
    O.run with flush_last), with the GPU's exported pre-flush state S_g [nh,
    dk, dv]: the state within its derived bound, then the codes, scales and
    compensators by check_quantized and the window-start state bar."""
    oc = U.ocfg(cfg)
    nh = cfg.B * cfg.H
    gv = lq.alloc_view(cfg)
    lq.lq_state_export_view(st, gv)
    got = U.gpu_view_to_oracle(cfg, gv, None)
    ratio = U.oracle_ratios(cfg, ref["S_pre"].astype(np.float32), None)
    flips = total = 0
    for h in range(nh):
        bound = U.window_state_bound(oc, U.head_view(ov_start, h), {k: v[:, h] for k, v in toks.items()})
        dS = np.abs(S_g[h] - ref["S_pre"][h])
        assert (dS <= bound).all(), f"{label}: pre-flush state above its bound"
        c = U.check_quantized(oc, U.head_view(got, h), U.head_view(ref["view"], h), ratio[h], ref["S_pre"][h], dS,
                              label=f"{label} head {h}")
        flips += c["n"]
        total += c["total"]
    U.assert_code_bar({"n": flips, "total": total}, label)
    U.assert_flush_params(cfg, got, ref["view"], ref["S_pre"], None, label, rel=STATE_REL)


def test_partial_window_flush_and_window_full():
    """A full window, the call past it (refused), a flush; then two tokens and
    a flush of the partial window (teacher-forced: the second window starts
    from the oracle's view).  Each flush is held to the per-window bars."""
    U.require_gpu()
    wl = _workload("gdn", 1, 2, 2, 128, 128, 4, 2, seed=50)
    cfg = lq.Config.from_workload(wl, fused_flush=0)
    S0 = torch.from_numpy(U.prefill_state(wl, 32)).cuda()
    tok = gen.token_inputs(wl, 8, device="cuda")
    oc = U.ocfg(cfg)
    ph = O.per_head_inputs(tok, 2)
    ov0 = O.empty_views(oc, 2)
    for h in range(2):
        q = O.quantize(oc, S0.cpu().numpy().reshape(2, 128, 128)[h])
        for k in ov0:
            ov0[k][h][...] = np.asarray(q[k]).reshape(ov0[k][h].shape)
    st = lq.lq_state_init(cfg, S0)
    lq.lq_state_import_view(st, U.oracle_view_to_gpu(cfg, ov0, None))
    o = torch.empty((1, 2, 128), device="cuda")
    for t in range(4):
        lq.lq_decode_step(st, *U.step_args(tok, t), o)
    with pytest.raises(lq.LqError) as ei:
        lq.lq_decode_step(st, *U.step_args(tok, 4), o)
    assert ei.value.code == lq.LQ_ERR_WINDOW_FULL
    Sg = torch.empty_like(S0)
    lq.lq_state_export_fp32(st, Sg)
    lq.lq_window_flush(st)
    assert lq.lq_state_buffered(st) == 0
    w1 = {k: v[:4] for k, v in ph.items()}
    a = O.run(oc, w1, view=ov0, flush_last=True)
    _check_flush_vs_oracle(cfg, st, Sg.cpu().numpy().reshape(2, 128, 128).astype(np.float64), a, ov0, w1,
                           "full window")
    # the second window starts from the oracle's view; two tokens, then a flush
    lq.lq_state_import_view(st, U.oracle_view_to_gpu(cfg, a["view"], None))
    lq.lq_decode_step(st, *U.step_args(tok, 4), o)
    lq.lq_decode_step(st, *U.step_args(tok, 5), o)
    assert lq.lq_state_buffered(st) == 2
    lq.lq_state_export_fp32(st, Sg)
    lq.lq_window_flush(st)
    w2 = {k: v[4:6] for k, v in ph.items()}
    b = O.run(O.Cfg(**{**oc.__dict__, "W": 2}), w2, view=a["view"], flush_last=True)
    _check_flush_vs_oracle(cfg, st, Sg.cpu().numpy().reshape(2, 128, 128).astype(np.float64), b, a["view"], w2,
                           "partial window")
    lq.lq_window_flush(st)   # nothing buffered: no-op
    assert lq.lq_state_buffered(st) == 0
    assert lq.lq_get_status(st) == lq.LQ_OK


def test_nonfinite_inputs_raise_status():
    U.require_gpu()
    wl = _workload("gdn", 1, 2, 2, 64, 64, 4, 1, seed=60)
    cfg = lq.Config.from_workload(wl)
    S0 = torch.from_numpy(U.prefill_state(wl, 16)).cuda()
    st = lq.lq_state_init(cfg, S0)
    tok = gen.token_inputs(wl, 2, device="cuda")
    v = tok["v"][0].clone()
    v[0, 1, 3] = float("nan")
    o = torch.empty((1, 2, 64), device="cuda")
    lq.lq_decode_step(st, tok["q"][0], tok["k"][0], v, tok["beta"][0], tok["alpha"][0], o)
    assert lq.lq_get_status(st) == lq.LQ_ERR_NONFINITE
