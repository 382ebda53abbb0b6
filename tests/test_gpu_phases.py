"""Staggered windows (per-entry window phases, lq_state_set_phases) on the GPU.

1. Against the oracle: teacher-forced windows with every batch entry on one
   phase p (first window W - p tokens), for GDN, KDA, the BF16 buffer, 4-bit
   codes and DAMP rows.
2. Batch independence: a batch of entries on mixed phases gives, bit for bit,
   what each entry gives alone on its phase -- the outputs of every token and
   the exported state -- across window ends, an explicit window flush (which
   restarts the schedule) and the window-end and buffering launches running
   side by side on two streams.
3. The launch configuration bench.py times (B = 1024, phases b mod W, window
   graphs replayed): sampled entries bit for bit against a small batch of the
   same entries and phases run step by step.
4. Argument and state errors.
"""
import numpy as np
import pytest
import torch

from quantized_recurrent_state_lq_b200 import configs, inputs as gen, lq, runner
from tests import gpu_util as U
from tests.test_gpu_decode import _rows_for, _teacher_forced, _workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("gate,B,H,Hk,dk,dv,W,r,phase,bf16,bits,P", [
    ("gdn", 2, 4, 2, 128, 128, 8, 4, 3, 0, 8, 0),
    ("kda", 2, 3, 3, 128, 128, 8, 4, 7, 0, 8, 0),     # a one-token first window
    ("kda", 2, 2, 2, 64, 128, 5, 2, 1, 0, 8, 0),
    ("gdn", 1, 2, 2, 64, 64, 16, 2, 5, 1, 8, 0),      # BF16 buffer
    ("gdn", 1, 2, 2, 128, 128, 6, 2, 2, 0, 4, 0),     # 4-bit codes
    ("gdn", 1, 2, 2, 128, 128, 8, 2, 4, 0, 8, 16),    # DAMP rows
])
def test_phased_teacher_forced(gate, B, H, Hk, dk, dv, W, r, phase, bf16, bits, P):
    U.require_gpu()
    wl = _workload(gate, B, H, Hk, dk, dv, W, r, seed=60 + W + phase, P=P, bf16=bf16, bits=bits)
    T = (W - phase) + 3 * W + W // 2
    _teacher_forced(wl, T, True, phase=phase,
                    label=f"phased p{phase} {gate} d{dk}x{dv} W{W} r{r} bf16{bf16} bits{bits} P{P}")


def _run_phased(wl, S0, tok, phases, rows, T, flush_at=None):
    cfg = lq.Config.from_workload(wl)
    st = lq.lq_state_init(cfg, S0.contiguous(), hp_rows=rows)
    lq.lq_state_set_phases(st, phases)
    out = torch.empty((T, wl.B, wl.H, wl.dv), device="cuda")
    for t in range(T):
        if flush_at is not None and t == flush_at:
            lq.lq_window_flush(st)
            assert lq.lq_state_buffered(st) == 0
        lq.lq_decode_step(st, *U.step_args(tok, t), out[t])
    S = torch.empty((wl.B, wl.H, wl.dk, wl.dv), device="cuda")
    lq.lq_state_export_fp32(st, S)
    torch.cuda.synchronize()
    assert lq.lq_get_status(st) == lq.LQ_OK
    return out, S, st


@pytest.mark.parametrize("flush_at", [None, 11])
@pytest.mark.parametrize("gate,B,H,Hk,dk,dv,W,r,bf16,bits,P", [
    ("gdn", 6, 3, 3, 128, 128, 8, 2, 0, 8, 0),
    ("kda", 5, 2, 1, 128, 64, 6, 2, 0, 8, 0),
    ("gdn", 5, 2, 2, 64, 64, 7, 2, 1, 8, 0),
    ("gdn", 4, 2, 2, 128, 128, 5, 2, 0, 4, 0),
    ("gdn", 4, 2, 2, 128, 128, 6, 2, 0, 8, 16),
])
def test_phased_batch_is_per_entry(gate, B, H, Hk, dk, dv, W, r, bf16, bits, P, flush_at):
    U.require_gpu()
    wl = _workload(gate, B, H, Hk, dk, dv, W, r, seed=70 + B, P=P, bf16=bf16, bits=bits)
    T = 3 * W + 3
    rows = _rows_for(wl)
    S0 = torch.from_numpy(U.prefill_state(wl, 32)).cuda()
    tok = gen.token_inputs(wl, T, device="cuda")
    phases = [(3 * b + 1) % W for b in range(B)]
    phases[0] = W - 1
    out, S, st = _run_phased(wl, S0, tok, phases, rows, T, flush_at)
    since = T - (flush_at or 0)
    want = max(min((since + p) % W, since) for p in phases)
    assert lq.lq_state_buffered(st) == want
    for b in range(B):
        w1 = wl.with_(B=1)
        tok1 = {k: v[:, b:b + 1].contiguous() for k, v in tok.items()}
        o1, S1, _ = _run_phased(w1, S0[b:b + 1], tok1, [phases[b]], rows, T, flush_at)
        assert torch.equal(out[:, b], o1[:, 0]), f"entry {b} (phase {phases[b]}): outputs differ"
        assert torch.equal(S[b], S1[0]), f"entry {b} (phase {phases[b]}): states differ"


def _random_states(wl, seed):
    """Low-rank plus noise states with the workload's outliers, drawn on the GPU."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    S = torch.empty((wl.B, wl.H, wl.dk, wl.dv), device="cuda")
    for i in range(0, wl.B, 64):
        j = min(wl.B, i + 64)
        a = torch.randn((j - i, wl.H, wl.dk, 4), generator=g, device="cuda")
        c = torch.randn((j - i, wl.H, 4, wl.dv), generator=g, device="cuda")
        S[i:j] = a @ c / 4 + 0.3 * torch.randn((j - i, wl.H, wl.dk, wl.dv), generator=g, device="cuda")
    return gen.apply_outliers(S, wl)


def test_full_size_phased_graphs_match_small_batch():
    U.require_gpu()
    wl = configs.GDN_PREFIX_CACHE
    W = wl.W
    phases = [b % W for b in range(wl.B)]
    S0 = _random_states(wl, 11)
    r = runner.WindowRunner(wl, S0, tokens=2 * W, phases=phases)
    r.capture()        # window 0 eagerly (every entry's first window), graphs of windows 0 and 1
    r.replay(0)
    r.replay(1)
    S = torch.empty_like(S0)
    lq.lq_state_export_fp32(r.st, S)
    torch.cuda.synchronize()
    assert lq.lq_get_status(r.st) == lq.LQ_OK
    sel = [0, 1, 62, 63, 64, 517, 960, wl.B - 1]
    ws = wl.with_(B=len(sel))
    cfg = lq.Config.from_workload(ws)
    st = lq.lq_state_init(cfg, S0[sel].contiguous())
    lq.lq_state_set_phases(st, [phases[b] for b in sel])
    o = torch.empty((ws.B, ws.H, ws.dv), device="cuda")
    tok = {k: v[:, sel].contiguous() for k, v in r.tok.items()}
    # the same token sequence: window 0 (warm-up), window 0 again, window 1
    for w, src in enumerate([0, 0, 1]):
        for t in range(W):
            lq.lq_decode_step(st, *U.step_args(tok, src * W + t), o)
            if w > 0:
                got = r.out[src * W + t][sel]
                assert torch.equal(got, o), f"window {w} token {t}: outputs differ"
    S1 = torch.empty((ws.B, ws.H, ws.dk, ws.dv), device="cuda")
    lq.lq_state_export_fp32(st, S1)
    torch.cuda.synchronize()
    assert torch.equal(S[sel], S1)
    assert lq.lq_get_status(st) == lq.LQ_OK


def test_phase_errors():
    U.require_gpu()
    wl = _workload("gdn", 2, 2, 2, 64, 64, 4, 1, seed=5)
    S0 = torch.from_numpy(U.prefill_state(wl, 16)).cuda()
    tok = gen.token_inputs(wl, 4, device="cuda")
    o = torch.empty((wl.B, wl.H, wl.dv), device="cuda")
    st = lq.lq_state_init(lq.Config.from_workload(wl), S0)
    for bad in ([0, 4], [-1, 0]):
        with pytest.raises(lq.LqError) as ei:
            lq.lq_state_set_phases(st, bad)
        assert ei.value.code == lq.LQ_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        lq.lq_state_set_phases(st, [0])
    lq.lq_state_set_phases(st, [1, 2])
    lq.lq_decode_step(st, *U.step_args(tok, 0), o)      # entry 1's first window is 2 tokens
    assert lq.lq_state_buffered(st) == 1
    with pytest.raises(lq.LqError) as ei:
        lq.lq_state_set_phases(st, [0, 0])               # not at a common window start
    assert ei.value.code == lq.LQ_ERR_UNSUPPORTED
    cfg = lq.Config.from_workload(wl)
    view = lq.alloc_view(cfg)
    for fn in (lq.lq_state_export_view, lq.lq_state_import_view):
        with pytest.raises(lq.LqError) as ei:
            fn(st, view)
        assert ei.value.code == lq.LQ_ERR_UNSUPPORTED
    lq.lq_decode_step(st, *U.step_args(tok, 1), o)      # entry 1's window ends
    assert lq.lq_state_buffered(st) == 2                 # entry 0: tokens 0 and 1
    lq.lq_window_flush(st)
    assert lq.lq_state_buffered(st) == 0
    lq.lq_state_export_view(st, view)
    lq.lq_state_set_phases(st, None)
    for kw in (dict(fused_flush=0), dict(mode="step")):
        st2 = lq.lq_state_init(lq.Config.from_workload(wl, **kw), S0)
        with pytest.raises(lq.LqError) as ei:
            lq.lq_state_set_phases(st2, [0, 0])
        assert ei.value.code == lq.LQ_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert lq.lq_get_status(st) == lq.LQ_OK
