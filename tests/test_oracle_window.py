"""Pins of the oracle's windowed decode (LeapQuant project page, window and
Compensator Tokens paragraphs) against the brute force and closed forms."""
import numpy as np
import pytest
import torch

from quantized_recurrent_state_lq_b200 import configs, inputs as gen
from tests import brute

f32 = np.float32


def tiny_tokens(seed, T, dk, dv, gate, nh=1):
    wl = configs.TINY_GDN.with_(dk=dk, dv=dv, gate=gate, B=1, H=nh, Hk=nh, seed=seed)
    tok = gen.token_inputs(wl, T)
    return {"q": tok["q"][:, 0].numpy(), "k": tok["k"][:, 0].numpy(), "v": tok["v"][:, 0].numpy(),
            "beta": tok["beta"][:, 0].numpy(), "alpha": tok["alpha"][:, 0].numpy()}


def tok_list(tok, h):
    T = tok["q"].shape[0]
    return [(tok["q"][t, h], tok["k"][t, h], tok["v"][t, h], float(tok["beta"][t, h]),
             np.atleast_1d(tok["alpha"][t, h])) for t in range(T)]


@pytest.mark.parametrize("gate", ["gdn", "kda"])
def test_identity_quantizer_is_plain_recurrence(orc, gate):
    dk, dv, T = 6, 5, 40
    tok = tiny_tokens(1, T, dk, dv, gate, nh=2)
    S0 = gen.random_state(2, dk, dv, seed=1).numpy()
    cfg = orc.Cfg(dk=dk, dv=dv, gate=gate, quantize=0, W=4)
    res = orc.run(cfg, tok, S0=S0)
    for h in range(2):
        outs, _ = brute.run_windowed(S0[h], tok_list(tok, h), W=4, r=0, K=0, gate=gate, quantize_on=False)
        np.testing.assert_allclose(res["o"][:, h], outs, rtol=1e-10, atol=1e-10)


def _codes_match(a, b, ratio):
    near_tie = np.abs(np.abs(ratio - np.trunc(ratio)) - 0.5) < 1e-3
    return np.all((a == b) | near_tie)


@pytest.mark.parametrize("gate", ["gdn", "kda"])
@pytest.mark.parametrize("W,r", [(4, 1), (1, 1), (3, 0)])
def test_brute_force_windowed_d4(orc, gate, W, r):
    """Everything at once on d = 4, T = 16: windows, compensators, smoothing."""
    dk = dv = 4
    T = 16
    tok = tiny_tokens(3 + W + r, T, dk, dv, gate, nh=1)
    S0 = (gen.random_state(1, dk, dv, seed=2, n_out=1, out_factor=5.0).numpy())
    cfg = orc.Cfg(dk=dk, dv=dv, gate=gate, W=W, r=r, K=8)
    res = orc.run(cfg, tok, S0=S0, flush_last=True)
    outs, view = brute.run_windowed(S0[0], tok_list(tok, 0), W=W, r=r, K=8, gate=gate)
    np.testing.assert_allclose(res["o"][:, 0], outs, rtol=1e-5, atol=1e-5 * np.abs(outs).max())
    ov = {k: res["view"][k][0] for k in ("codes", "m", "s", "c", "w")}
    np.testing.assert_allclose(ov["m"], view["m"], rtol=1e-5)
    np.testing.assert_allclose(ov["s"], view["s"], rtol=1e-5)
    # recompute the oracle's ratios for the tie-aware code comparison
    Sf = res["S_pre"][0].astype(f32)
    rq = orc.quantize(cfg, Sf, want_ratio=True)
    assert _codes_match(ov["codes"], view["codes"], rq["ratio"])


def test_window_one_is_per_step_requantization(orc):
    """W = 1: quantize after every token, which the brute force does literally."""
    dk = dv = 8
    tok = tiny_tokens(9, 12, dk, dv, "gdn")
    S0 = gen.random_state(1, dk, dv, seed=3).numpy()
    cfg = orc.Cfg(dk=dk, dv=dv, W=1, r=2, K=8)
    res = orc.run(cfg, tok, S0=S0)
    outs, _ = brute.run_windowed(S0[0], tok_list(tok, 0), W=1, r=2, K=8, gate="gdn")
    np.testing.assert_allclose(res["o"][:, 0], outs, rtol=1e-5, atol=1e-5 * np.abs(outs).max())


def test_window_longer_than_run_is_fp_from_dequantized_start(orc):
    dk, dv, T = 8, 8, 20
    tok = tiny_tokens(10, T, dk, dv, "kda")
    S0 = gen.random_state(1, dk, dv, seed=4).numpy()
    cfg = orc.Cfg(dk=dk, dv=dv, gate="kda", W=64, r=2, K=8)
    res = orc.run(cfg, tok, S0=S0)
    start = orc.dequantize(cfg, orc.quantize(cfg, S0[0]))
    Sp = start.T.copy()
    for t, (q, k, v, beta, alpha) in enumerate(tok_list(tok, 0)):
        Sp, o = brute.step_pages_form(Sp, q, k, v, beta, alpha, "kda")
        np.testing.assert_allclose(res["o"][t, 0], o, rtol=1e-11, atol=1e-11)
    assert res["n"][0] == T


def test_window_split_equals_continuous_run(orc):
    """Running two windows at once equals window 1 (flushed) then window 2 from its view."""
    dk = dv = 16
    W = 8
    tok = tiny_tokens(12, 2 * W, dk, dv, "gdn", nh=2)
    S0 = gen.random_state(2, dk, dv, seed=5).numpy()
    cfg = orc.Cfg(dk=dk, dv=dv, W=W, r=2, K=8)
    full = orc.run(cfg, tok, S0=S0, flush_last=True)
    first = orc.run(cfg, {k: v[:W] for k, v in tok.items()}, S0=S0, flush_last=True)
    second = orc.run(cfg, {k: v[W:] for k, v in tok.items()}, view=first["view"], flush_last=True)
    np.testing.assert_array_equal(full["o"][:W], first["o"])
    np.testing.assert_array_equal(full["o"][W:], second["o"])
    for k in ("codes", "m", "s", "c", "w"):
        np.testing.assert_array_equal(full["view"][k], second["view"][k])
    np.testing.assert_array_equal(full["S_pre"], second["S_pre"])


def test_no_flush_at_end_unless_asked(orc):
    dk = dv = 8
    W = 4
    tok = tiny_tokens(13, W, dk, dv, "gdn")
    S0 = gen.random_state(1, dk, dv, seed=6).numpy()
    cfg = orc.Cfg(dk=dk, dv=dv, W=W, r=1, K=8)
    a = orc.run(cfg, tok, S0=S0, flush_last=False)
    b = orc.run(cfg, tok, S0=S0, flush_last=True)
    assert a["n"][0] == W and b["n"][0] == 0
    np.testing.assert_array_equal(a["S"], b["S_pre"])
    np.testing.assert_array_equal(a["o"], b["o"])


def _tiny_workload_errors(orc):
    wl = configs.TINY_GDN
    pre = gen.token_inputs(wl, wl.prefill, stream="prefill")
    cfg = orc.Cfg(dk=wl.dk, dv=wl.dv, gate=wl.gate, W=wl.W, r=wl.r, K=wl.K)
    S0 = orc.prefill(cfg, orc.per_head_inputs(pre, wl.H))
    S0 = gen.apply_outliers(torch.from_numpy(S0.astype(f32)).reshape(wl.B, wl.H, wl.dk, wl.dv), wl)
    S0 = S0.reshape(-1, wl.dk, wl.dv).numpy()
    dec = orc.per_head_inputs(gen.token_inputs(wl, wl.T), wl.H)
    ref = orc.run(orc.Cfg(dk=wl.dk, dv=wl.dv, quantize=0), dec, S0=S0)["o"]

    def err(c):
        o = orc.run(c, dec, S0=S0)["o"]
        return np.abs(o - ref).max(axis=-1).mean() / np.abs(ref).max(axis=-1).mean()

    return {"window": err(cfg),
            "step": err(orc.Cfg(dk=wl.dk, dv=wl.dv, W=1, r=wl.r, K=wl.K)),
            "naive": err(orc.Cfg(dk=wl.dk, dv=wl.dv, W=1, r=0, K=wl.K, smoothing=0))}


def test_windowing_reduces_error_vs_per_step(orc):
    """LeapQuant: quantizing once per window accumulates less error than every
    token; naive per-step INT8 (no compensators, no smoothing) is worst."""
    e = _tiny_workload_errors(orc)
    assert e["window"] < e["step"] < e["naive"], e
    assert e["window"] < 0.5 * e["step"], e


def test_per_head_inputs_gqa_map(orc):
    wl = configs.GDN_SERVING.with_(B=2, H=4, Hk=2, dk=8, dv=8)
    tok = gen.token_inputs(wl, 3)
    ph = orc.per_head_inputs(tok, wl.H)
    assert ph["q"].shape == (3, 8, 8)
    # value head h of batch b reads q/k head h*Hk//H
    for b in range(2):
        for h in range(4):
            np.testing.assert_array_equal(ph["q"][:, b * 4 + h], tok["q"][:, b, h // 2].numpy())
            np.testing.assert_array_equal(ph["v"][:, b * 4 + h], tok["v"][:, b, h].numpy())
