"""Pins of the oracle's static key-row / value-column scales (STEPQuant
article: scales fitted jointly offline; reading in lqo_fit_static's header).

* The static quantizer given the per-window scales of a state is the
  per-window quantizer on that state (codes, scales, compensators equal).
* With narrower static scales every code is the nearest level of the width's
  saturating range (exhaustive argmin over [-qmax, qmax]).
* The fit: equal to an independent loop-by-loop coordinate descent on d = 4
  (no compensators: the residual is the state); its objective never
  increases; it improves on its start on outlier-heavy states; scaling every
  row weight by 2 changes nothing; with compensators it matches the brute
  force on the oracle's own residuals.
"""
import numpy as np
import pytest

from quantized_recurrent_state_lq_b200 import inputs as gen
from tests import brute

f32 = np.float32
QMAX = {8: 127, 6: 31, 4: 7}


@pytest.mark.parametrize("bits", [8, 4])
def test_static_with_window_scales_is_the_window_quantizer(orc, bits):
    S = gen.random_state(3, 32, 24, seed=12).numpy()
    for h in range(3):
        dyn = orc.quantize(orc.Cfg(dk=32, dv=24, r=2, K=8, bits=bits), S[h])
        cfg = orc.Cfg(dk=32, dv=24, r=2, K=8, bits=bits, smoothing=2, static_m=dyn["m"], static_s=dyn["s"])
        st = orc.quantize(cfg, S[h])
        for key in ("codes", "m", "s", "c", "w"):
            np.testing.assert_array_equal(st[key], dyn[key])


@pytest.mark.parametrize("bits", [8, 4])
def test_static_narrow_scales_saturate_to_nearest_level(orc, bits):
    qm = QMAX[bits]
    S = gen.random_state(1, 16, 12, seed=3).numpy()[0]
    dyn = orc.quantize(orc.Cfg(dk=16, dv=12, r=0, K=8, smoothing=1, bits=bits), S)
    sm = dyn["m"]
    ss = (dyn["s"] * f32(0.4)).astype(f32)
    v = orc.quantize(orc.Cfg(dk=16, dv=12, r=0, K=8, bits=bits, smoothing=2, static_m=sm, static_s=ss), S,
                     want_ratio=True)
    x = (S.astype(f32) / sm[:, None]).astype(f32)
    want = brute.codes_exhaustive(x, ss, qm)
    near_tie = np.abs(np.abs(v["ratio"] - np.trunc(v["ratio"])) - 0.5) < 1e-4
    assert np.all((v["codes"] == want) | near_tie)
    assert np.abs(v["codes"]).max() == qm and (np.abs(v["codes"]) == qm).sum() > 10   # saturated


@pytest.mark.parametrize("bits", [8, 4])
def test_fit_equals_brute_force_d4(orc, bits):
    rng = np.random.default_rng(bits)
    states = (rng.standard_normal((3, 4, 4)) * rng.uniform(0.2, 5, (3, 4, 1))).astype(f32)
    states[0, 1, 2] *= 30.0     # an outlier the fit may clip
    w = rng.uniform(0.5, 2.0, 4)
    cfg = orc.Cfg(dk=4, dv=4, r=0, K=8, bits=bits)
    got = orc.fit_static(cfg, states, weight=w)
    m, s = brute.fit_static(states, w, QMAX[bits])
    np.testing.assert_array_equal(got["m"], m)
    np.testing.assert_array_equal(got["s"], s)


def test_fit_objective_never_increases_and_improves(orc):
    S = gen.random_state(6, 32, 32, seed=21, n_out=2, out_factor=30.0).numpy()
    for bits in (8, 4):
        cfg = orc.Cfg(dk=32, dv=32, r=2, K=8, bits=bits)
        res = orc.fit_static(cfg, S)
        obj = res["obj"]
        assert np.all(np.diff(obj) <= 0), obj
        assert obj[-1] < 0.999 * obj[0], obj
        # the objective the oracle reports is the one the scales give
        R = np.stack([S[t] - _comps(orc, cfg, S[t]) for t in range(S.shape[0])]).astype(f32)
        e = sum(brute._fit_err(R[t, i, c], res["m"][i], res["s"][c], QMAX[bits])
                for t in range(R.shape[0]) for i in range(32) for c in range(32))
        assert e == pytest.approx(obj[-1], rel=1e-9)


def _comps(orc, cfg, S):
    v = orc.quantize(orc.Cfg(dk=cfg.dk, dv=cfg.dv, r=cfg.r, K=cfg.K), S)
    return sum(np.outer(c.astype(np.float64), w.astype(np.float64)) for c, w in zip(v["c"], v["w"]))


def test_fit_row_weight_scale_invariant_and_used(orc):
    S = gen.random_state(4, 16, 16, seed=5, n_out=2, out_factor=20.0).numpy()
    cfg = orc.Cfg(dk=16, dv=16, r=1, K=8, bits=4)
    w = np.linspace(0.5, 3.0, 16)
    a = orc.fit_static(cfg, S, weight=w)
    b = orc.fit_static(cfg, S, weight=2.0 * w)
    np.testing.assert_array_equal(a["m"], b["m"])
    np.testing.assert_array_equal(a["s"], b["s"])
    # with compensators: the brute force on the oracle's residuals
    R = np.stack([S[t] - _comps(orc, cfg, S[t]) for t in range(S.shape[0])]).astype(f32)
    m, s = brute.fit_static(R, w, 7)
    np.testing.assert_array_equal(a["m"], m)
    np.testing.assert_array_equal(a["s"], s)


def test_fit_objective_function_matches_fit(orc):
    S = gen.random_state(4, 16, 16, seed=7, n_out=2, out_factor=20.0).numpy()
    cfg = orc.Cfg(dk=16, dv=16, r=1, K=8, bits=8)
    res = orc.fit_static(cfg, S)
    assert orc.fit_objective(cfg, S, res["m"], res["s"]) == pytest.approx(res["obj"][-1], rel=1e-12)
