"""Pins of the oracle's 6-bit and 4-bit states (the LeapQuant page's results
table has 8-, 6- and 4-bit rows: the same quantizer with a narrower code range,
qmax = 2^(b-1) - 1 = 31 and 7).

* A state on an exact b-bit grid (codes in [-qmax, qmax] with a full-scale
  code in every column, power-of-two column steps, no compensators or
  smoothing) quantizes to exactly those codes and scales and dequantizes back
  bit for bit -- a wrong qmax in the scale or in the clamp fails it.
* At d = 4 and 8 every code is the nearest of the 2 qmax + 1 levels (ties to
  even), from the independent brute force with its own qmax.
* Every column's largest |code| is qmax and no code leaves [-qmax, qmax].
* The dequantization error is within half a step m_i s_c / 2 per entry.
* bits = 0 and bits = 8 are the INT8 quantizer.
* The quantization error grows as the step does, about as 127 / qmax.
* Windowed decode at d = 4 with 4-bit and 6-bit states equals the brute-force
  windowed run with the same qmax.
"""
import numpy as np
import pytest

from quantized_recurrent_state_lq_b200 import inputs as gen
from tests import brute
from tests.test_oracle_window import _codes_match, tiny_tokens, tok_list

f32 = np.float32
QMAX = {8: 127, 6: 31, 4: 7}


def _residual(S, v):
    R = S.astype(np.float64)
    for c, w in zip(v["c"], v["w"]):
        R = R - np.outer(c.astype(np.float64), w.astype(np.float64))
    return R


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_exact_grid_round_trips(orc, bits):
    qm = QMAX[bits]
    rng = np.random.default_rng(40 + bits)
    dk, dv = 16, 12
    C = rng.integers(-qm, qm + 1, (dk, dv))
    rows = rng.integers(0, dk, dv)
    C[rows, np.arange(dv)] = rng.choice([-qm, qm], dv)     # a full-scale code per column
    step = np.ldexp(1.0, rng.integers(-8, 4, dv)).astype(f32)
    S = (C * step[None, :]).astype(f32)
    cfg = orc.Cfg(dk=dk, dv=dv, r=0, K=8, smoothing=0, bits=bits)
    v = orc.quantize(cfg, S)
    np.testing.assert_array_equal(v["codes"], C)
    np.testing.assert_array_equal(v["s"], step)
    np.testing.assert_array_equal(v["m"], np.ones(dk, f32))
    np.testing.assert_array_equal(orc.dequantize(cfg, v), S.astype(np.float64))


@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("d", [4, 8])
def test_codes_are_exhaustive_argmin(orc, bits, d):
    qm = QMAX[bits]
    rng = np.random.default_rng(7 * d + bits)
    for _ in range(10):
        S = (rng.standard_normal((d, d)) * rng.uniform(0.1, 10, (d, 1))).astype(f32)
        cfg = orc.Cfg(dk=d, dv=d, r=1, K=8, bits=bits)
        v = orc.quantize(cfg, S, want_ratio=True)
        b = brute.quantize(S, r=1, K=8, qmax=qm)
        np.testing.assert_allclose(v["s"], b["s"], rtol=2e-6)
        mine = brute.codes_exhaustive(b["x"], b["s"], qm)
        assert _codes_match(v["codes"], mine, v["ratio"])


@pytest.mark.parametrize("bits", [4, 6])
def test_full_scale_and_range(orc, bits):
    qm = QMAX[bits]
    S = gen.random_state(3, 32, 24, seed=11).numpy()
    cfg = orc.Cfg(dk=32, dv=24, r=2, K=8, bits=bits)
    for h in range(3):
        v = orc.quantize(cfg, S[h])
        assert np.all(np.abs(v["codes"]).max(axis=0) == qm)
        assert np.abs(v["codes"]).max() <= qm


@pytest.mark.parametrize("bits", [4, 6])
def test_error_within_half_step(orc, bits):
    S = gen.random_state(2, 16, 12, seed=5).numpy()
    cfg = orc.Cfg(dk=16, dv=12, r=2, K=8, bits=bits)
    eps = np.finfo(f32).eps
    for h in range(2):
        v = orc.quantize(cfg, S[h])
        R = _residual(S[h], v)
        deq = ((v["codes"].astype(f32) * v["s"]).astype(f32) * v["m"][:, None]).astype(np.float64)
        bound = v["m"][:, None].astype(np.float64) * v["s"][None, :] / 2 * (1 + 4 * eps)
        assert np.all(np.abs(R - deq) <= bound + 4 * eps * np.abs(R))


def test_bits_zero_and_eight_are_int8(orc):
    S = gen.random_state(1, 16, 16, seed=4).numpy()[0]
    base = orc.quantize(orc.Cfg(dk=16, dv=16, r=2, K=8), S)
    for bits in (0, 8):
        v = orc.quantize(orc.Cfg(dk=16, dv=16, r=2, K=8, bits=bits), S)
        for key in ("codes", "m", "s", "c", "w"):
            np.testing.assert_array_equal(v[key], base[key])


def test_error_grows_with_the_step(orc):
    S = gen.random_state(4, 64, 64, seed=8).numpy()
    err = {}
    for bits in (8, 6, 4):
        cfg = orc.Cfg(dk=64, dv=64, r=2, K=8, bits=bits)
        e = 0.0
        for h in range(4):
            v = orc.quantize(cfg, S[h])
            e += float(np.sum((S[h] - orc.dequantize(cfg, v)) ** 2))
        err[bits] = np.sqrt(e)
    # a uniform rounding error scales with the step amax / qmax
    assert 0.75 < (err[6] / err[8]) / (127 / 31) < 1.33
    assert 0.75 < (err[4] / err[6]) / (31 / 7) < 1.33


@pytest.mark.parametrize("gate", ["gdn", "kda"])
@pytest.mark.parametrize("bits", [4, 6])
def test_brute_force_windowed_d4(orc, gate, bits):
    dk = dv = 4
    T, W, r = 16, 4, 1
    tok = tiny_tokens(50 + bits, T, dk, dv, gate, nh=1)
    S0 = gen.random_state(1, dk, dv, seed=6, n_out=1, out_factor=5.0).numpy()
    cfg = orc.Cfg(dk=dk, dv=dv, gate=gate, W=W, r=r, K=8, bits=bits)
    res = orc.run(cfg, tok, S0=S0, flush_last=True)
    outs, view = brute.run_windowed(S0[0], tok_list(tok, 0), W=W, r=r, K=8, gate=gate, qmax=QMAX[bits])
    np.testing.assert_allclose(res["o"][:, 0], outs, rtol=1e-5, atol=1e-5 * np.abs(outs).max())
    ov = {k: res["view"][k][0] for k in ("codes", "m", "s")}
    np.testing.assert_allclose(ov["s"], view["s"], rtol=1e-5)
    rq = orc.quantize(cfg, res["S_pre"][0].astype(f32), want_ratio=True)
    assert _codes_match(ov["codes"], view["codes"], rq["ratio"])
    assert np.abs(ov["codes"]).max() <= QMAX[bits]
