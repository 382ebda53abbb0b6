"""Pins of the oracle's staggered windows (per-head window phases): head h's
first window holds W - phase[h] tokens, every later one W -- one
requantization per W tokens of each sequence (LeapQuant project page, window
paragraph), the sequences' window ends shifted against each other.

* Against the brute force of literal matrices with the same first-window
  length (d = 4, every phase of a W = 4 window, GDN and KDA).
* A zero phase is the unphased run, bit for bit.
* Composition: a phased run equals its first window run alone (ending in a
  flush) followed by an unphased run from that window's quantized state, bit
  for bit -- the phase only moves the first window end.
"""
import numpy as np
import pytest

from tests import brute
from tests.test_oracle_window import tiny_tokens, tok_list
from quantized_recurrent_state_lq_b200 import inputs as gen

f32 = np.float32


@pytest.mark.parametrize("gate", ["gdn", "kda"])
def test_phases_match_brute_force_d4(orc, gate):
    dk = dv = 4
    W, r, T = 4, 1, 14
    phases = np.array([0, 1, 2, 3], np.int32)
    nh = len(phases)
    tok = tiny_tokens(21, T, dk, dv, gate, nh=nh)
    S0 = gen.random_state(nh, dk, dv, seed=5, n_out=1, out_factor=5.0).numpy()
    cfg = orc.Cfg(dk=dk, dv=dv, gate=gate, W=W, r=r, K=8)
    res = orc.run(cfg, tok, S0=S0, phase=phases)
    for h in range(nh):
        outs, _ = brute.run_windowed(S0[h], tok_list(tok, h), W=W, r=r, K=8, gate=gate,
                                     first=W - int(phases[h]))
        np.testing.assert_allclose(res["o"][:, h], outs, rtol=1e-5, atol=1e-5 * np.abs(outs).max())
        # tokens since the last flush (the last token makes none: no flush_last)
        first = W - int(phases[h])
        n_exp = T if T <= first else (T - first - 1) % W + 1
        assert res["n"][h] == n_exp


@pytest.mark.parametrize("gate", ["gdn", "kda"])
def test_zero_phase_is_unphased(orc, gate):
    dk, dv, W, T, nh = 8, 6, 5, 17, 2
    tok = tiny_tokens(22, T, dk, dv, gate, nh=nh)
    S0 = gen.random_state(nh, dk, dv, seed=6).numpy()
    cfg = orc.Cfg(dk=dk, dv=dv, gate=gate, W=W, r=2, K=8)
    a = orc.run(cfg, tok, S0=S0)
    b = orc.run(cfg, tok, S0=S0, phase=np.zeros(nh, np.int32))
    np.testing.assert_array_equal(a["o"], b["o"])
    np.testing.assert_array_equal(a["S"], b["S"])


@pytest.mark.parametrize("gate", ["gdn", "kda"])
@pytest.mark.parametrize("p", [1, 3, 4])
def test_phase_is_a_shorter_first_window(orc, gate, p):
    dk, dv, W, T = 8, 8, 5, 19
    tok = tiny_tokens(23 + p, T, dk, dv, gate, nh=1)
    S0 = gen.random_state(1, dk, dv, seed=7).numpy()
    cfg = orc.Cfg(dk=dk, dv=dv, gate=gate, W=W, r=2, K=8)
    full = orc.run(cfg, tok, S0=S0, phase=np.array([p], np.int32))
    L = W - p
    head = orc.run(cfg, {k: v[:L] for k, v in tok.items()}, S0=S0, phase=np.array([p], np.int32),
                   flush_last=True)
    assert head["n"][0] == 0
    np.testing.assert_array_equal(full["o"][:L], head["o"])
    rest = orc.run(cfg, {k: v[L:] for k, v in tok.items()}, view=head["view"])
    np.testing.assert_array_equal(full["o"][L:], rest["o"])
    np.testing.assert_array_equal(full["S"], rest["S"])
