"""Pins of the oracle's BF16-buffer mode (the traffic-lean buffer: each
token's rank-one update stored as bf16(k / Gamma) and bf16(u), compensators
and the INT8 state unchanged).

* When every stored value is BF16-representable -- unit keys, beta = 1, no
  decay, BF16 values v on an empty state -- the mode equals the FP32 buffer
  exactly.
* One token on an empty window: the output is q_0 * Gamma * bf16(k_0 / Gamma)
  * bf16(v) with BF16 rounding from torch and the division in numpy float32 --
  the key side is divided by the window's decay before rounding, not rounded
  as k.
* Many tokens: the recurrence's linear part (I - beta k k^T) D is
  non-expansive for |k| = 1, beta in (0, 1), 0 < D <= 1, so the BF16 run stays
  within the sum of its per-token rounding errors (each at most a BF16 half
  unit on both factors) of the FP32 run, and differs from it.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O

f32 = np.float32


def bf16(x):
    return torch.tensor(np.asarray(x, f32)).to(torch.bfloat16).to(torch.float32).numpy()


def run(cfg, q, k, v, beta, alpha):
    T, nh = q.shape[0], q.shape[1]
    inputs = {"q": q, "k": k, "v": v, "beta": beta, "alpha": alpha}
    S0 = np.zeros((nh, cfg.dk, cfg.dv), f32)
    return O.run(cfg, inputs, S0=S0)


def cfgs(dk, dv, W, gate="gdn"):
    base = dict(dk=dk, dv=dv, gate=gate, W=W, r=0, K=8, smoothing=1)
    return O.Cfg(**base, bf16_buffer=0), O.Cfg(**base, bf16_buffer=1)


def test_bf16_buffer_equals_fp32_buffer_on_representable_values():
    rng = np.random.default_rng(1)
    d, T = 8, 6
    c32, c16 = cfgs(d, d, 16)
    q = rng.standard_normal((T, 1, d)).astype(f32)
    k = np.zeros((T, 1, d), f32)
    for t in range(T):
        k[t, 0, t] = 1.0                                  # orthogonal unit keys: y_k = 0
    v = bf16(rng.standard_normal((T, 1, d)))               # BF16 values: u = v exactly
    beta = np.ones((T, 1), f32)
    alpha = np.ones((T, 1), f32)
    a, b = run(c32, q, k, v, beta, alpha), run(c16, q, k, v, beta, alpha)
    assert np.array_equal(a["o"], b["o"])
    assert np.array_equal(a["S"], b["S"])


@pytest.mark.parametrize("gate", ["gdn", "kda"])
def test_one_token_closed_form(gate):
    rng = np.random.default_rng(2)
    d = 8
    _, c16 = cfgs(d, d, 16, gate)
    q = rng.standard_normal((1, 1, d)).astype(f32)
    kappa = f32(0.3)
    k = np.zeros((1, 1, d), f32)
    k[0, 0, 0] = kappa
    v = rng.standard_normal((1, 1, d)).astype(f32)         # not BF16-representable
    beta = np.ones((1, 1), f32)
    a0 = f32(0.7)
    alpha = np.full((1, 1, d) if gate == "kda" else (1, 1), a0, f32)
    got = run(c16, q, k, v, beta, alpha)["o"][0, 0]
    gam = a0 * f32(1.0)                                    # Gamma after one token of a fresh window
    khat = bf16(np.float32(kappa) / gam)                   # float32 division, then BF16
    want = np.float64(q[0, 0, 0]) * np.float64(gam) * np.float64(khat) * bf16(v[0, 0]).astype(np.float64)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=0)
    # rounding k itself would give a different result here
    wrong = np.float64(q[0, 0, 0]) * np.float64(bf16(kappa)) * bf16(v[0, 0]).astype(np.float64)
    assert not np.allclose(wrong, want, rtol=1e-9, atol=0)


@pytest.mark.parametrize("gate", ["gdn", "kda"])
def test_many_tokens_within_the_rounding_bound(gate):
    rng = np.random.default_rng(3)
    d, T, W = 16, 24, 32                                   # one window, no flush
    c32, c16 = cfgs(d, d, W, gate)
    q = rng.standard_normal((T, 1, d)).astype(f32)
    k = rng.standard_normal((T, 1, d)).astype(f32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, 1, d)).astype(f32)
    beta = (1 / (1 + np.exp(-rng.standard_normal((T, 1))))).astype(f32)
    shape = (T, 1, d) if gate == "kda" else (T, 1)
    alpha = np.exp(-np.log1p(np.exp(rng.normal(-2.0, 0.5, shape)))).astype(f32)
    a, b = run(c32, q, k, v, beta, alpha), run(c16, q, k, v, beta, alpha)
    # per token: |Gamma bf16(k/Gamma) bf16(u) - k u| <= (2^-8 + 2^-16) |k| |u|,
    # |u| <= beta (|v| + |S|) with |S| bounded by the FP32 run's state plus slack
    smax = max(np.linalg.norm(a["S"][0]), 1.0) * 2.0
    eps = 2.0 ** -8 + 2.0 ** -16
    bound_S = 0.0
    for t in range(T):
        u_bound = float(beta[t, 0]) * (np.linalg.norm(v[t, 0]) + smax)
        bound_S += eps * u_bound                           # |k| = 1
        do = np.linalg.norm(b["o"][t, 0] - a["o"][t, 0])
        assert do <= bound_S * np.linalg.norm(q[t, 0]) * (1 + 1e-6)
    dS = np.linalg.norm(b["S"][0] - a["S"][0])
    assert dS <= bound_S
    assert dS > 0                                          # the rounding did happen


def test_zero_decay_restarts_the_key_chain():
    """A decay of exactly 0 wipes the state; the token then enters with the
    key chain restarted at 1: S = bf16(k) bf16(beta v)^T (y = 0 on the wiped
    state), o = S^T q -- finite, where k / Gamma with Gamma = 0 is not."""
    rng = np.random.default_rng(4)
    d = 8
    for gate in ("gdn", "kda"):
        _, c16 = cfgs(d, d, 16, gate)
        q = rng.standard_normal((2, 1, d)).astype(f32)
        k = rng.standard_normal((2, 1, d)).astype(f32)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        v = rng.standard_normal((2, 1, d)).astype(f32)
        beta = np.array([[0.6], [0.8]], f32)
        shape = (2, 1, d) if gate == "kda" else (2, 1)
        alpha = np.full(shape, 0.7, f32)
        alpha[1] = 0.0
        got = run(c16, q, k, v, beta, alpha)
        u = bf16((np.float32(beta[1, 0]) * v[1, 0]).astype(f32)).astype(np.float64)
        S = np.outer(bf16(k[1, 0]).astype(np.float64), u)
        np.testing.assert_allclose(got["S"][0], S, rtol=1e-15, atol=0)
        np.testing.assert_allclose(got["o"][1, 0], S.T @ q[1, 0].astype(np.float64), rtol=1e-12, atol=1e-300)


@pytest.mark.parametrize("gate", ["gdn", "kda"])
def test_power_of_two_decays_past_the_fp32_range(gate):
    """Decays of 2^-10 a token for 30 tokens take Gamma to 2^-300, far below
    FP32.  With a power-of-two decay chain, G bf16(k / G) = bf16(k) exactly
    (scaling by a power of two commutes with rounding), so each token enters
    as bf16(k) bf16(u)^T with u = bf16(fp32(beta (v - y))) and the state
    decaying exactly: the whole window has this closed form, finite."""
    rng = np.random.default_rng(5)
    d, T = 8, 30
    _, c16 = cfgs(d, d, 64, gate)
    q = rng.standard_normal((T, 1, d)).astype(f32)
    k = rng.standard_normal((T, 1, d)).astype(f32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, 1, d)).astype(f32)
    beta = (1 / (1 + np.exp(-rng.standard_normal((T, 1))))).astype(f32)
    shape = (T, 1, d) if gate == "kda" else (T, 1)
    alpha = np.full(shape, 2.0 ** -10, f32)
    if gate == "kda":
        alpha[:, :, ::2] = 0.5                              # channels at different depths
    got = run(c16, q, k, v, beta, alpha)
    S = np.zeros((d, d))
    for t in range(T):
        a = alpha[t, 0].astype(np.float64)
        S = (a[:, None] if gate == "kda" else a) * S
        y = S.T @ k[t, 0].astype(np.float64)
        u = bf16((np.float64(beta[t, 0]) * (v[t, 0].astype(np.float64) - y)).astype(f32)).astype(np.float64)
        S = S + np.outer(bf16(k[t, 0]).astype(np.float64), u)
        np.testing.assert_allclose(got["o"][t, 0], S.T @ q[t, 0].astype(np.float64), rtol=1e-12, atol=1e-300)
    assert np.isfinite(got["S"]).all()
    np.testing.assert_allclose(got["S"][0], S, rtol=1e-12, atol=1e-300)
