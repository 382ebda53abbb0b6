"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a closed form, a library routine, a hand
worked example (tests/golden/hand_worked.json) or the independent brute force
in tests/brute.py, chosen so that a dropped term, a sign, a transposed operand
or a wrong operator order in the oracle fails at least one of them.
"""
import json
import os

import numpy as np
import pytest
import torch

from tests import brute

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))
f32 = np.float32


def rnd(seed):
    return np.random.default_rng(seed)


def unit(x):
    return x / np.linalg.norm(x)


def rand_token(rng, dk, dv, gate):
    q = unit(rng.standard_normal(dk)).astype(f32)
    k = unit(rng.standard_normal(dk)).astype(f32)
    v = rng.standard_normal(dv).astype(f32)
    beta = f32(1 / (1 + np.exp(-rng.standard_normal())))
    if gate == "gdn":
        alpha = np.array([np.exp(-np.log1p(np.exp(rng.normal(-1, 1))))], f32)
    else:
        alpha = np.exp(-np.log1p(np.exp(rng.normal(-1, 1, dk)))).astype(f32)
    return q, k, v, beta, alpha


# ---------------------------------------------------------------- recurrence

@pytest.mark.parametrize("case", GOLD["steps"], ids=lambda c: c["name"])
def test_step_hand_worked(orc, case):
    S0 = np.array(case["S0"], np.float64)
    cfg = orc.Cfg(dk=S0.shape[0], dv=S0.shape[1], gate=case["gate"])
    S1, o = orc.step(cfg, S0, case["q"], case["k"], case["v"], case["beta"], case["alpha"])
    np.testing.assert_array_equal(S1, np.array(case["S1"]))
    np.testing.assert_array_equal(o, np.array(case["o"]))


@pytest.mark.parametrize("gate", ["gdn", "kda"])
@pytest.mark.parametrize("dk,dv", [(4, 4), (4, 6), (6, 3)])
def test_step_matches_pages_matrix_form(orc, gate, dk, dv):
    """Table 3 in the pages' own (d_v x d_k) orientation, literal matrices."""
    rng = rnd(dk * 10 + dv + (gate == "kda"))
    cfg = orc.Cfg(dk=dk, dv=dv, gate=gate)
    S = rng.standard_normal((dk, dv))
    Sp = S.T.copy()
    for _ in range(5):
        q, k, v, beta, alpha = rand_token(rng, dk, dv, gate)
        S, o = orc.step(cfg, S, q, k, v, float(beta), alpha)
        Sp, op = brute.step_pages_form(Sp, q, k, v, float(beta), alpha, gate)
        np.testing.assert_allclose(S, Sp.T, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o, op, rtol=1e-12, atol=1e-12)


def test_kda_operator_order_is_decay_then_projection(orc):
    """D and (I - b k k^T) do not commute for a per-channel D; the oracle must
    follow the page's order S diag(a) (I - b k k^T), which the other order fails."""
    rng = rnd(7)
    dk = dv = 4
    cfg = orc.Cfg(dk=dk, dv=dv, gate="kda")
    S = rng.standard_normal((dk, dv))
    q, k, v, beta, alpha = rand_token(rng, dk, dv, "kda")
    S1, _ = orc.step(cfg, S, q, k, v, float(beta), alpha)
    kk = k.astype(np.float64)
    P = np.eye(dk) - float(beta) * np.outer(kk, kk)
    D = np.diag(alpha.astype(np.float64))
    right = P @ D @ S + float(beta) * np.outer(kk, v)
    wrong = D @ P @ S + float(beta) * np.outer(kk, v)
    np.testing.assert_allclose(S1, right, rtol=1e-12, atol=1e-12)
    assert np.abs(S1 - wrong).max() > 1e-3


@pytest.mark.parametrize("gate", ["gdn", "kda"])
def test_beta_zero_is_pure_decay(orc, gate):
    """beta = 0: S_t = Gamma_t S_0 with Gamma_t the product of the gates."""
    rng = rnd(11)
    dk, dv = 5, 3
    cfg = orc.Cfg(dk=dk, dv=dv, gate=gate)
    S0 = rng.standard_normal((dk, dv))
    S = S0.copy()
    gam = np.ones(dk)
    for _ in range(6):
        q, k, v, _, alpha = rand_token(rng, dk, dv, gate)
        S, o = orc.step(cfg, S, q, k, v, 0.0, alpha)
        gam *= np.broadcast_to(alpha.astype(np.float64), (dk,)) if gate == "kda" else float(alpha[0])
        np.testing.assert_allclose(S, gam[:, None] * S0, rtol=1e-13)
        np.testing.assert_allclose(o, (gam[:, None] * S0).T @ q.astype(np.float64), rtol=1e-12, atol=1e-14)


def test_unit_key_full_write_replaces_row(orc):
    """k = e_i, beta = 1: row i of S_t is v_t; other rows are only decayed."""
    rng = rnd(12)
    dk, dv = 4, 5
    cfg = orc.Cfg(dk=dk, dv=dv, gate="kda")
    S0 = rng.standard_normal((dk, dv))
    k = np.zeros(dk, f32); k[2] = 1
    v = rng.standard_normal(dv).astype(f32)
    alpha = np.array([0.5, 0.25, 0.75, 0.125], f32)
    S1, _ = orc.step(cfg, S0, np.ones(dk, f32), k, v, 1.0, alpha)
    # exact in the mathematics; the rank-one form a + (v - a) rounds once
    np.testing.assert_allclose(S1[2], v.astype(np.float64), rtol=1e-15, atol=1e-15)
    for i in (0, 1, 3):
        np.testing.assert_array_equal(S1[i], alpha[i] * S0[i])


def test_alpha_one_reduces_to_deltanet(orc):
    """alpha = 1: the DeltaNet row of Table 3, S_t = S (I - b k k^T) + b v k^T (pages' form)."""
    rng = rnd(13)
    dk, dv = 4, 4
    cfg = orc.Cfg(dk=dk, dv=dv, gate="gdn")
    S = rng.standard_normal((dk, dv))
    for _ in range(4):
        q, k, v, beta, _ = rand_token(rng, dk, dv, "gdn")
        Sp = S.T
        kk = k.astype(np.float64)
        want = Sp @ (np.eye(dk) - float(beta) * np.outer(kk, kk)) + float(beta) * np.outer(v, kk)
        S, _ = orc.step(cfg, S, q, k, v, float(beta), np.ones(1, f32))
        np.testing.assert_allclose(S.T, want, rtol=1e-12, atol=1e-13)


def test_alpha_one_beta_zero_is_gemv(orc):
    rng = rnd(14)
    cfg = orc.Cfg(dk=6, dv=5, gate="gdn")
    S0 = rng.standard_normal((6, 5))
    q = rng.standard_normal(6).astype(f32)
    _, o = orc.step(cfg, S0, q, np.ones(6, f32), np.ones(5, f32), 0.0, np.ones(1, f32))
    np.testing.assert_allclose(o, np.dot(S0.T, q.astype(np.float64)), rtol=1e-13)


# ---------------------------------------------------------------- quantizer

@pytest.mark.parametrize("case", GOLD["codecs"], ids=lambda c: c["name"])
def test_codec_hand_worked(orc, case):
    S = np.array(case["S"], f32)
    cfg = orc.Cfg(dk=S.shape[0], dv=S.shape[1], r=case["r"], K=case["K"], smoothing=case["smoothing"])
    v = orc.quantize(cfg, S)
    np.testing.assert_array_equal(v["codes"], np.array(case["codes"]))
    np.testing.assert_allclose(v["m"], case["m"], rtol=1e-7)
    np.testing.assert_allclose(v["s"] * 127, case["s_times_127"], rtol=1e-6)


def test_compensator_hand_worked(orc):
    case = GOLD["compensators"][0]
    S = np.array(case["S"], f32)
    cfg = orc.Cfg(dk=2, dv=2, r=case["r"], K=case["K"])
    v = orc.quantize(cfg, S)
    sign = np.sign(v["w"][0][0])
    np.testing.assert_allclose(sign * v["w"][0], case["w"], rtol=1e-6)
    np.testing.assert_allclose(sign * v["c"][0], case["c"], rtol=1e-6)
    np.testing.assert_allclose(orc.dequantize(cfg, v), S, atol=1e-5)


def _residual(S, v):
    R = S.astype(np.float64)
    for c, w in zip(v["c"], v["w"]):
        R = R - np.outer(c.astype(np.float64), w.astype(np.float64))
    return R


@pytest.mark.parametrize("r,smoothing", [(0, 0), (0, 1), (2, 1), (4, 1)])
def test_dequantization_error_within_half_step(orc, r, smoothing):
    """|R_ic - Deq_ic| <= m_i s_c / 2 (1 + 4 eps) for every entry, and the
    compensators are exact rank-one terms: S - Deq(Q(S)) = R - Deq(codes)."""
    import quantized_recurrent_state_lq_b200.inputs as gen
    S = gen.random_state(3, 16, 12, seed=5).numpy()
    cfg = orc.Cfg(dk=16, dv=12, r=r, K=8, smoothing=smoothing)
    eps = np.finfo(f32).eps
    for h in range(3):
        v = orc.quantize(cfg, S[h])
        R = _residual(S[h], v)
        deq = ((v["codes"].astype(f32) * v["s"]).astype(f32) * v["m"][:, None]).astype(np.float64)
        bound = v["m"][:, None].astype(np.float64) * v["s"][None, :] / 2 * (1 + 4 * eps) + 1e-30
        assert np.all(np.abs(R - deq) <= bound + 4 * eps * np.abs(R))
        full = orc.dequantize(cfg, v)
        np.testing.assert_allclose(S[h] - full, R - deq, atol=1e-5 * np.abs(S[h]).max())


def test_codes_are_exhaustive_argmin_d4(orc):
    """At d = 4 the stored code is the nearest of all 255 levels (ties to even)."""
    rng = rnd(21)
    for trial in range(20):
        S = (rng.standard_normal((4, 4)) * rng.uniform(0.1, 10, (4, 1))).astype(f32)
        cfg = orc.Cfg(dk=4, dv=4, r=1, K=8)
        v = orc.quantize(cfg, S, want_ratio=True)
        b = brute.quantize(S, r=1, K=8)
        np.testing.assert_allclose(v["c"], b["c"], rtol=2e-6, atol=1e-6 * np.abs(S).max())
        np.testing.assert_allclose(v["w"], b["w"], rtol=2e-6, atol=2e-7)
        x = b["x"]
        mine = brute.codes_exhaustive(x, b["s"])
        near_tie = np.abs(np.abs(v["ratio"] - np.trunc(v["ratio"])) - 0.5) < 1e-4
        assert np.all((v["codes"] == mine) | near_tie)


def test_column_amax_maps_to_full_scale(orc):
    import quantized_recurrent_state_lq_b200.inputs as gen
    S = gen.random_state(2, 32, 24, seed=9).numpy()
    cfg = orc.Cfg(dk=32, dv=24, r=2, K=8)
    for h in range(2):
        v = orc.quantize(cfg, S[h])
        assert np.all(np.abs(v["codes"]).max(axis=0) == 127)
        assert np.abs(v["codes"]).max() <= 127


def test_smoothing_scale_is_row_rms_of_residual(orc):
    import quantized_recurrent_state_lq_b200.inputs as gen
    S = gen.random_state(1, 16, 16, seed=3).numpy()[0]
    cfg = orc.Cfg(dk=16, dv=16, r=2, K=8)
    v = orc.quantize(cfg, S)
    R = _residual(S, v).astype(f32).astype(np.float64)
    np.testing.assert_allclose(v["m"], np.sqrt((R ** 2).mean(axis=1)), rtol=1e-7)


# ---------------------------------------------------------------- compensators

def test_compensators_match_svd_with_spectral_gap(orc):
    """K large on a matrix with a clear gap: c_j w_j^T = sigma_j u_j v_j^T (numpy SVD)."""
    rng = rnd(31)
    dk, dv = 6, 8
    U, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    V, _ = np.linalg.qr(rng.standard_normal((dv, dv)))
    sig = np.array([10.0, 4.0, 1.0, 0.5, 0.25, 0.1])
    S = (U[:, :dk] * sig) @ V[:, :dk].T
    cfg = orc.Cfg(dk=dk, dv=dv, r=2, K=200)
    v = orc.quantize(cfg, S.astype(f32))
    u_, s_, vt_ = np.linalg.svd(S.astype(f32).astype(np.float64))
    for j in range(2):
        want = s_[j] * np.outer(u_[:, j], vt_[j])
        got = np.outer(v["c"][j], v["w"][j])
        np.testing.assert_allclose(got, want, atol=1e-5 * s_[0])


def test_power_iterate_equals_closed_form_K8(orc):
    """After K = 8 steps from w0 = 1/sqrt(d_v), w_1 is (R^T R)^8 w0 normalised."""
    import quantized_recurrent_state_lq_b200.inputs as gen
    S = gen.random_state(2, 12, 10, seed=4).numpy()
    cfg = orc.Cfg(dk=12, dv=10, r=2, K=8)
    for h in range(2):
        v = orc.quantize(cfg, S[h])
        w1 = brute.power_closed_form(S[h].astype(np.float64), 8)
        np.testing.assert_allclose(v["w"][0], w1, atol=1e-6)
        np.testing.assert_allclose(v["c"][0], S[h].astype(np.float64) @ v["w"][0].astype(np.float64),
                                   rtol=1e-6, atol=1e-6)
        R1 = S[h].astype(np.float64) - np.outer(v["c"][0], v["w"][0])
        w2 = brute.power_closed_form(R1, 8)
        np.testing.assert_allclose(v["w"][1], w2, atol=1e-5)


def test_low_rank_state_leaves_empty_residual(orc):
    rng = rnd(33)
    a = rng.standard_normal((8, 2)) * np.array([5.0, 1.0])
    b = rng.standard_normal((2, 8))
    S = (a @ b).astype(f32)
    cfg = orc.Cfg(dk=8, dv=8, r=2, K=300)
    v = orc.quantize(cfg, S)
    R = _residual(S, v)
    assert np.abs(R).max() < 1e-5 * np.abs(S).max()
    np.testing.assert_allclose(orc.dequantize(cfg, v), S, atol=1e-5 * np.abs(S).max())


def test_zero_state(orc):
    cfg = orc.Cfg(dk=8, dv=8, r=2, K=8)
    v = orc.quantize(cfg, np.zeros((8, 8), f32))
    assert np.all(v["codes"] == 0) and np.all(v["c"] == 0) and np.all(v["w"] == 0)
    assert np.all(v["m"] == 1) and np.all(v["s"] == 0)
    assert np.all(orc.dequantize(cfg, v) == 0)


def test_outlier_ratio_drops_after_compensators_and_smoothing(orc):
    """LeapQuant smoothing paragraph: compensators + smoothing shrink max/median."""
    import quantized_recurrent_state_lq_b200.inputs as gen
    S = gen.random_state(4, 64, 64, seed=8, out_factor=30.0).numpy()
    cfg = orc.Cfg(dk=64, dv=64, r=2, K=8)
    for h in range(4):
        v = orc.quantize(cfg, S[h])
        R = _residual(S[h], v)
        x = R / v["m"][:, None]
        before = np.abs(S[h]).max() / np.median(np.abs(S[h]))
        after = np.abs(x).max() / np.median(np.abs(x))
        assert after < before / 3, (before, after)


# ---------------------------------------------------------------- bf16 rows

def test_bf16_rounding_matches_torch(orc):
    rng = rnd(41)
    xs = np.concatenate([rng.standard_normal(2000) * 10 ** rng.uniform(-30, 30, 2000),
                         [0.0, -0.0, 1.0, 3.0, 1.00390625, 1.01171875, 65504.0, 3.3e38]]).astype(f32)
    want = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([orc.bf16_rne(float(x)) for x in xs], np.uint16)
    np.testing.assert_array_equal(got, want)


def test_damp_rows_stored_in_bf16_and_excluded(orc):
    import quantized_recurrent_state_lq_b200.inputs as gen
    S = gen.random_state(1, 16, 8, seed=2).numpy()[0]
    rows = np.array([1, 5, 9], np.int32)
    cfg = orc.Cfg(dk=16, dv=8, r=1, K=8, P=3)
    v = orc.quantize(cfg, S, hp_rows=rows)
    R = _residual(S, v).astype(f32)
    want = torch.from_numpy(R[rows]).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    np.testing.assert_array_equal(v["hp"][:3], want)
    assert np.all(v["codes"][rows] == 0)
    others = np.setdiff1d(np.arange(16), rows)
    x = R[others] / v["m"][others, None]
    np.testing.assert_allclose(v["s"] * 127, np.abs(x).max(axis=0), rtol=1e-6)
    full = orc.dequantize(cfg, v, hp_rows=rows)
    hp_f = torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy()
    comp = np.outer(v["c"][0].astype(np.float64), v["w"][0].astype(np.float64))[rows]
    np.testing.assert_allclose(full[rows], hp_f + comp, rtol=1e-12, atol=1e-12)


def test_damp_select_ties_to_lower_index(orc):
    score = np.array([1.0, 3.0, 3.0, 2.0, 3.0, 0.5])
    rows = orc.damp_select(score, 3)
    np.testing.assert_array_equal(rows, [1, 2, 4])
    rows = orc.damp_select(score, 2)
    np.testing.assert_array_equal(rows, [1, 2])
    rng = rnd(43)
    sc = rng.standard_normal(128)
    want = np.sort(np.argsort(-sc, kind="stable")[:16])
    np.testing.assert_array_equal(orc.damp_select(sc, 16), want)


def test_damp_energy_definition(orc):
    import quantized_recurrent_state_lq_b200.inputs as gen
    S = gen.random_state(3, 16, 8, seed=6).numpy()
    cfg = orc.Cfg(dk=16, dv=8, r=2, K=8)
    E = orc.damp_energy(cfg, S)
    want = np.zeros(16)
    for h in range(3):
        b = brute.quantize(S[h], r=2, K=8)
        deq = ((b["codes"].astype(f32) * b["s"]).astype(f32) * b["m"][:, None]).astype(f32)
        want += ((b["R32"].astype(np.float64) - deq.astype(np.float64)) ** 2).sum(axis=1)
    np.testing.assert_allclose(E, want, rtol=1e-3)


@pytest.mark.parametrize("case", GOLD["damp_scores"], ids=lambda c: c["name"])
def test_damp_score_hand_worked(orc, case):
    """DAMP abstract: rows are chosen by error energy and decay persistence;
    the worked cases (exact binary fractions) include one where per-channel
    persistence (KDA) reorders rows that energy alone ranks the other way."""
    score = orc.damp_score(case["E"], np.asarray(case["gates"], f32))
    np.testing.assert_array_equal(score, np.asarray(case["score"]))
    np.testing.assert_array_equal(orc.damp_select(score, case["P"]), case["rows"])
    by_energy = orc.damp_select(np.asarray(case["E"]), case["P"])
    assert (not np.array_equal(by_energy, case["rows"])) == (case["gate"] == "kda")


def test_damp_score_persistence_limits(orc):
    """Decays of 0 leave the energy unchanged; a mean decay of 1 - 2^-j
    multiplies it by exactly 2^j; GDN's one decay scales every row alike."""
    E = np.array([1.0, 2.0, 3.0, 5.0])
    np.testing.assert_array_equal(orc.damp_score(E, np.zeros((3, 4), f32)), E)
    g = np.array([[1 - 2.0 ** -1, 1 - 2.0 ** -2, 1 - 2.0 ** -3, 1 - 2.0 ** -10]], f32)
    np.testing.assert_array_equal(orc.damp_score(E, g), E * np.array([2.0, 4.0, 8.0, 1024.0]))
    np.testing.assert_array_equal(orc.damp_score(E, np.full((5, 1), 0.75, f32)), 4.0 * E)
