"""DAMP row selection on the GPU (lq_damp_select) against the oracle's error
energies and top-P choice, on identical calibration states."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_recurrent_state_lq_b200 import configs, inputs as gen, lq
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("gate", ["gdn", "kda"])
def test_damp_select_matches_oracle(gate):
    U.require_gpu()
    n_cal, H, d, P, toks = 6, 4, 128, 16, 96
    wl = configs.GDN_DAMP.with_(gate=gate, B=n_cal, H=H, Hk=H, dk=d, dv=d, P=P, r=2, seed=70)
    cal = gen.token_inputs(wl, toks, stream="calib")
    oc = O.Cfg(dk=d, dv=d, gate=gate, quantize=0)
    states = O.prefill(oc, O.per_head_inputs(cal, H)).astype(np.float32).reshape(n_cal, H, d, d)
    states = gen.apply_outliers(torch.from_numpy(states), wl).numpy()
    gates = cal["alpha"].reshape(toks * n_cal, H, -1).contiguous()
    cfg = lq.Config(B=1, H=H, Hk=H, dk=d, dv=d, gate=gate, r=2, power_iters=8, n_hp_rows=P)
    energy = torch.zeros((H, d), dtype=torch.float64, device="cuda")
    rows = torch.zeros((H, P), dtype=torch.int32, device="cuda")
    lq.lq_damp_select(cfg, torch.from_numpy(states).cuda(), gates.cuda(), energy, rows)
    energy = energy.cpu().numpy()
    rows = rows.cpu().numpy()
    qc = O.Cfg(dk=d, dv=d, gate=gate, r=2, K=8)
    g = gates.numpy()
    for h in range(H):
        E = O.damp_energy(qc, np.ascontiguousarray(states[:, h]))
        np.testing.assert_allclose(energy[h], E, rtol=2e-3)
        score = O.damp_score(E, np.ascontiguousarray(g[:, h, :]))
        want = O.damp_select(score, P)
        if not np.array_equal(rows[h], want):
            # only a near-tie at the cut may differ
            cut = np.sort(score)[::-1][P - 1]
            diff = np.setxor1d(rows[h], want)
            assert np.all(np.abs(score[diff] - cut) <= 2e-3 * cut), (h, rows[h], want)
        assert np.all(np.diff(rows[h]) > 0)


def test_selected_rows_carry_large_error_share():
    """DAMP abstract: quantization-error energy concentrates in a few channels;
    on outlier-injected states the chosen rows hold a large share of it."""
    U.require_gpu()
    n_cal, H, d, P = 8, 2, 128, 16
    wl = configs.GDN_DAMP.with_(B=n_cal, H=H, Hk=H, P=P, seed=71)
    cal = gen.token_inputs(wl, 64, stream="calib")
    states = O.prefill(O.Cfg(dk=d, dv=d, quantize=0), O.per_head_inputs(cal, H)).astype(np.float32)
    states = gen.apply_outliers(torch.from_numpy(states.reshape(n_cal, H, d, d)), wl)
    cfg = lq.Config(B=1, H=H, Hk=H, dk=d, dv=d, r=2, n_hp_rows=P)
    energy = torch.zeros((H, d), dtype=torch.float64, device="cuda")
    rows = torch.zeros((H, P), dtype=torch.int32, device="cuda")
    lq.lq_damp_select(cfg, states.cuda(), cal["alpha"].reshape(-1, H, 1).contiguous().cuda(), energy, rows)
    e = energy.cpu().numpy()
    for h in range(H):
        share = e[h, rows[h].cpu().numpy()].sum() / e[h].sum()
        assert share > 2 * P / d, share
