"""Failure detection on the GPU without a fault: a bounded device wait that
runs out (lq_selftest_wait) raises the state's timeout status, which the host
reads with lq_get_status; the context stays usable afterwards."""
import pytest
import torch

from quantized_recurrent_state_lq_b200 import configs, inputs as gen, lq
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    U.require_gpu()
    wl = configs.TINY_GDN.with_(B=1, H=2, Hk=2)
    cfg = lq.Config.from_workload(wl)
    S0 = gen.random_state(2, wl.dk, wl.dv, seed=9).reshape(1, 2, wl.dk, wl.dv).cuda()
    st = lq.lq_state_init(cfg, S0)
    assert lq.lq_get_status(st) == lq.LQ_OK
    lq.lq_selftest_wait(st, limit_ns=1_000_000)     # 1 ms, then the kernel returns
    assert lq.lq_get_status(st) == lq.LQ_ERR_TIMEOUT
    # the timeout is this state's: another state decodes normally afterwards
    st2 = lq.lq_state_init(cfg, S0)
    tok = gen.token_inputs(wl, 3, device="cuda")
    o = torch.empty((1, 2, wl.dv), device="cuda")
    for t in range(3):
        lq.lq_decode_step(st2, *U.step_args(tok, t), o)
    assert lq.lq_get_status(st2) == lq.LQ_OK
    assert torch.isfinite(o).all()
    with pytest.raises(lq.LqError) as ei:
        lq.lq_selftest_wait(st2, limit_ns=10)        # below the accepted range: refused on the host
    assert ei.value.code == lq.LQ_ERR_INVALID_ARG
    assert lq.lq_get_status(st2) == lq.LQ_OK
