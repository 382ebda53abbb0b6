"""lq_quantize_state_static: quantizing a state without the library allocating
any device memory.

The regular lq_quantize_state puts the BF16 row list in a temporary it
allocates on the stream.  Callers whose device memory is owned by their own
allocator (reserved up front), or that must not allocate after start-up, use
this variant, which keeps the row list in a fixed array inside liblq.so.  The
GPU test checks it against the regular call on two calls in a row (and with a
changed row list, since every call overwrites the shared array); the CPU test
checks the size limit is reported before anything touches the GPU.
"""
import ctypes as C

import pytest
import torch

from quantized_recurrent_state_lq_b200 import inputs as gen, lq


def _rows(H, dk, P, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.sort(torch.randperm(dk, generator=g)[:P]).values for _ in range(H)]).int().numpy()


@pytest.mark.gpu
def test_static_variant_matches_allocating_call():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    cfg = lq.Config(B=2, H=4, Hk=4, dk=128, dv=128, r=2, power_iters=8, n_hp_rows=16)
    S = gen.random_state(cfg.B * cfg.H, cfg.dk, cfg.dv, seed=21).reshape(cfg.B, cfg.H, cfg.dk, cfg.dv).cuda()
    for seed in (1, 2):                      # a changed row list between calls
        rows = _rows(cfg.H, cfg.dk, cfg.n_hp_rows, seed)
        want = lq.alloc_view(cfg)
        lq.lq_quantize_state(cfg, S, want, hp_rows=rows)
        for _ in range(2):                   # two calls in a row
            got = lq.alloc_view(cfg)
            lq.lq_quantize_state_static(cfg, S, got, hp_rows=rows)
            torch.cuda.synchronize()
            for k in ("codes", "bf16_rows"):
                assert torch.equal(got[k], want[k]), k
            for k in ("m", "s", "comp_k", "comp_v"):
                torch.testing.assert_close(got[k], want[k], rtol=1e-5, atol=0), k


def test_static_variant_rejects_row_lists_beyond_its_array():
    L = lq.lib()
    H, P = 100, 100                          # 10000 > LQ_STATIC_ROWS_MAX
    assert H * P > lq.LQ_STATIC_ROWS_MAX
    cfg = lq.Config(B=1, H=H, Hk=H, dk=128, dv=128, r=2, n_hp_rows=P)
    rows = (C.c_int32 * (H * P))(*[p for _ in range(H) for p in range(P)])
    fake = 0x7f0000000000                    # never dereferenced: the check comes first
    view = lq.lq_qstate_view(fake, fake, fake, fake, fake, fake)
    rc = L.lq_quantize_state_static(C.byref(cfg.c()), C.c_void_p(fake), rows, C.byref(view), None)
    assert rc == lq.LQ_ERR_UNSUPPORTED
