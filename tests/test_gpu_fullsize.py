"""Parity at the workloads' full sizes, in the launch configuration bench.py
times (whole batch, CUDA-graph replay of one window, fused flush), on a sample
of heads the oracle recomputes one by one.

1. The GPU prefill (the chunked prefill, all heads, the full prefill length)
   is compared with the oracle's prefill of the sampled heads on the same
   inputs.
2. The sampled heads' initial states are replaced by the oracle's, both sides
   quantize them (codes compared with the rounding-tie slack).
3. For each of three windows, the sampled heads' window-start views are set
   to the oracle's (teacher forcing) and the window is replayed from its
   captured graph; outputs and the flushed state of the sampled heads are
   compared with the oracle.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_recurrent_state_lq_b200 import configs, inputs as gen, lq, runner
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

WINDOWS = 3   # windows replayed per workload, each teacher-forced on the sampled heads


def _sample(wl, n=16):
    g = torch.Generator().manual_seed(wl.seed + 1000)
    pts = {(0, 0), (wl.B - 1, wl.H - 1)}
    while len(pts) < n:
        pts.add((int(torch.randint(wl.B, (1,), generator=g)), int(torch.randint(wl.H, (1,), generator=g))))
    return sorted(pts)


def _rows(wl):
    if not wl.P:
        return None
    g = torch.Generator().manual_seed(wl.seed + 2000)
    return torch.stack([torch.sort(torch.randperm(wl.dk, generator=g)[:wl.P]).values
                        for _ in range(wl.H)]).int().numpy()


def _wid(w):
    return w.name + (f"-{w.bits}bit" if w.bits != 8 else "") + ("-bf16buf" if w.buffer_bf16 else "")


@pytest.mark.parametrize("wl", configs.WORKLOADS[1:] + [configs.KDA_B256.with_(bits=4),
                                                        configs.GDN_PREFIX_CACHE.with_(bits=6),
                                                        configs.GDN_PREFIX_CACHE.with_(buffer_bf16=1)], ids=_wid)
def test_full_size_sampled_heads(wl):
    U.require_gpu()
    heads = _sample(wl)
    S, cap = runner.gpu_prefill(wl, capture_heads=heads)
    bsel = sorted({b for b, _ in heads})
    local = [(bsel.index(b), h) for b, h in heads]
    oc0 = O.Cfg(dk=wl.dk, dv=wl.dv, gate=wl.gate, quantize=0)
    pre = O.prefill(oc0, O.per_head_inputs(cap, wl.H, heads=local))
    idx_b = torch.tensor([b for b, _ in heads])
    idx_h = torch.tensor([h for _, h in heads])
    got0 = S[idx_b.cuda(), idx_h.cuda()].cpu().numpy()
    e0 = U.rel_inf_rows(got0.reshape(len(heads), -1), pre.reshape(len(heads), -1))
    print(f"{_wid(wl)}: prefill ({wl.prefill} tokens, chunked) max rel err {e0.max():.2e}")
    assert e0.max() < 1e-3

    # both sides start from the oracle's prefilled state of the sampled heads
    S[idx_b.cuda(), idx_h.cuda()] = torch.from_numpy(pre.astype(np.float32)).cuda()
    S = gen.apply_outliers(S, wl)
    S_s = S[idx_b.cuda(), idx_h.cuda()].cpu().numpy()
    rows = _rows(wl)
    hr = None if rows is None else np.ascontiguousarray(rows[idx_h.numpy()])
    r = runner.WindowRunner(wl, S, hp_rows=rows, tokens=WINDOWS * wl.W)
    cfg = r.cfg
    oc = U.ocfg(cfg)
    ns = len(heads)
    ov = O.empty_views(oc, ns)
    for i in range(ns):
        q = O.quantize(oc, S_s[i], hp_rows=None if hr is None else hr[i], want_ratio=True)
        for k in ov:
            ov[k][i][...] = np.asarray(q[k]).reshape(ov[k][i].shape)
        ov.setdefault("ratio", np.zeros((ns, wl.dk, wl.dv)))[i] = q["ratio"]
    ratio0 = ov.pop("ratio")
    gv = lq.alloc_view(cfg)
    lq.lq_state_export_view(r.st, gv)
    sub = lq.Config(**{**cfg.__dict__, "B": 1, "H": ns})
    pick = {k: v[idx_b.cuda(), idx_h.cuda()].unsqueeze(0).contiguous() for k, v in gv.items()}
    got = U.gpu_view_to_oracle(sub, pick, None if hr is None else hr)
    flips = total = 0
    for i in range(ns):
        hri = None if hr is None else hr[i]
        c = U.check_quantized(oc, U.head_view(got, i), U.head_view(ov, i), ratio0[i], S_s[i].astype(np.float64),
                              0.0, hp_rows=hri, label=f"{wl.name} initial head {i}")
        flips += c["n"]
        total += c["total"]
    print(f"{wl.name}: initial codes {flips}/{total} differ")
    U.assert_code_bar({"n": flips, "total": total}, wl.name + " initial")

    # teacher forcing, window by window: the sampled heads start each window
    # from the oracle's view; every window is a replay of its captured graph
    r.capture()
    tok_all = O.per_head_inputs(r.tok, wl.H, heads=heads)
    flips = total = n_risk = n_undet = 0
    for w in range(WINDOWS):
        lq.lq_state_export_view(r.st, gv)
        ovg = U.oracle_view_to_gpu(sub, ov, None if hr is None else hr)
        for k in gv:
            gv[k][idx_b.cuda(), idx_h.cuda()] = ovg[k][0]
        lq.lq_state_import_view(r.st, gv)
        r.replay(w)
        torch.cuda.synchronize()
        assert lq.lq_get_status(r.st) == lq.LQ_OK
        sl = slice(w * wl.W, (w + 1) * wl.W)
        assert torch.isfinite(r.out[sl]).all()
        tok_s = {k: v[sl] for k, v in tok_all.items()}
        ref = O.run(oc, tok_s, view=ov, hp_rows=hr, flush_last=True)
        out = r.out[sl][:, idx_b.cuda(), idx_h.cuda()].cpu().numpy()
        e = U.rel_inf_rows(out, ref["o"])
        print(f"{_wid(wl)} window {w}: outputs max rel err {e.max():.2e}")
        assert e.max() < 1e-3
        lq.lq_state_export_view(r.st, gv)
        pick = {k: v[idx_b.cuda(), idx_h.cuda()].unsqueeze(0).contiguous() for k, v in gv.items()}
        got = U.gpu_view_to_oracle(sub, pick, None if hr is None else hr)
        ratio = U.oracle_ratios(sub, ref["S_pre"].astype(np.float32), hr)
        fw = 0
        for i in range(ns):
            hri = None if hr is None else hr[i]
            # the fused flush's FP32 pre-flush state is bounded, not exported
            bound, risk = U.window_state_bound(oc, U.head_view(ov, i), {k: v[:, i] for k, v in tok_s.items()},
                                               hp_rows=hri, risk_cols=True)
            c = U.check_quantized(oc, U.head_view(got, i), U.head_view(ref["view"], i), ratio[i],
                                  ref["S_pre"][i], bound, hp_rows=hri, label=f"{wl.name} window {w} head {i}",
                                  risk_cols=risk)
            if risk.any():   # a BF16 u tie reaches every column through the compensators
                c = dict(c, n=0, n_risk=c["n"] + c["n_risk"])
            fw += c["n"]
            flips += c["n"]
            total += c["total"]
            n_risk += c["n_risk"]
            n_undet += c["n_undetermined"]
        print(f"{_wid(wl)} window {w}: flushed codes {fw} differ")
        U.assert_flush_params(sub, got, ref["view"], ref["S_pre"], hr, f"{wl.name} window {w} flushed")
        ov = ref["view"]
    print(f"{_wid(wl)}: flushed codes over {WINDOWS} windows {flips}/{total} differ "
          f"({n_risk} more in BF16-tie columns, {n_undet} undetermined)")
    U.assert_code_bar({"n": flips, "total": total}, f"{wl.name} flushed", U.FLUSH_FLIP_FRAC)
