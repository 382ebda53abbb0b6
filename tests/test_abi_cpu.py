"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/lq_state.h declares, validates configs and rejects
bad arguments before launching anything."""
import ctypes as C
import os
import re
import subprocess

import pytest

from quantized_recurrent_state_lq_b200 import configs, lq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lq_state.h")


@pytest.fixture(scope="module")
def L():
    return lq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["lq_state_init", "lq_decode_step", "lq_window_flush", "lq_quantize_state",
                 "lq_dequantize_state"]:
        assert must in names
    assert sorted(lq.EXPORTED) == names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", lq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (lq_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert getattr(L, n) is not None


@pytest.mark.parametrize("wl", configs.WORKLOADS, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", ["fp32", "step", "window"])
def test_workload_configs_are_valid(L, wl, mode):
    cfg = lq.Config.from_workload(wl, mode=mode)
    assert lq.lq_config_check(cfg) == lq.LQ_OK
    assert lq.lq_workspace_bytes(cfg) > 0


def test_workspace_size_matches_record_layout(L):
    wl = configs.KDA_B256
    cfg = lq.Config.from_workload(wl)
    dk, dv, r, W = wl.dk, wl.dv, wl.r, wl.W
    # codes, m and s, entries, and the decay guard's G and sigma per key channel
    payload = (dk * dv) + 4 * (dk + dv) + 4 * (r + W) * (dk + dv) + 2 * 4 * dk
    per_head = (lq.lq_workspace_bytes(cfg) - 256) / wl.heads
    assert payload <= per_head <= payload + 128 + 64
    fp = lq.Config.from_workload(wl, mode="fp32")
    assert lq.lq_workspace_bytes(fp) == 256 + wl.heads * dk * dv * 4


@pytest.mark.parametrize("field,value,code", [
    ("dk", 96, lq.LQ_ERR_UNSUPPORTED), ("dv", 256, lq.LQ_ERR_UNSUPPORTED),
    ("Hk", 3, lq.LQ_ERR_SHAPE), ("B", 0, lq.LQ_ERR_SHAPE), ("H", 0, lq.LQ_ERR_SHAPE),
    ("W", 0, lq.LQ_ERR_INVALID_ARG), ("r", 129, lq.LQ_ERR_INVALID_ARG), ("r", -1, lq.LQ_ERR_INVALID_ARG),
    ("power_iters", -1, lq.LQ_ERR_INVALID_ARG), ("n_hp_rows", 128, lq.LQ_ERR_INVALID_ARG),
    ("smoothing", 3, lq.LQ_ERR_INVALID_ARG), ("fused_flush", 7, lq.LQ_ERR_INVALID_ARG),
    ("W", 4097, lq.LQ_ERR_UNSUPPORTED),
])
def test_config_errors(L, field, value, code):
    cfg = lq.Config.from_workload(configs.GDN_SERVING)
    setattr(cfg, field, value)
    assert lq.lq_config_check(cfg) == code
    assert lq.lq_workspace_bytes(cfg) == 0


def test_long_windows_are_accepted(L):
    # the window's buffered entries stream from the workspace; nothing of
    # their size has to fit in shared memory
    for W in (400, 4096):
        cfg = lq.Config.from_workload(configs.GDN_SERVING)
        cfg.W = W
        assert lq.lq_config_check(cfg) == lq.LQ_OK
        assert lq.lq_workspace_bytes(cfg) > 0


def test_step_mode_requires_window_one(L):
    cfg = lq.Config.from_workload(configs.GDN_SERVING, mode="step")
    assert lq.lq_config_check(cfg) == lq.LQ_OK
    cfg.W = 4
    assert lq.lq_config_check(cfg) == lq.LQ_ERR_INVALID_ARG


def _init(L, cfg, ws, nbytes, s0, rows=None):
    h = C.c_void_p()
    return L.lq_state_init(C.byref(h), C.byref(cfg.c()), C.c_void_p(ws), nbytes, C.c_void_p(s0), rows, None)


def test_state_init_rejects_bad_arguments_without_launching(L):
    """All of these fail on the host; the fake device addresses are never touched."""
    cfg = lq.Config.from_workload(configs.TINY_GDN)
    need = lq.lq_workspace_bytes(cfg)
    fake_ws, fake_s0 = 0x7f0000000000, 0x7f1000000000
    h = C.c_void_p()
    assert L.lq_state_init(None, C.byref(cfg.c()), C.c_void_p(fake_ws), need, C.c_void_p(fake_s0), None, None) \
        == lq.LQ_ERR_INVALID_ARG
    assert _init(L, cfg, None, need, fake_s0) == lq.LQ_ERR_INVALID_ARG
    assert _init(L, cfg, fake_ws, need, None) == lq.LQ_ERR_INVALID_ARG
    assert _init(L, cfg, fake_ws + 64, need, fake_s0) == lq.LQ_ERR_WORKSPACE
    assert _init(L, cfg, fake_ws, need - 1, fake_s0) == lq.LQ_ERR_WORKSPACE
    bad = lq.Config.from_workload(configs.TINY_GDN)
    bad.Hk = 3
    assert _init(L, bad, fake_ws, need, fake_s0) == lq.LQ_ERR_SHAPE


def test_state_init_checks_bf16_row_lists(L):
    cfg = lq.Config.from_workload(configs.TINY_GDN, n_hp_rows=2)
    need = lq.lq_workspace_bytes(cfg)
    fake_ws, fake_s0 = 0x7f0000000000, 0x7f1000000000
    assert _init(L, cfg, fake_ws, need, fake_s0, None) == lq.LQ_ERR_INVALID_ARG
    dup = (C.c_int32 * 4)(1, 1, 2, 3)
    assert _init(L, cfg, fake_ws, need, fake_s0, dup) == lq.LQ_ERR_INVALID_ARG
    oob = (C.c_int32 * 4)(1, 64, 2, 3)
    assert _init(L, cfg, fake_ws, need, fake_s0, oob) == lq.LQ_ERR_INVALID_ARG
    neg = (C.c_int32 * 4)(-1, 5, 2, 3)
    assert _init(L, cfg, fake_ws, need, fake_s0, neg) == lq.LQ_ERR_INVALID_ARG


def test_null_handles_and_pointers(L):
    assert L.lq_decode_step(None, *([C.c_void_p(16)] * 6), None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_window_flush(None, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_state_export_fp32(None, C.c_void_p(16), None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_get_status(None, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_selftest_wait(None, 1000000, None) == lq.LQ_ERR_INVALID_ARG
    fake = C.c_void_p(0x7f0000000000)    # never dereferenced: the limit is checked first
    assert L.lq_selftest_wait(fake, 999, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_selftest_wait(fake, 2000000000, None) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_state_buffered(None) == 0
    assert L.lq_state_set_phases(None, None, None) == lq.LQ_ERR_INVALID_ARG
    L.lq_state_destroy(None)
    cfg = lq.Config.from_workload(configs.TINY_GDN)
    view = lq.lq_qstate_view(None, None, None, None, None, None)
    assert L.lq_quantize_state(C.byref(cfg.c()), C.c_void_p(256), None, C.byref(view), None) \
        == lq.LQ_ERR_INVALID_ARG
    assert L.lq_damp_select(C.byref(cfg.c()), 0, C.c_void_p(256), 1, C.c_void_p(256), C.c_void_p(256),
                            C.c_void_p(256), None) == lq.LQ_ERR_INVALID_ARG


def test_strerror_covers_every_status(L):
    for code in range(-8, 1):
        assert lq.strerror(code) != "unknown status"
    assert lq.strerror(-99) == "unknown status"


def test_effective_bits_per_state_value():
    # payload: codes + BF16 rows; total: + FP32 m, s and r compensators
    # (8 (dk-P) + 16 P) / dk and 32 (dk + dv)(1 + r) / (dk dv)
    from quantized_recurrent_state_lq_b200 import traffic
    b = traffic.bits_per_value(configs.GDN_DAMP)          # P = 16 of 128 rows, r = 2
    assert b["payload"] == pytest.approx(9.0) and b["total"] == pytest.approx(10.5)
    b = traffic.bits_per_value(configs.GDN_PREFIX_CACHE)  # r = 4
    assert b["payload"] == pytest.approx(8.0) and b["total"] == pytest.approx(10.5)
    b = traffic.bits_per_value(configs.TINY_GDN)          # d = 64, r = 2
    assert b["payload"] == pytest.approx(8.0) and b["total"] == pytest.approx(11.0)


def test_bf16_buffer_config(L):
    cfg = lq.Config.from_workload(configs.GDN_PREFIX_CACHE)
    full = lq.lq_workspace_bytes(cfg)
    cfg.buffer_bf16 = 1
    assert lq.lq_config_check(cfg) == lq.LQ_OK
    lean = lq.lq_workspace_bytes(cfg)
    # the W buffered tokens take half the bytes
    wl = configs.GDN_PREFIX_CACHE
    saved = wl.heads * wl.W * (wl.dk + wl.dv) * 2
    assert full - lean == pytest.approx(saved, rel=0.01)
    cfg.buffer_bf16 = 2
    assert lq.lq_config_check(cfg) == lq.LQ_ERR_INVALID_ARG
    for mode in ("fp32", "step"):
        c2 = lq.Config.from_workload(configs.GDN_PREFIX_CACHE, mode=mode)
        c2.buffer_bf16 = 1
        assert lq.lq_config_check(c2) == lq.LQ_ERR_INVALID_ARG


def test_bf16_buffer_with_bf16_rows_is_not_built(L):
    cfg = lq.Config.from_workload(configs.GDN_DAMP)      # P = 16 BF16 rows
    cfg.buffer_bf16 = 1
    assert lq.lq_config_check(cfg) == lq.LQ_ERR_UNSUPPORTED


def test_bf16_buffer_traffic_model():
    # the window buffer's bytes halve; everything else is unchanged
    from quantized_recurrent_state_lq_b200 import traffic
    wl = configs.GDN_PREFIX_CACHE
    lean = wl.with_(buffer_bf16=1)
    assert traffic.token_entry_bytes(lean) * 2 == traffic.token_entry_bytes(wl) == 4 * (wl.dk + wl.dv)
    n = 10
    d = traffic.decode_launch_bytes(wl, n) - traffic.decode_launch_bytes(lean, n)
    assert d == (n + 1) * 2 * (wl.dk + wl.dv)     # n entries read + one appended


def test_state_bits_config(L):
    base = lq.Config.from_workload(configs.GDN_PREFIX_CACHE)
    full = lq.lq_workspace_bytes(base)
    wl = configs.GDN_PREFIX_CACHE
    for bits, code_bytes in ((8, 1.0), (6, 0.75), (4, 0.5)):
        for mode in ("window", "step"):
            c = lq.Config.from_workload(wl.with_(bits=bits), mode=mode)
            assert c.state_bits == bits
            assert lq.lq_config_check(c) == lq.LQ_OK
        c = lq.Config.from_workload(wl.with_(bits=bits))
        # the codes shrink to bits / 8 bytes each; nothing else changes (records
        # are 128-byte aligned)
        saved = wl.heads * wl.dk * wl.dv * (1 - code_bytes)
        assert full - lq.lq_workspace_bytes(c) == pytest.approx(saved, abs=wl.heads * 128)
    zero = lq.Config.from_workload(wl)
    zero.state_bits = 0                                   # reads as 8
    assert lq.lq_config_check(zero) == lq.LQ_OK and lq.lq_workspace_bytes(zero) == full
    for bad in (1, 2, 3, 5, 7, 9, 16, -4):
        c = lq.Config.from_workload(wl)
        c.state_bits = bad
        assert lq.lq_config_check(c) == lq.LQ_ERR_INVALID_ARG
    f = lq.Config.from_workload(wl, mode="fp32")
    f.state_bits = 4
    assert lq.lq_config_check(f) == lq.LQ_ERR_INVALID_ARG


def test_packed_codes_with_bf16_rows_are_not_built(L):
    cfg = lq.Config.from_workload(configs.GDN_DAMP)       # P = 16 BF16 rows
    for bits in (6, 4):
        cfg.state_bits = bits
        assert lq.lq_config_check(cfg) == lq.LQ_ERR_UNSUPPORTED


def test_low_bit_traffic_and_bits_per_value():
    from quantized_recurrent_state_lq_b200 import traffic
    wl = configs.GDN_PREFIX_CACHE                          # d = 128, r = 4
    for bits in (6, 4):
        lb = wl.with_(bits=bits)
        assert traffic.state_bytes(wl) - traffic.state_bytes(lb) == wl.dk * wl.dv * (8 - bits) // 8
        b = traffic.bits_per_value(lb)
        assert b["payload"] == pytest.approx(bits)
        assert b["total"] == pytest.approx(bits + 2.5)     # 32 * 256 * 5 / 16384


def test_prefill_argument_checks(L):
    """lq_prefill validates on the host and launches nothing on error."""
    cfg = lq.Config(B=2, H=4, Hk=2, dk=128, dv=128, gate="kda", mode="fp32", r=0)
    p = C.c_void_p(256)
    args = lambda T=8, q=p, out=p, **kw: (C.byref(kw.get("c", cfg).c()), C.c_int32(T), q, p, p, p, p, None,
                                          out, None, None)
    assert L.lq_prefill(*args(T=-1)) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_prefill(*args(T=(1 << 30) + 1)) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_prefill(*args(out=None)) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_prefill(*args(q=None)) == lq.LQ_ERR_INVALID_ARG
    assert L.lq_prefill(*args(q=C.c_void_p(258))) == lq.LQ_ERR_INVALID_ARG     # not 4-byte aligned
    for bad, code in ((dict(dk=96), lq.LQ_ERR_UNSUPPORTED), (dict(Hk=3), lq.LQ_ERR_SHAPE),
                      (dict(B=0), lq.LQ_ERR_SHAPE), (dict(H=2, Hk=4), lq.LQ_ERR_SHAPE)):
        c2 = lq.Config(**{**cfg.__dict__, **bad})
        assert L.lq_prefill(*args(c=c2)) == code, bad
    assert L.lq_prefill(None, C.c_int32(1), p, p, p, p, p, None, p, None, None) == lq.LQ_ERR_INVALID_ARG


def test_prefill_flops_model():
    """Arithmetic of the chunked prefill per head and chunk (the ALU roofline's
    numerator): the three dk x dv products dominate."""
    from quantized_recurrent_state_lq_b200 import traffic
    wl = configs.KDA_B256
    f = traffic.prefill_flops(wl, 2048)
    C16 = 16
    big = 3 * 2 * C16 * wl.dk * wl.dv * (2048 // C16)
    assert big < f < 1.25 * big
    g = traffic.prefill_flops(configs.GDN_PREFIX_CACHE, 2048)
    assert g < f                                  # KDA's per-channel pair decays cost more


def test_static_scales_config(L):
    wl = configs.KDA_B256
    c = lq.Config.from_workload(wl, smoothing=2)
    assert lq.lq_config_check(c) == lq.LQ_OK
    base = lq.lq_workspace_bytes(lq.Config.from_workload(wl))
    # the [H][dk+dv] table of fixed scales, 256-byte aligned
    assert lq.lq_workspace_bytes(c) - base == (wl.H * (wl.dk + wl.dv) * 4 + 255) // 256 * 256
    f = lq.Config.from_workload(wl, mode="fp32", smoothing=2)
    assert lq.lq_config_check(f) == lq.LQ_ERR_INVALID_ARG
    d = lq.Config.from_workload(configs.GDN_DAMP, smoothing=2)
    assert lq.lq_config_check(d) == lq.LQ_ERR_UNSUPPORTED          # no BF16 rows with fixed scales
    # the state init needs the scales, the static init needs smoothing 2
    h = C.c_void_p()
    p = C.c_void_p(256)
    assert L.lq_state_init(C.byref(h), C.byref(c.c()), p, C.c_size_t(1 << 40), p, None, None) == \
        lq.LQ_ERR_INVALID_ARG
    c1 = lq.Config.from_workload(wl)
    assert L.lq_state_init_static(C.byref(h), C.byref(c1.c()), p, C.c_size_t(1 << 40), p, p, p, None) == \
        lq.LQ_ERR_INVALID_ARG
    assert L.lq_state_init_static(C.byref(h), C.byref(c.c()), p, C.c_size_t(1 << 40), p, None, p, None) == \
        lq.LQ_ERR_INVALID_ARG
    # the stateless quantizer has no scale arguments
    assert L.lq_quantize_state(C.byref(c.c()), p, None, None, None) in (lq.LQ_ERR_INVALID_ARG,
                                                                      lq.LQ_ERR_UNSUPPORTED)
    # the fit's argument checks
    fit = lambda cfg, n, ng, g: L.lq_fit_static_scales(C.byref(cfg.c()), C.c_int32(n), p, C.c_int32(ng), g, p, p,
                                                       None)
    assert fit(c, 0, 0, None) == lq.LQ_ERR_INVALID_ARG
    assert fit(c, 4, 8, C.c_void_p(258)) == lq.LQ_ERR_INVALID_ARG      # misaligned decays
    assert fit(c, 4, 0, p) == lq.LQ_ERR_INVALID_ARG                    # decays without samples
    assert fit(d, 4, 0, None) == lq.LQ_ERR_UNSUPPORTED


def test_profiled_source_hash_ignores_comments_only():
    """The traffic figure of the ncu record is tied to the profiled kernel's
    code: a comment or blank-line edit keeps the hash, a code edit changes it."""
    import bench
    code = "int f(int x) {\n    return x + 1;  // add one\n}\n/* block\n comment */\n"
    same = "// header\nint f(int x) {\n\n    return x + 1;\n}\n"
    other = "int f(int x) {\n    return x + 2;\n}\n"
    assert bench._code_only(code) == bench._code_only(same)
    assert bench._code_only(code) != bench._code_only(other)


def test_binding_constants_match_the_header():
    """Every #define and enum value of include/lq_state.h that the binding
    mirrors has the header's value, and lq_config has the header's fields in
    the header's order."""
    text = open(HEADER).read()
    for name, val in re.findall(r"#define (LQ_[A-Z_]+) (\d+)", text):
        if hasattr(lq, name):
            assert getattr(lq, name) == int(val), name
    for name, val in re.findall(r"\b(LQ_[A-Z_]+)\s*=\s*(-?\d+)", text):
        if hasattr(lq, name):
            assert getattr(lq, name) == int(val), name
    body = re.search(r"typedef struct \{(.*?)\} lq_config;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = [f.strip() for decl in re.findall(r"int32_t ([^;]+);", body) for f in decl.split(",")]
    assert fields == [n for n, _ in lq.lq_config._fields_]


def test_static_quantize_checks_match_the_allocating_call(L):
    """lq_quantize_state_static returns the same status as lq_quantize_state
    for the same bad arguments (its checks run in the same order), before any
    device access; fake device addresses are never touched."""
    base = lq.Config.from_workload(configs.GDN_SERVING)
    good_view = lq.lq_qstate_view(*([C.c_void_p(0x7f0000000000)] * 6))
    bad_view = lq.lq_qstate_view(None, None, None, None, None, None)
    S = C.c_void_p(0x7f1000000000)
    cases = []
    c = lq.Config(**base.__dict__)
    c.smoothing = 2
    cases += [(c, bad_view, S), (c, good_view, S)]
    c = lq.Config(**base.__dict__)
    cases += [(c, bad_view, S), (c, good_view, C.c_void_p(0x7f1000000004)), (c, good_view, None)]
    c = lq.Config(**base.__dict__)
    c.dk = 96
    cases += [(c, good_view, S)]
    c = lq.Config(**base.__dict__)
    c.B = 0
    cases += [(c, good_view, S)]
    for cfg, view, s in cases:
        a = L.lq_quantize_state(C.byref(cfg.c()), s, None, C.byref(view), None)
        b = L.lq_quantize_state_static(C.byref(cfg.c()), s, None, C.byref(view), None)
        assert a == b != lq.LQ_OK, (cfg.__dict__, a, b)
