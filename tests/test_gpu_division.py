"""The codec's division routine (one correctly rounded reciprocal per divisor
and Markstein's FMA correction step, IEEE division near the subnormal range)
must agree bit for bit with IEEE round-to-nearest division: the smoothed
residual x = R / m and the code argument x / s decide INT8 codes, which are
compared with the oracle's IEEE quotients.

Operands: seeded float32 bit patterns over every exponent (subnormals
included), with all-ones and all-zero mantissas over-represented, zeros, and
a block shaped like the codec's own operands (|x| <= sqrt(128), divisors
near the RMS / amax/127 of such values)."""
import numpy as np
import pytest
import torch

from quantized_recurrent_state_lq_b200 import lq


def _operands(n_pairs: int, seed: int):
    rng = np.random.default_rng(seed)
    n = 2 * n_pairs

    def floats(count, exp_lo, exp_hi):
        e = rng.integers(exp_lo, exp_hi + 1, count)
        m = rng.integers(0, 1 << 23, count, dtype=np.uint32)
        sel = rng.random(count)
        m[sel < 0.1] = (1 << 23) - 1
        m[(sel >= 0.1) & (sel < 0.2)] = 0
        u = np.where(e >= -126, ((e + 127).astype(np.uint32) << 23) | m,
                     m >> np.minimum(-126 - e, 31).astype(np.uint32))
        return u.astype(np.uint32).view(np.float32)

    a = floats(n, -149, 127)
    a[rng.random(n) < 0.5] *= -1
    a[rng.random(n) < 0.01] = 0.0
    b = floats(n_pairs, -149, 127)
    b[b == 0] = 1.0
    # codec-shaped block: x up to sqrt(128) in size, divisors around 1 / scales
    k = n // 4
    a[:k] = (rng.standard_normal(k) * 3).astype(np.float32)
    b[: k // 2] = np.abs(rng.standard_normal(k // 2) * 0.05 + 0.09).astype(np.float32) + np.float32(1e-3)
    b = np.repeat(b, 2)            # pairs share the divisor
    return a, b


@pytest.mark.gpu
@pytest.mark.parametrize("seed", [0, 1])
def test_division_routine_is_ieee(seed):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    a, b = _operands(1 << 22, seed)
    da, db = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    fast, pair, ieee = lq.lq_selftest_division(da, db)
    torch.cuda.synchronize()
    fast, pair, ieee = (t.cpu().numpy().view(np.uint32) for t in (fast, pair, ieee))
    with np.errstate(all="ignore"):
        ref = (a / b).astype(np.float32).view(np.uint32)    # numpy: IEEE float32 division
    assert np.array_equal(ieee, ref), "device IEEE division differs from float32 division"
    assert np.array_equal(fast, ref), f"{int((fast != ref).sum())} quotients differ"
    assert np.array_equal(pair, ref), f"{int((pair != ref).sum())} paired quotients differ"


def test_division_selftest_rejects_odd_length():
    assert lq.lib().lq_selftest_division(None, None, None, None, None, 3, None) == lq.LQ_ERR_INVALID_ARG
