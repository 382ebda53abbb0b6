"""CPU pins of the bit-packed 6- and 4-bit code layout the kernels use
(lq_common.cuh: nib_off, pair_off, lowbit_kslot, chunk_swz), compiled for the
host from the library's own header:

* the nibble plane and the pair plane are each covered exactly once, at the
  alignment of the word that holds a group;
* 8 consecutive columns read with one shared-memory matrix load hit 8
  different 16-byte bank groups;
* the tensor-core GEMV of the buffering step -- an emulation of `ldmatrix.x4`
  and `mma.sync m16n8k32` (s8) fragments over the packed planes, unpacked to
  bytes c * 2^(8-b) as the kernel does, against digits placed by lowbit_kslot
  -- equals the exact dot products of the codes for every column.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    if not os.path.exists(NVCC) and not shutil.which("nvcc"):
        pytest.skip("nvcc not available")
    exe = str(tmp_path_factory.mktemp("layout") / "layout_host")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O1",
                    "-I" + os.path.join(ROOT, "include"), os.path.join(HERE, "layout_host.cu"), "-o", exe],
                   check=True)

    def tables(dk, dv):
        out = subprocess.run([exe, str(dk), str(dv)], check=True, capture_output=True, text=True).stdout
        t = {}
        for line in out.splitlines():
            key, *vals = line.split()
            t[key] = np.array([int(v) for v in vals])
        t["nib"] = t["nib"].reshape(dv, dk // 8)
        t["pair"] = t["pair"].reshape(dv, dk // 8)
        t["swz"] = t["swz"].reshape(dv, 2)
        return t
    return tables


SHAPES = [(128, 128), (64, 64), (64, 128), (128, 64)]


@pytest.mark.parametrize("dk,dv", SHAPES)
def test_planes_covered_once_and_aligned(probe, dk, dv):
    t = probe(dk, dv)
    assert sorted(t["nib"].ravel()) == list(range(0, dv * dk // 2, 4))
    assert sorted(t["pair"].ravel()) == list(range(dv * dk // 2, dv * dk // 2 + dv * dk // 4, 2))
    assert sorted(t["kslot"]) == list(range(dk))


@pytest.mark.parametrize("dk,dv", SHAPES)
def test_matrix_loads_free_of_bank_conflicts(probe, dk, dv):
    t = probe(dk, dv)
    for plane, rb in ((0, dk // 2), (1, dk // 4)):
        nch = rb // 16
        for c0 in range(0, dv, 8):
            for ch in range(nch):
                addr = [c * rb + 16 * (ch ^ t["swz"][c, plane]) for c in range(c0, c0 + 8)]
                groups = {(a % 128) // 16 for a in addr}
                assert len(groups) == min(8, 128 // 16), (plane, c0, ch, addr)


def _pack(codes, t, dk, dv, bits):
    buf = np.zeros(dv * dk * bits // 8, np.uint8)
    for c in range(dv):
        for g in range(dk // 8):
            nw = pw = 0
            for k in range(8):
                v = int(codes[8 * g + k, c]) & 0xFF
                nw |= (v & 15) << (4 * k)
                pw |= ((v >> 4) & 3) << (2 * k)
            o = t["nib"][c, g]
            buf[o:o + 4] = np.frombuffer(np.uint32(nw).tobytes(), np.uint8)
            if bits == 6:
                o = t["pair"][c, g]
                buf[o:o + 2] = np.frombuffer(np.uint16(pw).tobytes(), np.uint8)
    return buf


def _u32(buf, o):
    return int(np.frombuffer(buf[o:o + 4].tobytes(), np.uint32)[0])


def _perm(x, sel):
    b = list(np.uint32(x).tobytes()) + [0, 0, 0, 0]
    return sum(b[(sel >> (4 * j)) & 7] << (8 * j) for j in range(4))


def _unpack(bits, nib, pr):
    if bits == 4:
        return (nib << 4) & 0xF0F0F0F0, nib & 0xF0F0F0F0
    lo = ((nib << 2) & 0x3C3C3C3C) | ((pr << 6) & 0x00C000C0) | ((pr << 2) & 0xC000C000)
    hi = ((nib >> 2) & 0x3C3C3C3C) | ((pr << 4) & 0x00C000C0) | (pr & 0xC000C000)
    return lo & 0xFFFFFFFF, hi & 0xFFFFFFFF


def _bytes(w):
    return np.frombuffer(np.uint32(w).tobytes(), np.int8).astype(np.int64)


def _ldmatrix(buf, addrs, nmat):
    """Lane T receives, from matrix m, bytes 4 (T % 4) .. +3 of the row whose
    address lane 8 m + T / 4 gave."""
    return [[_u32(buf, addrs[8 * m + T // 4] + 4 * (T % 4)) for m in range(nmat)] for T in range(32)]


def _gemv(buf, t, dig, dk, dv, bits):
    slot = np.zeros(dk, np.int64)
    slot[t["kslot"]] = dig                 # the digit of key row i sits at k-slot kslot(i)
    nb, pb = dk // 2, dk // 4
    y = np.zeros(dv, np.int64)
    for c0 in range(0, dv, 16):
        col = [c0 + ((ln >> 3) & 1) * 8 + (ln & 7) for ln in range(32)]
        blk = [ln >> 4 for ln in range(32)]
        pr = [[0, 0, 0, 0] for _ in range(32)]
        if bits == 6:
            base = dv * nb
            if dk >= 128:
                pr = _ldmatrix(buf, [base + col[ln] * pb + ((blk[ln] ^ t["swz"][col[ln], 1]) << 4)
                                     for ln in range(32)], 4)
            else:
                two = _ldmatrix(buf, [base + col[ln] * pb for ln in range(32)], 2)
                pr = [r + [0, 0] for r in two]
        acc = np.zeros((32, 2), np.int64)
        for kp in range(dk // 64):
            x = _ldmatrix(buf, [col[ln] * nb + (((2 * kp + blk[ln]) ^ t["swz"][col[ln], 0]) << 4)
                                for ln in range(32)], 4)
            for hf in range(2):
                ks = 2 * kp + hf
                for T in range(32):
                    tq = T & 3
                    sel = 0x3322 if hf else 0x1100
                    pa = _perm(pr[T][2 * kp], sel) if bits == 6 else 0
                    pb_ = _perm(pr[T][2 * kp + 1], sel) if bits == 6 else 0
                    l0, h0 = _unpack(bits, x[T][2 * hf], pa)
                    l1, h1 = _unpack(bits, x[T][2 * hf + 1], pb_)
                    b0 = slot[32 * ks + 4 * tq: 32 * ks + 4 * tq + 4]
                    b1 = slot[32 * ks + 16 + 4 * tq: 32 * ks + 16 + 4 * tq + 4]
                    acc[T, 0] += int((_bytes(l0) * b0).sum() + (_bytes(h0) * b1).sum())
                    acc[T, 1] += int((_bytes(l1) * b0).sum() + (_bytes(h1) * b1).sum())
        for T in range(32):
            y[c0 + (T >> 2)] += acc[T, 0]
            y[c0 + (T >> 2) + 8] += acc[T, 1]
    return y


@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64)])
def test_tensor_core_gemv_of_packed_codes(probe, bits, dk, dv):
    t = probe(dk, dv)
    rng = np.random.default_rng(bits * 100 + dk)
    q = (1 << (bits - 1)) - 1
    codes = rng.integers(-q, q + 1, (dk, dv))
    dig = rng.integers(-128, 128, dk)
    y = _gemv(_pack(codes, t, dk, dv, bits), t, dig, dk, dv, bits)
    np.testing.assert_array_equal(y, (codes * dig[:, None]).sum(axis=0) << (8 - bits))
