"""Pins for the oracle's number codecs, checked against things other than the oracle.

E2M1: the OCP MX FP4 value table (tests/golden/e2m1_grid.txt) and an independent
per-binade rounding built on numpy's round-half-even. E4M3: torch's float8_e4m3fn
conversion (a library routine) plus saturation closed forms. fp16: numpy's fp64->fp16
cast. exp/silu: math.exp in fp64 within an ulp bound.
"""
import math
import os
import struct

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------------------- E2M1

def test_e2m1_decode_matches_ocp_table(orc):
    rows = _read_table("e2m1_grid.txt")
    assert len(rows) == 16
    for code_s, value_s in rows:
        code = int(code_s, 16)
        v = orc.e2m1_value(code)
        want = float(value_s)
        assert v == want and math.copysign(1.0, v) == math.copysign(1.0, want), (code, v, want)


def _e2m1_by_binade(y: np.ndarray) -> np.ndarray:
    """Independent E2M1 rounding: the grid has spacing 0.5 on [0,2), 1 on [2,4), 2 on [4,6];
    numpy's rint is round-half-even, and within each binade the multiple's parity is the
    code's parity, so half-even on the multiple is ties-to-even-code. Saturate at 6."""
    a = np.abs(y.astype(np.float64))
    val = np.where(a < 2, np.rint(a * 2) / 2, np.where(a < 4, np.rint(a), 2 * np.rint(a / 2)))
    val = np.minimum(val, 6.0)
    val = np.where(np.isinf(a), 6.0, val)
    table = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    mag = np.vectorize(table.__getitem__, otypes=[np.uint8])(val)
    return (mag | (np.signbit(y).astype(np.uint8) << 3)).astype(np.uint8)


def test_e2m1_encode_dense_sweep(orc):
    # every fp32 multiple of 2^-20 in [-8, 8]: all midpoints, both sides of each, and the
    # saturation region
    y = (np.arange(-(8 << 20), (8 << 20) + 1, dtype=np.int64) * 2.0 ** -20).astype(np.float32)
    got = orc.e2m1_encode(y)
    want = _e2m1_by_binade(y)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (y[bad[:10]], got[bad[:10]], want[bad[:10]])


def test_e2m1_encode_specials(orc):
    y = np.array([0.0, -0.0, 1e-30, -1e-30, 6.0, 6.0000005, 7.0, 1e30, np.inf, -np.inf,
                  np.float32(np.nextafter(np.float32(0.25), np.float32(1))),
                  np.float32(np.nextafter(np.float32(0.25), np.float32(0)))], np.float32)
    got = orc.e2m1_encode(y)
    want = [0x0, 0x8, 0x0, 0x8, 0x7, 0x7, 0x7, 0x7, 0x7, 0xF, 0x1, 0x0]
    assert list(got) == want


def test_e2m1_ties_golden(orc):
    rows = _read_table("e2m1_ties.txt")
    y = np.array([float(r[0]) for r in rows], np.float32)
    want = np.array([int(r[1], 16) for r in rows], np.uint8)
    assert (orc.e2m1_encode(y) == want).all()


def test_e2m1_roundtrip(orc):
    for c in range(16):
        v = orc.e2m1_value(c)
        assert orc.e2m1_encode(np.float32(v))[0] == c


# ------------------------------------------------------------------------------- E4M3

def test_e4m3_decode_all_codes_vs_torch(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    for c in range(256):
        v = orc.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(v), c
        else:
            assert v == float(ref[c]), (c, v, ref[c])
    assert orc.e4m3_value(0x7E) == 448.0


def _e4m3_probe_values():
    vals = [np.float32(0.0)]
    # all E4M3 values, midpoints between neighbours and the fp32 values next to those
    dec = sorted({orc_v for orc_v in _all_e4m3_values()})
    for a, b in zip(dec[:-1], dec[1:]):
        mid = np.float32((a + b) / 2)
        vals += [np.float32(a), mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9))]
    # a strided sweep over fp32 bit patterns from 2^-40 to just below 464
    lo = np.float32(2.0 ** -40).view(np.uint32)
    hi = np.float32(464.0).view(np.uint32)
    vals = np.concatenate([np.array(vals, np.float32),
                           np.arange(lo, hi, 61, dtype=np.uint32).view(np.float32)])
    return vals[vals < 464.0]


def _all_e4m3_values():
    import oracle
    return [oracle.e4m3_value(c) for c in range(0x7F)]


def test_e4m3_encode_vs_torch(orc):
    s = _e4m3_probe_values()
    got = orc.e4m3_encode(s)
    ref = torch.from_numpy(s).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (s[bad[:8]], got[bad[:8]], ref[bad[:8]])


def test_e4m3_saturation_closed_forms(orc):
    s = np.array([448.0, 448.0 * (1 + 2 ** -4), 463.99, 464.0, 480.0, 1e30, np.inf,
                  2.0 ** -10, 1.5 * 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -9, 2.0 ** -6], np.float32)
    want = [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x00, 0x01, 0x02, 0x01, 0x08]
    assert list(orc.e4m3_encode(s)) == want


def test_e4m3_roundtrip(orc):
    for c in range(0x7F):
        assert orc.e4m3_encode(np.float32(orc.e4m3_value(c)))[0] == c


# ------------------------------------------------------------------------------- fp16 / bf16

def test_f64_to_f16_vs_numpy(orc):
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(200000) * 10.0 ** rng.integers(-9, 6, 200000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e9, 2.0 ** -24, 2.0 ** -25,
                  1.5 * 2.0 ** -25, 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25,
                  1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 1 + 2.0 ** -11 + 2.0 ** -40]),
    ])
    # exact ties of every binade
    for e in range(-14, 16):
        v = np.append(v, (2.0 ** e) * (1 + 2.0 ** -11 * np.arange(1, 40, 2)))
    got = orc.f64_to_f16(v)
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:8]], got[bad[:8]], want[bad[:8]])
    assert orc.f64_to_f16(1 + 2.0 ** -11 + 2.0 ** -40)[0] == struct.unpack("<H", struct.pack("<e", 1 + 2.0 ** -10))[0]


def test_f16_to_f32_all_patterns(orc):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = orc.f16_to_f32(h)
    want = h.view(np.float16).astype(np.float32)
    same = (got.view(np.uint32) == want.view(np.uint32)) | (np.isnan(got) & np.isnan(want))
    assert same.all()


def test_bf16_to_f32_vs_torch(orc):
    h = np.arange(0, 65536, 7, dtype=np.uint32).astype(np.uint16)
    want = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    L = orc.lib()
    got = np.array([L.orc_bf16_to_f32(int(x)) for x in h], np.float32)
    same = (got.view(np.uint32) == want.view(np.uint32)) | (np.isnan(got) & np.isnan(want))
    assert same.all()


# ------------------------------------------------------------------------------- exp / silu

def _ulp32(x):
    x = np.abs(np.float32(x))
    return np.float64(np.nextafter(x, np.float32(np.inf))) - np.float64(x)


def test_exp_within_two_ulp(orc):
    x = np.linspace(-87.0, 88.0, 400001, dtype=np.float32)
    x = np.concatenate([x, np.float32(np.random.default_rng(1).uniform(-10, 10, 200000))])
    got = orc.exp32(x).astype(np.float64)
    want = np.exp(x.astype(np.float64))
    ulps = np.abs(got - want) / np.vectorize(_ulp32)(want.astype(np.float32))
    assert ulps.max() <= 2.0, (ulps.max(), x[np.argmax(ulps)])


def test_exp_special_points(orc):
    assert orc.exp32(0.0)[0] == 1.0
    assert orc.exp32(-100.0)[0] == orc.exp32(-87.0)[0]
    assert orc.exp32(100.0)[0] == orc.exp32(88.0)[0]
    assert np.isfinite(orc.exp32(88.0)[0])
    # e(1) close to Euler's number
    assert abs(float(orc.exp32(1.0)[0]) - math.e) <= 2 * float(_ulp32(np.float32(math.e)))


def test_silu_limits_and_accuracy(orc):
    assert orc.silu32(0.0)[0] == 0.0
    big = np.array([20.0, 50.0, 1e4], np.float32)
    assert (orc.silu32(big) == big).all()
    assert np.abs(orc.silu32(np.array([-30.0, -60.0], np.float32))).max() < 1e-11
    x = np.linspace(-20, 20, 100001, dtype=np.float32)
    got = orc.silu32(x).astype(np.float64)
    xd = x.astype(np.float64)
    want = xd / (1.0 + np.exp(-xd))
    rel = np.abs(got - want) / np.maximum(np.abs(want), 1e-30)
    assert rel.max() < 5e-7, rel.max()
