"""Pins for the oracle's quantize path: hand-derived blocks, closed forms and invariants."""
import os

import numpy as np
import pytest
import torch

from nvfp4_block_scaled_10_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FLT_MAX = float(np.finfo(np.float32).max)


def _worked_blocks():
    out = []
    with open(os.path.join(GOLDEN, "quant_worked_blocks.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            name, g, xs, s, qs = [p.strip() for p in line.split("|")]
            out.append((name, float(g), [float(v) for v in xs.split()], int(s, 16),
                        [int(v, 16) for v in qs.split()]))
    return out


@pytest.mark.parametrize("case", _worked_blocks(), ids=lambda c: c[0])
def test_worked_blocks(orc, case):
    name, g, xs, s_want, q_want = case
    s, q = orc.quantize_block(np.array(xs, np.float32), g)
    assert s == s_want, name
    assert list(q) == q_want, name


def test_packing_low_nibble_first(orc):
    # element 0 -> low nibble of byte 0, element 1 -> high nibble (6 encodes as 0x7)
    x = torch.zeros(1, 16, dtype=torch.bfloat16)
    x[0, 0] = 6.0
    q, sf, _ = orc.quantize(workloads.bits16(x), g=1.0)
    assert q[0, 0] == 0x07 and sf[0, 0] == 0x38
    x = torch.zeros(1, 16, dtype=torch.bfloat16)
    x[0, 1] = 6.0
    q, _, _ = orc.quantize(workloads.bits16(x), g=1.0)
    assert q[0, 0] == 0x70


def test_global_scale_closed_form(orc):
    assert orc.global_scale_from_amax(0.0) == 1.0
    assert orc.global_scale_from_amax(6.0) == 448.0
    assert orc.global_scale_from_amax(2688.0) == 1.0
    for amax in [0.37, 1.0, 3.14159, 50.0 * 4.1, 1e-3]:
        assert orc.global_scale_from_amax(amax) == float(np.float32(2688.0) / np.float32(amax))
    assert orc.global_scale_from_amax(1e-37) == FLT_MAX


def _dequant(q, sf, g):
    """Independent dequantization: E2M1 grid (golden table) and torch's E4M3 decode."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])
    lo = grid[q & 0xF]
    hi = grid[q >> 4]
    vals = np.stack([lo, hi], axis=-1).reshape(q.shape[0], -1)
    s = torch.from_numpy(sf.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    g = np.asarray(g, np.float64).reshape(-1, 1) if np.size(g) > 1 else np.float64(np.asarray(g).reshape(-1)[0])
    return vals * np.repeat(s, 16, axis=1) / g, np.repeat(s, 16, axis=1)


def _check_error_bound(x, q, sf, g):
    xhat, sdec = _dequant(q, sf, g)
    gg = np.asarray(g, np.float64).reshape(-1, 1) if np.size(g) > 1 else np.float64(np.asarray(g).reshape(-1)[0])
    d = sdec / gg  # dequant factor per element
    y = np.where(d > 0, x / np.where(d > 0, d, 1), 0.0)  # x in E2M1 units
    grid_q = np.abs(xhat / np.where(d > 0, d, 1))
    gap = np.where(grid_q < 2, 0.5, np.where(grid_q < 4, 1.0, 2.0))
    # a value that rounds down into a smaller binade sits within half of that binade's gap
    gap_below = np.where(grid_q <= 2, 0.5, np.where(grid_q <= 4, 1.0, 2.0))
    gap = np.maximum(gap, gap_below)
    err = np.abs(y - np.where(d > 0, grid_q * np.sign(xhat + 0.0), 0.0))
    sat = np.abs(y) > 6.0
    bound = np.where(sat, np.abs(y) - 6.0, gap / 2) + 1e-5 * np.abs(y) + 1e-12
    ok = (err <= bound) | (d == 0)
    assert ok.all(), (x[~ok][:5], xhat[~ok][:5])
    # saturation is bounded by the E4M3 rounding of the block scale (normal range: 2^-4)
    normal = sdec >= 2.0 ** -6
    assert (np.abs(y)[normal] <= 6.0 * (1 + 2.0 ** -4) * (1 + 1e-6)).all()


def test_error_bound_and_scale_invariant_per_tensor(orc):
    x = workloads.with_outliers((64, 512), seed=11)
    xb = workloads.bits16(x)
    g = orc.global_scale(xb)
    q, sf, _ = orc.quantize(xb, g=g)
    # the block holding the tensor's amax gets the largest finite block scale
    assert sf.max() == 0x7E
    _check_error_bound(x.to(torch.float64).numpy(), q, sf, g)


def test_per_token_scales_and_invariant(orc):
    x = workloads.with_outliers((48, 1024), seed=12)
    xb = workloads.bits16(x)
    q, sf, g = orc.quantize(xb, per_token=True)
    xf = x.to(torch.float32).numpy()
    row_amax = np.abs(xf).max(axis=1)
    want_g = np.float32(2688.0) / row_amax.astype(np.float32)
    assert (g.view(np.uint32) == want_g.view(np.uint32)).all()
    assert (sf.max(axis=1) == 0x7E).all()
    _check_error_bound(x.to(torch.float64).numpy(), q, sf, g)


def test_zero_row_per_token(orc):
    x = torch.zeros(2, 32, dtype=torch.bfloat16)
    x[1, 3] = -2.0
    q, sf, g = orc.quantize(workloads.bits16(x), per_token=True)
    assert g[0] == 1.0 and (sf[0] == 0).all() and (q[0] == 0).all()
    assert g[1] == np.float32(1344.0) and sf[1, 0] == 0x7E


def test_exactly_representable_roundtrip(orc):
    # grid values times 2^-2 with a block amax of 1.5: scale 0.25 is exact, r = 4, q exact
    rng = np.random.default_rng(3)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    vals = rng.choice(grid, size=(8, 64)) * rng.choice([-1, 1], size=(8, 64)) * 0.25
    vals[:, ::16] = 1.5
    x = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16)
    q, sf, _ = orc.quantize(workloads.bits16(x), g=1.0)
    xhat, _ = _dequant(q, sf, 1.0)
    assert (sf == 0x28).all()
    assert np.array_equal(xhat, vals)


def test_fp16_and_bf16_inputs_agree_on_shared_values(orc):
    rng = np.random.default_rng(4)
    v = (rng.integers(-64, 64, size=(4, 64)) / 8.0).astype(np.float32)  # exact in both
    xb = workloads.bits16(torch.from_numpy(v).to(torch.bfloat16))
    xh = workloads.bits16(torch.from_numpy(v).to(torch.float16))
    a = orc.quantize(xb, orc.BF16, g=3.0)
    b = orc.quantize(xh, orc.FP16, g=3.0)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_swiglu_saturated_gate_reduces_to_product(orc):
    # gate >= 20: e(-gate) < 2^-28 so 1 + e(-gate) == 1 and silu(gate) == gate exactly;
    # Y is then the plain fp32 product gate * up, quantized as any tensor
    rng = np.random.default_rng(5)
    gate = rng.uniform(20, 40, size=(4, 64)).astype(np.float32)
    up = rng.standard_normal((4, 64)).astype(np.float32)
    gb = torch.from_numpy(gate).to(torch.bfloat16)
    ub = torch.from_numpy(up).to(torch.bfloat16)
    xs = workloads.bits16(torch.cat([gb, ub], dim=1))
    y = (gb.to(torch.float32) * ub.to(torch.float32)).numpy()
    assert np.array_equal(orc.swiglu(xs), y)
    g = 2.5
    q1, s1 = orc.swiglu_quantize(xs, g)
    for r in range(4):
        for b in range(4):
            s, codes = orc.quantize_block(y[r, 16 * b:16 * b + 16], g)
            assert s == s1[r, b]
            packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
            assert np.array_equal(packed, q1[r, 8 * b:8 * b + 8])


def test_swiglu_zero_gate(orc):
    x = torch.zeros(1, 64, dtype=torch.bfloat16)
    x[0, 32:] = 3.0  # up = 3, gate = 0 -> y = 0
    assert (orc.swiglu(workloads.bits16(x)) == 0).all()
    q, s = orc.swiglu_quantize(workloads.bits16(x), 1.0)
    assert (q == 0).all() and (s == 0).all()


# ------------------------------------------------------------------------------ SwiGLU + FP8


def _e4m3_decode(codes):
    """Value of signed E4M3 codes (OCP OFP8: bias 7, subnormals at exponent 0, 0x7F NaN)."""
    c = np.asarray(codes, np.int64)
    e, m = (c >> 3) & 15, c & 7
    mag = np.where(e > 0, (1.0 + m / 8.0) * 2.0 ** (e - 7.0), (m / 8.0) * 2.0 ** -6)
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return np.where(c & 0x80, -mag, mag)


def test_e4m3_signed_encoder(orc):
    v = np.float32(np.concatenate([np.linspace(0, 470, 20001), [1e-9, 0.0019, 2 ** -9, 1e30, np.inf]]))
    pos = orc.e4m3_encode_signed(v)
    assert np.array_equal(pos, orc.e4m3_encode(v))                   # magnitudes: the scale encoder
    neg = orc.e4m3_encode_signed(-v)
    assert np.array_equal(neg, pos | 0x80)                            # sign bit, -0 included
    assert orc.e4m3_encode_signed(np.float32(np.nan))[0] == 0x7F
    # against torch's float8_e4m3fn cast (round to nearest even) where no saturation applies
    import torch
    w = np.float32(np.random.default_rng(3).uniform(-463, 463, 50000))
    t = torch.from_numpy(w).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(orc.e4m3_encode_signed(w), t)


def test_swiglu_fp8_bounds_and_saturation(orc):
    """q = E4M3_sat(y * scale): decode(q) is within half an E4M3 step of y * scale below 448,
    exactly +-448 at or above, and the sign of y is kept (zero included)."""
    from nvfp4_block_scaled_10_b200 import workloads
    x = workloads.swiglu(8, 64, seed=9)
    bits = workloads.bits16(x)
    for scale in (1.0, 37.0, 900.0):
        q = orc.swiglu_fp8(bits, scale)
        y = orc.swiglu(bits).astype(np.float64)
        t = np.float32(y * scale).astype(np.float64)  # one fp32 product, as defined
        d = _e4m3_decode(q)
        big = np.abs(t) >= 448
        assert np.all(np.abs(d[big]) == 448.0) and np.all(np.sign(d[big]) == np.sign(t[big]))
        small = ~big
        # half a step: the E4M3 spacing at |t| is 2^(floor(log2|t|) - 3), subnormals 2^-9
        ex = np.floor(np.log2(np.maximum(np.abs(t[small]), 2.0 ** -6)))
        half = 2.0 ** (ex - 3) / 2
        assert np.all(np.abs(d[small] - t[small]) <= half + 1e-30)
        assert np.all((q[small] & 0x80 != 0) == np.signbit(t[small]))


def test_swiglu_fp8_traffic_reading(orc):
    """The fused SwiGLU + FP8 call reads X and writes Q only: its input and output buffers add
    up to the fused byte count recomputed from the shapes (5NH), not to the printed 9NH."""
    from nvfp4_block_scaled_10_b200 import workloads
    N, H = 16, 64
    bits = workloads.bits16(workloads.swiglu(N, H, seed=4))
    q = orc.swiglu_fp8(bits, 1.0)
    _, fused = orc.swiglu_quant_traffic_from_shapes(N, H, out="fp8")
    assert bits.nbytes + q.nbytes == fused == 5 * N * H
