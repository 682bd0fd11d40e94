"""Pins for the oracle's scale layouts, its GEMM and the pages' byte counts."""
import os

import numpy as np
import pytest
import torch

from nvfp4_block_scaled_10_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------- layouts

def _pad(s, rmul, cmul):
    R, C = s.shape
    Rp, Cp = -(-R // rmul) * rmul, -(-C // cmul) * cmul
    out = np.zeros((Rp, Cp), np.uint8)
    out[:R, :C] = s
    return out


def _swz128_by_reshape(s):
    """The 128x4 block-scale layout as a reshape/transpose: row = 128a + 32b + c,
    column = 4d + e  ->  byte order [a][d][c][b][e]."""
    p = _pad(s, 128, 4)
    Rp, Cp = p.shape
    return p.reshape(Rp // 128, 4, 32, Cp // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1)


def _swz8_by_reshape(s):
    """The 8x4 layout: row = 8a + b, column = 4c + d  ->  byte order [a][c][b][d]."""
    p = _pad(s, 8, 4)
    Rp, Cp = p.shape
    return p.reshape(Rp // 8, 8, Cp // 4, 4).transpose(0, 2, 1, 3).reshape(-1)


SHAPES = [(1, 1), (16, 32), (128, 4), (130, 7), (300, 33), (8, 448), (33, 512)]


@pytest.mark.parametrize("R,C", SHAPES)
def test_swizzle_128x4_matches_reshape(orc, R, C):
    s = workloads.random_bytes((R, C), seed=R * 1000 + C, low=1, high=255)
    got = orc.swizzle(s, orc.L128x4)
    assert np.array_equal(got, _swz128_by_reshape(s))
    assert np.array_equal(orc.unswizzle(got, R, C, orc.L128x4), s)


@pytest.mark.parametrize("R,C", SHAPES)
def test_swizzle_8x4_matches_reshape(orc, R, C):
    s = workloads.random_bytes((R, C), seed=R * 1000 + C + 7, low=1, high=255)
    got = orc.swizzle(s, orc.L8x4)
    assert np.array_equal(got, _swz8_by_reshape(s))
    assert np.array_equal(orc.unswizzle(got, R, C, orc.L8x4), s)


@pytest.mark.parametrize("layout", [1, 2])
def test_offsets_are_a_bijection_and_padding_is_zero(orc, layout):
    R, C = 131, 9
    nbytes = orc.sf_bytes(layout, R, C)
    Rp = -(-R // (128 if layout == 1 else 8)) * (128 if layout == 1 else 8)
    Cp = -(-C // 4) * 4
    offs = sorted(orc.sf_offset(layout, r, c, R, C) for r in range(Rp) for c in range(Cp))
    assert offs == list(range(nbytes))
    s = np.full((R, C), 0xFF, np.uint8)
    buf = orc.swizzle(s, layout)
    assert int((buf == 0xFF).sum()) == R * C and int((buf == 0).sum()) == nbytes - R * C


def test_sf_bytes_at_workload_shapes(orc):
    assert orc.sf_bytes(orc.L128x4, 16, 512 // 16) == 4096
    assert orc.sf_bytes(orc.L8x4, 16, 512 // 16) == 512
    assert orc.sf_bytes(orc.L128x4, 8192, 7168 // 16) == 3670016
    assert orc.sf_bytes(orc.L128x4, 4096, 14336 // 16) == 3670016
    assert orc.sf_bytes(orc.L128x4, 28672, 8192 // 16) == 14680064
    assert orc.sf_bytes(orc.L8x4, 1, 8192 // 16) == 8 * 512
    assert orc.sf_bytes(orc.L128x4, 1, 8192 // 16) == 128 * 512


# ------------------------------------------------------------------------------- GEMM

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])


def _deq_numpy(q, sf, g):
    vals = np.stack([E2M1[q & 0xF], E2M1[q >> 4]], axis=-1).reshape(q.shape[0], -1)
    s = torch.from_numpy(np.ascontiguousarray(sf)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return vals * np.repeat(s, 16, axis=1) / np.float64(np.float32(g))


def test_gemm_ones_gives_k(orc):
    M, N, K = 3, 5, 256
    a = np.full((M, K // 2), 0x22, np.uint8)  # both nibbles = E2M1 1.0
    w = np.full((N, K // 2), 0x22, np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)  # E4M3 1.0
    sw = np.full((N, K // 16), 0x38, np.uint8)
    for fn in (orc.gemm, orc.gemm_loops):
        out16, out64 = fn(a, sa, 1.0, w, sw, 1.0, want_f64=True)
        assert (out64 == K).all()
        assert (out16.view(np.float16) == K).all()


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (3, 5, 64), (8, 16, 128), (7, 3, 96), (16, 256, 512)])
def test_gemm_loops_brute_force_vs_numpy(orc, M, N, K):
    seed = M * 100 + N * 10 + K
    a = workloads.random_bytes((M, K // 2), seed)
    w = workloads.random_bytes((N, K // 2), seed + 1)
    sa = workloads.random_bytes((M, K // 16), seed + 2, 0x20, 0x50)
    sw = workloads.random_bytes((N, K // 16), seed + 3, 0x20, 0x50)
    ga, gw = 37.5, 1234.0
    out16, out64 = orc.gemm_loops(a, sa, ga, w, sw, gw, want_f64=True)
    want = _deq_numpy(a, sa, ga) @ _deq_numpy(w, sw, gw).T
    np.testing.assert_allclose(out64, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    assert np.array_equal(out16, out64.astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("M,N,K", [(3, 5, 64), (16, 256, 512), (33, 70, 1024)])
def test_gemm_matmul_path_equals_loops(orc, M, N, K):
    # the fast oracle (C dequantize + fp64 matmul) against the plain triple loop
    seed = M * 7 + N * 3 + K
    a = workloads.random_bytes((M, K // 2), seed)
    w = workloads.random_bytes((N, K // 2), seed + 1)
    sa = workloads.random_bytes((M, K // 16), seed + 2, 0x20, 0x50)
    sw = workloads.random_bytes((N, K // 16), seed + 3, 0x20, 0x50)
    l16, l64 = orc.gemm_loops(a, sa, 3.0, w, sw, 700.0, want_f64=True)
    m16, m64 = orc.gemm(a, sa, 3.0, w, sw, 700.0, want_f64=True)
    np.testing.assert_allclose(m64, l64, rtol=1e-12, atol=1e-12 * np.abs(l64).max())
    diff = np.abs(m16.view(np.float16).astype(np.float64) - l16.view(np.float16).astype(np.float64))
    ulp = np.abs(l16.view(np.float16).astype(np.float64)) * 2.0 ** -10 + 2.0 ** -24
    assert (diff <= ulp).all()


def test_dequantize_matches_independent_decode(orc):
    q = workloads.random_bytes((5, 32), 9)
    s = workloads.random_bytes((5, 4), 10, 0, 0x7F)
    assert np.array_equal(orc.dequantize(q, s, 2.5), _deq_numpy(q, s, 2.5))


def test_gemm_is_not_transposed(orc):
    # A row 0 is all 1.0 and W row 1 is all 2.0, everything else zero: only D[0,1] != 0
    K = 64
    a = np.zeros((2, K // 2), np.uint8)
    w = np.zeros((3, K // 2), np.uint8)
    a[0, :] = 0x22
    w[1, :] = 0x44
    s1 = lambda r: np.full((r, K // 16), 0x38, np.uint8)
    want = np.zeros((2, 3), np.float16)
    want[0, 1] = 2 * K
    for fn in (orc.gemm, orc.gemm_loops):
        assert np.array_equal(fn(a, s1(2), 1.0, w, s1(3), 1.0).view(np.float16), want)


def test_gemm_global_scales_divide(orc):
    K = 32
    a = np.full((1, K // 2), 0x22, np.uint8)
    w = np.full((1, K // 2), 0x22, np.uint8)
    s = np.full((1, K // 16), 0x38, np.uint8)
    for fn in (orc.gemm, orc.gemm_loops):
        out16, out64 = fn(a, s, 4.0, w, s, 0.5, want_f64=True)
        assert out64[0, 0] == K / (4.0 * 0.5)


# ------------------------------------------------------------------------------- byte counts

def _traffic_golden():
    vals = {}
    with open(os.path.join(GOLDEN, "swiglu_fp8_traffic.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split()
                vals[k] = float(v)
    return vals


def test_page_byte_counts_follow_from_printed_steps(orc):
    gold = _traffic_golden()
    N, H = 1, 1
    unfused, fused, red = orc.swiglu_quant_traffic_as_printed(N, H)
    assert unfused == gold["unfused_total"] == gold["unfused_read_x"] + gold["unfused_write_y_bf16"] + \
        gold["unfused_read_y_bf16"] + gold["unfused_write_q_fp8"]
    assert fused == gold["fused_total"] == gold["fused_read_x"] + gold["fused_write_q_fp8"]
    assert round(100 * red) == round(100 * 4 / 13) == 31 and int(100 * red) == gold["reduction_percent"]


def test_byte_counts_from_shapes(orc):
    N, H = 4096, 14336
    NH = N * H
    u8, f8 = orc.swiglu_quant_traffic_from_shapes(N, H, "fp8")
    assert (u8, f8) == (9 * NH, 5 * NH)
    u4, f4 = orc.swiglu_quant_traffic_from_shapes(N, H, "nvfp4")
    assert f4 == 4 * NH + NH // 2 + NH // 16 == 267911168
    # the fused SwiGLU + NVFP4 workload moves 4.5625 NH bytes
    assert f4 / NH == 4.5625


def test_gemm_per_row_activation_scales(orc):
    """Per-token activation scales: with every row scale equal it is the scalar GEMM, and
    otherwise output row m is the unit-scale GEMM's row divided by g[m] (the scale factors
    out of the sum, so the fp64 results agree to rounding)."""
    rng = np.random.default_rng(11)
    M, N, K = 6, 40, 96
    a = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    w = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(0x28, 0x48, (M, K // 16), dtype=np.uint8)
    sw = rng.integers(0x28, 0x48, (N, K // 16), dtype=np.uint8)
    g_rows = np.array([0.5, 3.0, 17.25, 1.0, 250.0, 0.125], np.float32)
    same = np.full(M, 7.5, np.float32)
    _, ref_same = orc.gemm(a, sa, 7.5, w, sw, 2.0, want_f64=True)
    _, got_same = orc.gemm(a, sa, same, w, sw, 2.0, want_f64=True)
    np.testing.assert_array_equal(got_same, ref_same)
    _, unit = orc.gemm(a, sa, 1.0, w, sw, 2.0, want_f64=True)
    _, rows = orc.gemm(a, sa, g_rows, w, sw, 2.0, want_f64=True)
    np.testing.assert_allclose(rows, unit / g_rows[:, None].astype(np.float64), rtol=1e-12, atol=0)
    # and against the triple loop, one row at a time with that row's scalar scale
    for m in range(M):
        _, loop_m = orc.gemm_loops(a[m:m + 1], sa[m:m + 1], float(g_rows[m]), w, sw, 2.0,
                                   want_f64=True)
        np.testing.assert_allclose(rows[m:m + 1], loop_m, rtol=1e-12, atol=1e-300)


def _e4m3_values(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def test_gemm_act_f32_equals_scalar_contract_for_product_scales(orc):
    """fp32 activation scales that are E4M3 scale / g exactly (g a power of two) and a weight
    scale 1 / gw give the scalar-contract GEMM bit for bit: the two contracts name the same
    real numbers then."""
    rng = np.random.default_rng(21)
    M, N, K = 5, 24, 128
    a = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    w = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(0x08, 0x7F, (M, K // 16), dtype=np.uint8)
    sw = rng.integers(0x20, 0x60, (N, K // 16), dtype=np.uint8)
    ga, gw = 64.0, 0.25
    sa32 = (_e4m3_values(sa) / ga).astype(np.float32)
    assert np.array_equal(sa32.astype(np.float64) * ga, _e4m3_values(sa))  # exact
    ref16, ref64 = orc.gemm(a, sa, ga, w, sw, gw, want_f64=True)
    got16, got64 = orc.gemm_act_f32(a, sa32, w, sw, 1.0 / gw, want_f64=True)
    np.testing.assert_array_equal(got64, ref64)
    np.testing.assert_array_equal(got16, ref16)
    # the [B,1,K/16] shape of the plugin reads the same
    np.testing.assert_array_equal(orc.gemm_act_f32(a, sa32.reshape(M, 1, K // 16), w, sw, 4.0), ref16)


def test_gemm_act_f32_brute_force_exact(orc):
    """Against an exact rational sum (fractions) of the defining products, on a tiny case
    with fp32 scales spread over many binades; the weight scale multiplies."""
    from fractions import Fraction
    rng = np.random.default_rng(5)
    M, N, K = 3, 4, 64
    a = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    w = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sw = rng.integers(0x10, 0x70, (N, K // 16), dtype=np.uint8)
    sa32 = np.float32(2.0 ** rng.uniform(-20, 20, (M, K // 16)) * rng.uniform(1, 2, (M, K // 16)))
    w_scale = np.float32(0.0037)
    e2m1 = lambda b: E2M1[b]  # noqa: E731
    swv = _e4m3_values(sw)
    got16, got64 = orc.gemm_act_f32(a, sa32, w, sw, w_scale, want_f64=True)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                av = e2m1((a[m, k // 2] >> (4 * (k % 2))) & 0xF)
                wv = e2m1((w[n, k // 2] >> (4 * (k % 2))) & 0xF)
                acc += (Fraction(float(av)) * Fraction(float(sa32[m, k // 16])) * Fraction(float(wv))
                        * Fraction(float(swv[n, k // 16])) * Fraction(float(w_scale)))
            exact = float(acc)
            assert abs(got64[m, n] - exact) <= 1e-13 * max(abs(exact), 1e-300)
            assert got16[m, n] == np.float16(exact).view(np.uint16)


def test_gemm_act_f32_weight_scale_multiplies(orc):
    rng = np.random.default_rng(8)
    M, N, K = 2, 8, 64
    a = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    w = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sw = rng.integers(0x20, 0x60, (N, K // 16), dtype=np.uint8)
    sa32 = np.float32(rng.uniform(0.01, 3.0, (M, K // 16)))
    _, one = orc.gemm_act_f32(a, sa32, w, sw, 1.0, want_f64=True)
    _, three = orc.gemm_act_f32(a, sa32, w, sw, 3.0, want_f64=True)
    _, eighth = orc.gemm_act_f32(a, sa32, w, sw, 0.125, want_f64=True)
    np.testing.assert_allclose(three, 3.0 * one, rtol=1e-15, atol=0)
    np.testing.assert_array_equal(eighth, one / 8.0)


def test_gemm_row_parallel_reading(orc):
    """tp = 1 is the GEMM itself; for tp = 2 and 4 the unrounded shard sums add up to the
    full GEMM's fp64 sum (the shards partition K exactly) and the result is the full GEMM's
    value to within the extra fp16 roundings of the partials."""
    rng = np.random.default_rng(40)
    M, N, K = 5, 24, 512
    a = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    w = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(0x28, 0x48, (M, K // 16), dtype=np.uint8)
    sw = rng.integers(0x28, 0x48, (N, K // 16), dtype=np.uint8)
    full16, full64 = orc.gemm(a, sa, 2.0, w, sw, 30.0, want_f64=True)
    one16, one64 = orc.gemm_row_parallel(a, sa, 2.0, w, sw, 30.0, tp=1, want_f64=True)
    np.testing.assert_array_equal(one16, full16)
    np.testing.assert_array_equal(one64, full64)
    for t in (2, 4):
        o16, o64 = orc.gemm_row_parallel(a, sa, 2.0, w, sw, 30.0, tp=t, want_f64=True)
        np.testing.assert_allclose(o64, full64, rtol=1e-12, atol=1e-12 * np.abs(full64).max())
        got = o16.view(np.float16).astype(np.float64)
        # t partial roundings and one final rounding, each at most half an fp16 ulp
        bound = (t + 1) * 2.0 ** -11 * (np.abs(full64) + np.abs(full64).max() * 2.0 ** -4)
        assert np.all(np.abs(got - full64) <= bound)
    with pytest.raises(AssertionError):
        orc.gemm_row_parallel(a[:, :96], sa[:, :12], 2.0, w[:, :96], sw[:, :12], 30.0, tp=2)


def test_gemm_row_parallel_rounds_each_rank(orc):
    """Each rank's output is rounded to fp16 before the AllReduce adds it ("Fused Nvfp4 GEMM
    All Reduce Plugin": rank-local FP16 [B,N] output, then the AllReduce). A hand-built case
    where that rounding decides the result, M = N = 1, K = 128, tp = 2, unit global scales:
      rank 0 (K 0..63):   1*1 (scales 1) + 0.5*0.5 (scales 2^-4, 2^-4)           = 1 + 2^-10
      rank 1 (K 64..127): 1*1 + 0.5*0.5 (2^-4, 2^-4) + 0.5*0.5 (2^-4, 2^-5)
                          + 0.5*0.5 (2^-5, 2^-5)                  = 1 + 7*2^-12 -> fp16 1 + 2^-9
    The fp16 partials add to 2 + 3*2^-10, halfway between fp16 2 + 2^-9 and 2 + 2^-8, which
    rounds to the even 2 + 2^-8 (0x4002). Adding the unrounded partials instead gives
    2 + 11*2^-12, which rounds to 2 + 2^-9 (0x4001)."""
    one, half = 0x2, 0x1                                # E2M1 codes of 1.0 and 0.5
    s1, s4, s5 = 0x38, 0x18, 0x10                       # E4M3 codes of 1, 2^-4, 2^-5
    codes_a, codes_w = np.zeros(128, np.uint8), np.zeros(128, np.uint8)
    sa, sw = np.full((1, 8), s1, np.uint8), np.full((1, 8), s1, np.uint8)
    for blk, (ca, cw, xa, xw) in {0: (one, one, s1, s1), 1: (half, half, s4, s4),
                                  4: (one, one, s1, s1), 5: (half, half, s4, s4),
                                  6: (half, half, s4, s5), 7: (half, half, s5, s5)}.items():
        codes_a[16 * blk], codes_w[16 * blk] = ca, cw
        sa[0, blk], sw[0, blk] = xa, xw
    pack = lambda c: (c[0::2] | (c[1::2] << 4)).astype(np.uint8).reshape(1, 64)  # noqa: E731
    a, w = pack(codes_a), pack(codes_w)
    out16, sum64 = orc.gemm_row_parallel(a, sa, 1.0, w, sw, 1.0, tp=2, want_f64=True)
    assert sum64[0, 0] == 2 + 11 * 2.0 ** -12
    assert out16[0, 0] == 0x4002
    assert orc.gemm(a, sa, 1.0, w, sw, 1.0)[0, 0] == 0x4001   # the one-rank GEMM of the same data


def test_flashinfer_sf_layout_bytes(orc):
    """The 128x4 and 8x4 layouts pinned to FlashInfer's own bytes on the CPU: for each shape
    in tests/golden/flashinfer_sf_layouts.txt (written on a GPU by
    tests/golden/make_flashinfer_sf_layouts.py, which runs only FlashInfer's fp4_quantize,
    the routine of "feature: add fp4 mm using trtllm backend" that introduced both layouts),
    the oracle's swizzle of FlashInfer's linear scales must give FlashInfer's 128x4 and 8x4
    buffers byte for byte, padding included. Shapes have ragged rows and, for K = 96,
    ragged scale columns."""
    path = os.path.join(os.path.dirname(__file__), "golden", "flashinfer_sf_layouts.txt")
    lines = [ln.strip() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    shapes = 0
    ragged_cols = False
    while lines:
        head, lin_hex, s128_hex, s84_hex = lines[:4]
        lines = lines[4:]
        _, M, K = head.split()
        M, K = int(M), int(K)
        C = K // 16
        lin = np.frombuffer(bytes.fromhex(lin_hex), np.uint8).reshape(M, C)
        assert len(np.unique(lin)) >= 8
        for hx, layout in ((s128_hex, orc.L128x4), (s84_hex, orc.L8x4)):
            want = np.frombuffer(bytes.fromhex(hx), np.uint8)
            got = orc.swizzle(lin, layout)
            assert got.size == want.size, (M, K, layout, got.size, want.size)
            assert np.array_equal(got, want), (M, K, layout)
        shapes += 1
        ragged_cols |= C % 4 != 0
    assert shapes >= 2 and ragged_cols
