"""GPU parity of the quantize kernels against the oracle: bit-exact bytes.

Small shapes span several CTAs, ragged tails and every layout; the full per-token and
SwiGLU workloads are compared in full. Outputs carry canary guard bands (helpers.Guarded)
that must be untouched after each launch."""
import numpy as np
import pytest
import torch

import oracle as orc
from nvfp4_block_scaled_10_b200 import workloads
from tests.helpers import (Guarded, assert_bytes_equal, check_guards, guarded, host_bytes,
                           require_cuda, to_dev_bits)

pytestmark = pytest.mark.gpu

DT = {"bf16": (torch.bfloat16, orc.BF16), "fp16": (torch.float16, orc.FP16)}


def _inputs(M, K, pad, seed, dtype):
    x = workloads.with_outliers((M, K + pad), seed=seed, dtype=DT[dtype][0])
    return x


def _quantize_both(nv, xt, dtype, per_token, layout, K):
    """Runs GPU and oracle on the same bits (x may have a row stride > K)."""
    tdt, odt = DT[dtype]
    xs = xt[:, :K]
    bits = workloads.bits16(xs.contiguous())
    M = xs.shape[0]
    xd = xt.cuda()[:, :K]
    if per_token:
        gg = guarded((M,), torch.float32)
        q_o, sf_o, g_o = orc.quantize(bits, odt, per_token=True)
    else:
        g = orc.global_scale(bits, odt)
        gg = guarded((1,), torch.float32)
        gg.view(torch.float32).fill_(g)
        q_o, sf_o, g_o = orc.quantize(bits, odt, g=g)
    gsf = Guarded(nv.nvfp4_sf_bytes(M, K, layout))
    gq = guarded((M, K // 2))
    g_dev, q_dev, sf_dev = gg.view(torch.float32), gq.view(torch.uint8, (M, K // 2)), gsf.view()
    nv.nvfp4_quantize(xd, g_dev, per_token=per_token, sf_layout=layout, q=q_dev, sf=sf_dev)
    torch.cuda.synchronize()
    check_guards(q=gq, sf=gsf, g=gg)
    assert_bytes_equal(host_bytes(q_dev), q_o, "q")
    assert_bytes_equal(host_bytes(sf_dev), orc.swizzle(sf_o, layout), "sf")
    if per_token:
        assert_bytes_equal(host_bytes(g_dev), g_o.view(np.uint8), "g")


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("layout", [0, 1, 2])
@pytest.mark.parametrize("M,K,pad", [(1, 16, 0), (3, 48, 8), (17, 512, 0), (130, 1040, 16),
                                     (257, 64, 0), (300, 7168, 0)])
def test_quantize_parity_small(M, K, pad, layout, per_token, dtype):
    nv = require_cuda()
    xt = _inputs(M, K, pad, seed=M * 31 + K, dtype=dtype)
    _quantize_both(nv, xt, dtype, per_token, layout, K)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("M,K,pad", [(1300, 4096, 8), (700, 16384, 0), (350, 20480, 8),
                                     (40, 32768, 0), (9, 32784, 0)])
def test_quantize_per_token_row_shapes(M, K, pad, dtype):
    # every register-resident row shape (1, 2, 4, 8 blocks per thread; 128 and 256 threads),
    # more rows than resident CTAs so rows roll through the registers, rows whose stride is
    # not a multiple of 32 bytes, and the first K past the register path (two-pass)
    nv = require_cuda()
    xt = _inputs(M, K, pad, seed=M + 7 * K, dtype=dtype)
    _quantize_both(nv, xt, dtype, True, 1, K)


def test_quantize_per_token_long_rows_two_pass():
    # rows of 65536 elements (128 KB) do not fit twice in shared memory: two-pass path
    nv = require_cuda()
    xt = _inputs(3, 65536, 0, seed=5, dtype="bf16")
    _quantize_both(nv, xt, "bf16", True, 1, 65536)


def test_quantize_worked_blocks_and_edges():
    nv = require_cuda()
    # hand-derived blocks (ties, saturation after scale rounding, zeros, -0) as GPU input
    rows = []
    with open(__file__.replace("test_quantize_gpu.py", "golden/quant_worked_blocks.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                parts = [p.strip() for p in line.split("|")]
                rows.append((float(parts[1]), [float(v) for v in parts[2].split()]))
    for g, xs in rows:
        x = torch.tensor([xs], dtype=torch.float32).to(torch.bfloat16)
        bits = workloads.bits16(x)
        q_o, sf_o, _ = orc.quantize(bits, orc.BF16, g=g)
        q, sf, _ = nv.nvfp4_quantize(x.cuda(), torch.tensor([g], device="cuda"),
                                     sf_layout=nv.SF_LINEAR)
        torch.cuda.synchronize()
        assert_bytes_equal(host_bytes(q), q_o, f"q g={g} {xs}")
        assert_bytes_equal(host_bytes(sf), sf_o, f"sf g={g} {xs}")
    # tiny negatives (-> -0 codes), exact zeros, a huge g (scale overflow -> saturation)
    x = torch.tensor([[-1e-3, -0.0, 0.0, 1e-3] * 4, [65000.0] + [-1e-30] * 15],
                     dtype=torch.float32).to(torch.bfloat16)
    for g in [1.0, 2688.0, 3.0e38]:
        bits = workloads.bits16(x)
        q_o, sf_o, _ = orc.quantize(bits, orc.BF16, g=g)
        q, sf, _ = nv.nvfp4_quantize(x.cuda(), torch.tensor([g], device="cuda"),
                                     sf_layout=nv.SF_LINEAR)
        torch.cuda.synchronize()
        assert_bytes_equal(host_bytes(q), q_o, f"q g={g}")
        assert_bytes_equal(host_bytes(sf), sf_o, f"sf g={g}")


def test_quantize_empty_is_noop():
    nv = require_cuda()
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    q, sf, g = nv.nvfp4_quantize(x, per_token=True)
    assert q.numel() == 0 and g.numel() == 0


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("M,K,pad", [(1, 16, 0), (16, 512, 0), (256, 512, 0), (77, 1040, 24),
                                     (1000, 4096, 0)])
def test_global_scale_parity(M, K, pad, dtype):
    nv = require_cuda()
    xt = _inputs(M, K, pad, seed=M + K + pad, dtype=dtype)
    bits = workloads.bits16(xt[:, :K].contiguous())
    g_o = orc.global_scale(bits, DT[dtype][1])
    gg = guarded((1,), torch.float32)
    gws = Guarded(max(nv.nvfp4_global_scale_workspace_bytes(M, K), 16))
    g = nv.nvfp4_global_scale(xt.cuda()[:, :K], g_out=gg.view(torch.float32), workspace=gws.view())
    torch.cuda.synchronize()
    check_guards(g=gg, workspace=gws)
    assert g.item() == g_o


def test_global_scale_zero_tensor():
    nv = require_cuda()
    g = nv.nvfp4_global_scale(torch.zeros(5, 32, dtype=torch.bfloat16, device="cuda"))
    assert g.item() == 1.0


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("layout", [0, 1, 2])
@pytest.mark.parametrize("M,H,pad", [(1, 16, 0), (5, 48, 8), (33, 512, 0), (130, 1024, 16),
                                     (64, 14336, 0)])
def test_swiglu_parity_small(M, H, pad, layout, dtype):
    nv = require_cuda()
    tdt, odt = DT[dtype]
    xt = workloads.normal((M, 2 * H + pad), 1.0, seed=M * 13 + H, dtype=tdt)
    xs = xt[:, :2 * H].contiguous()
    bits = workloads.bits16(xs)
    g = orc.global_scale_from_amax(orc.swiglu_amax(bits, odt))
    q_o, sf_o = orc.swiglu_quantize(bits, g, odt)
    gsf = Guarded(nv.nvfp4_sf_bytes(M, H, layout))
    gq = guarded((M, H // 2))
    q, sf = nv.swiglu_nvfp4_quantize(xt.cuda()[:, :2 * H], torch.tensor([g], device="cuda"),
                                     sf_layout=layout, q=gq.view(torch.uint8, (M, H // 2)),
                                     sf=gsf.view())
    torch.cuda.synchronize()
    check_guards(q=gq, sf=gsf)
    assert_bytes_equal(host_bytes(q), q_o, "q")
    assert_bytes_equal(host_bytes(sf), orc.swizzle(sf_o, layout), "sf")


def test_swiglu_extreme_gates():
    nv = require_cuda()
    # gates far outside the exp clamp range and around zero
    gate = torch.tensor([[-200.0, -90.0, -88.5, -87.5, -20.0, -1e-3, 0.0, 1e-3, 0.5, 1.0,
                          20.0, 87.0, 88.5, 200.0, -5.0, 5.0]], dtype=torch.float32)
    up = torch.linspace(-3, 3, 16).reshape(1, 16)
    x = torch.cat([gate, up], dim=1).to(torch.bfloat16)
    bits = workloads.bits16(x)
    for g in [1.0, 100.0]:
        q_o, sf_o = orc.swiglu_quantize(bits, g, orc.BF16)
        q, sf = nv.swiglu_nvfp4_quantize(x.cuda(), torch.tensor([g], device="cuda"),
                                         sf_layout=nv.SF_LINEAR)
        torch.cuda.synchronize()
        assert_bytes_equal(host_bytes(q), q_o, "q")
        assert_bytes_equal(host_bytes(sf), sf_o, "sf")


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_swiglu_infinite_and_signed_zero_gates(dtype):
    # blocks holding an infinite gate take the kernel's exact-special-value quotient; the
    # neighbouring blocks (finite gates, -0 among them) take the form without it
    nv = require_cuda()
    tdt, odt = DT[dtype]
    inf = float("inf")
    gate = torch.tensor([[inf, -inf, -0.0, 0.0, 1.5, -2.0, 3.0, -0.25, 7.0, -7.0, 0.5, 1.0,
                          -1.0, 2.0, -3.0, 4.0] + [-0.0, 0.0, 0.125, -0.125] * 4,
                         [-inf] + [0.5] * 15 + [inf] + [-0.5] * 15], dtype=torch.float32)
    up = torch.linspace(0.5, 3.0, 32).reshape(1, 32).repeat(2, 1)
    x = torch.cat([gate, up], dim=1).to(tdt)
    bits = workloads.bits16(x)
    for g in [1.0, 37.5]:
        q_o, sf_o = orc.swiglu_quantize(bits, g, odt)
        q, sf = nv.swiglu_nvfp4_quantize(x.cuda(), torch.tensor([g], device="cuda"),
                                         sf_layout=nv.SF_LINEAR)
        torch.cuda.synchronize()
        assert_bytes_equal(host_bytes(q), q_o, "q")
        assert_bytes_equal(host_bytes(sf), sf_o, "sf")


@pytest.mark.parametrize("layout", [0, 1, 2])
@pytest.mark.parametrize("R,C", [(1, 1), (130, 7), (300, 33), (28672, 512)])
def test_swizzle_unswizzle_parity(R, C, layout):
    nv = require_cuda()
    lin = workloads.random_bytes((R, C), seed=R + C + layout, low=1, high=255)
    want = orc.swizzle(lin, layout)
    gout = Guarded(want.size)
    gback = guarded((R, C))
    got = nv.nvfp4_sf_swizzle(torch.from_numpy(lin).cuda(), layout, out=gout.view())
    back = nv.nvfp4_sf_unswizzle(got, R, C, layout, out=gback.view(torch.uint8, (R, C)))
    torch.cuda.synchronize()
    check_guards(swizzled=gout, unswizzled=gback)
    assert_bytes_equal(host_bytes(got), want, "swizzle")
    assert_bytes_equal(host_bytes(back), lin, "unswizzle")


# ------------------------------------------------------------------------------ full size

def test_per_token_workload_full():
    """[8192, 7168] bf16 with 0.1% x50 outliers, per-token g, 128x4 scales: every byte."""
    nv = require_cuda()
    x = workloads.per_token()
    M, K = x.shape
    bits = workloads.bits16(x)
    q_o, sf_o, g_o = orc.quantize(bits, orc.BF16, per_token=True)
    gq, gsf, gg = guarded((M, K // 2)), Guarded(nv.nvfp4_sf_bytes(M, K, nv.SF_128x4)), guarded((M,), torch.float32)
    q, sf, g = nv.nvfp4_quantize(x.cuda(), gg.view(torch.float32), per_token=True,
                                 sf_layout=nv.SF_128x4, q=gq.view(torch.uint8, (M, K // 2)),
                                 sf=gsf.view())
    torch.cuda.synchronize()
    check_guards(q=gq, sf=gsf, g=gg)
    assert_bytes_equal(host_bytes(g), g_o.view(np.uint8), "g")
    assert_bytes_equal(host_bytes(q), q_o, "q")
    assert_bytes_equal(host_bytes(sf), orc.swizzle(sf_o, orc.L128x4), "sf")


def test_swiglu_workload_full():
    """[4096, 2 x 14336] bf16, per-tensor g from amax(Y) by the oracle, 128x4: every byte."""
    nv = require_cuda()
    x = workloads.swiglu()
    M, H = x.shape[0], x.shape[1] // 2
    bits = workloads.bits16(x)
    g = orc.global_scale_from_amax(orc.swiglu_amax(bits, orc.BF16))
    q_o, sf_o = orc.swiglu_quantize(bits, g, orc.BF16)
    gq, gsf = guarded((M, H // 2)), Guarded(nv.nvfp4_sf_bytes(M, H, nv.SF_128x4))
    q, sf = nv.swiglu_nvfp4_quantize(x.cuda(), torch.tensor([g], device="cuda"),
                                     sf_layout=nv.SF_128x4, q=gq.view(torch.uint8, (M, H // 2)),
                                     sf=gsf.view())
    torch.cuda.synchronize()
    check_guards(q=gq, sf=gsf)
    assert_bytes_equal(host_bytes(q), q_o, "q")
    assert_bytes_equal(host_bytes(sf), orc.swizzle(sf_o, orc.L128x4), "sf")


def test_tiny_workload_quantize():
    """A [16,512] and W [256,512], per-tensor g from the GPU amax kernel, both layouts."""
    nv = require_cuda()
    a, w = workloads.tiny()
    for t in (a, w):
        bits = workloads.bits16(t)
        g_o = orc.global_scale(bits, orc.BF16)
        g = nv.nvfp4_global_scale(t.cuda())
        torch.cuda.synchronize()
        assert g.item() == g_o
        q_o, sf_o, _ = orc.quantize(bits, orc.BF16, g=g_o)
        for layout in (nv.SF_128x4, nv.SF_8x4):
            q, sf, _ = nv.nvfp4_quantize(t.cuda(), g, sf_layout=layout)
            torch.cuda.synchronize()
            assert_bytes_equal(host_bytes(q), q_o, "q")
            assert_bytes_equal(host_bytes(sf), orc.swizzle(sf_o, layout), "sf")


# ------------------------------------------------------------------------------ SwiGLU + FP8


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("M,H,pad,scale", [(1, 16, 0, 1.0), (5, 48, 8, 37.0), (130, 1040, 16, 3.0),
                                           (64, 14336, 0, 448.0 / 60.0), (3, 512, 0, 5000.0)])
def test_swiglu_fp8_parity(M, H, pad, scale, dtype):
    nv = require_cuda()
    tdt, odt = DT[dtype]
    x = workloads.normal((M, 2 * H + pad), 1.0, seed=M + H, dtype=tdt)
    xs = x[:, :2 * H].contiguous()
    q_o = orc.swiglu_fp8(workloads.bits16(xs), scale, odt)
    gq = guarded((M, H))
    q = nv.swiglu_fp8_quantize(x.cuda()[:, :2 * H], torch.tensor([scale], device="cuda"),
                               q=gq.view(torch.uint8, (M, H)))
    torch.cuda.synchronize()
    check_guards(q=gq)
    assert_bytes_equal(host_bytes(q), q_o, "q")


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_swiglu_fp8_special_values(dtype):
    # infinite gates and ups (saturation to +-448), NaN (0x7F), signed zeros, tiny values
    nv = require_cuda()
    tdt, odt = DT[dtype]
    inf, nan = float("inf"), float("nan")
    gate = torch.tensor([[inf, -inf, -0.0, 0.0, 1.5, -2.0, 3e-5, -3e-5, 7.0, -7.0, 60.0, 1.0,
                          nan, 2.0, -3.0, 4.0]], dtype=torch.float32)
    up = torch.tensor([[2.0, 2.0, 1.0, -1.0, inf, -inf, 1.0, 1.0, 1e4, 1e4, -100.0, nan,
                        1.0, 0.0, -0.0, 0.5]], dtype=torch.float32)
    x = torch.cat([gate, up], dim=1).to(tdt)
    for scale in [1.0, 10.0]:
        q_o = orc.swiglu_fp8(workloads.bits16(x), scale, odt)
        q = nv.swiglu_fp8_quantize(x.cuda(), torch.tensor([scale], device="cuda"))
        torch.cuda.synchronize()
        assert_bytes_equal(host_bytes(q), q_o, "q")


def test_swiglu_fp8_workload_full():
    nv = require_cuda()
    x = workloads.swiglu(4096, 14336)
    scale = 448.0 / 60.0
    q_o = orc.swiglu_fp8(workloads.bits16(x), scale, orc.BF16)
    gq = guarded((4096, 14336))
    q = nv.swiglu_fp8_quantize(x.cuda(), torch.tensor([scale], device="cuda"),
                               q=gq.view(torch.uint8, (4096, 14336)))
    torch.cuda.synchronize()
    check_guards(q=gq)
    assert_bytes_equal(host_bytes(q), q_o, "q")


@pytest.mark.parametrize("up_value", [1.0, 3.0])
def test_swiglu_every_bf16_gate(up_value):
    """Every one of the 65536 bf16 gate patterns (in order, 16 consecutive patterns per block,
    so each block lies inside or outside the kernels' SiLU table range as a whole, and the
    blocks around 2^-26 and 2^7 and the zero, subnormal, infinite and NaN patterns take the
    per-element path) through both fused SwiGLU kernels, bit-exact against the oracle. The
    FP8 output (scale 1) keeps about four significant bits of each silu(gate) * up, so a
    table entry taken for a neighbouring gate shows up here."""
    nv = require_cuda()
    gates = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(64, 1024)
    up = np.full((64, 1024), np.float32(up_value)).view(np.uint32) >> 16
    bits = np.concatenate([gates, up.astype(np.uint16)], axis=1)
    x = to_dev_bits(bits, torch.bfloat16)
    # the NVFP4 encoding has no NaN; NaN gates (covered by the FP8 output below) become zeros
    nan = ((gates & 0x7F80) == 0x7F80) & ((gates & 0x7F) != 0)
    bits_nv = np.concatenate([np.where(nan, 0, gates).astype(np.uint16), up.astype(np.uint16)], axis=1)
    x_nv = to_dev_bits(bits_nv, torch.bfloat16)
    for g in [1.0, 448.0 * 6.0 / 128.0]:
        q_o, sf_o = orc.swiglu_quantize(bits_nv, g, orc.BF16)
        q, sf = nv.swiglu_nvfp4_quantize(x_nv, torch.tensor([g], device="cuda"), sf_layout=nv.SF_LINEAR)
        torch.cuda.synchronize()
        assert_bytes_equal(host_bytes(q), q_o, f"swiglu nvfp4 q g={g}")
        assert_bytes_equal(host_bytes(sf), sf_o, f"swiglu nvfp4 sf g={g}")
    for scale in [1.0, 0.5]:
        f_o = orc.swiglu_fp8(bits, scale, orc.BF16)
        f = nv.swiglu_fp8_quantize(x, torch.tensor([scale], device="cuda"))
        torch.cuda.synchronize()
        assert_bytes_equal(host_bytes(f), f_o, f"swiglu fp8 scale={scale}")
