"""The oracle's 128x4 and 8x4 scale layouts against FlashInfer's fp4_quantize, the library
routine behind "feature: add fp4 mm using trtllm backend" (FlashInfer PR #1355), which
writes both layouts. FlashInfer quantizes the same input three times (linear, 128x4, 8x4
scales); the oracle's swizzle of FlashInfer's own linear scales must reproduce its swizzled
bytes exactly, padding included. Only the byte permutation is compared, so the two
quantizers' arithmetic does not enter. No kernel of this library runs here.

FlashInfer is part of the GPU image: if it cannot be imported these tests fail (they are
the live form of the layout pin; tests/golden/flashinfer_sf_layouts.txt holds FlashInfer's
bytes for a few ragged shapes so that the pin also holds on the CPU)."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.helpers import require_cuda

pytestmark = pytest.mark.gpu


def _flashinfer():
    try:
        import flashinfer
    except Exception as e:  # a missing library must not turn the pin into a skip
        pytest.fail(f"flashinfer is needed for the layout pin and could not be imported: {e}")
    return flashinfer


@pytest.mark.parametrize("M,K", [(40, 512), (130, 320), (17, 64), (256, 1024)])
def test_scale_layouts_match_flashinfer(M, K):
    require_cuda()
    flashinfer = _flashinfer()
    g = torch.Generator(device="cuda").manual_seed(M * 7 + K)
    # block magnitudes spread over several binades so the scale codes vary
    x = torch.randn(M, K, device="cuda", generator=g) * torch.exp(
        2 * torch.randn(M, K // 16, device="cuda", generator=g)).repeat_interleave(16, dim=1)
    x = x.bfloat16()
    gs = torch.tensor([2688.0 / x.float().abs().max().item()], device="cuda")
    _, lin = flashinfer.fp4_quantize(x, gs, 16, False, is_sf_swizzled_layout=False)
    _, s128 = flashinfer.fp4_quantize(x, gs, 16, False, is_sf_swizzled_layout=True,
                                      is_sf_8x4_layout=False)
    _, s84 = flashinfer.fp4_quantize(x, gs, 16, False, is_sf_swizzled_layout=True,
                                     is_sf_8x4_layout=True)
    torch.cuda.synchronize()
    lin = lin.view(torch.uint8).cpu().numpy().reshape(-1)[:M * (K // 16)].reshape(M, K // 16)
    assert len(np.unique(lin)) >= 8  # enough distinct codes for a permutation to show
    for got, layout in ((s128, orc.L128x4), (s84, orc.L8x4)):
        g_bytes = got.view(torch.uint8).cpu().numpy().reshape(-1)
        want = orc.swizzle(lin, layout)
        assert g_bytes.size == want.size
        assert np.array_equal(g_bytes, want)


def _e2m1_steps(a, b):
    """Distance in E2M1 grid steps between two packed codes' nibbles (same sign required)."""
    out = []
    for x, y in ((a & 0xF, b & 0xF), (a >> 4, b >> 4)):
        same_sign = (x & 8) == (y & 8)
        out.append(np.where(same_sign, np.abs((x & 7).astype(int) - (y & 7).astype(int)), 99))
    return np.maximum(out[0], out[1])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,K,seed", [(64, 1024, 1), (130, 2048, 2), (512, 7168, 3)])
def test_quantize_against_flashinfer(M, K, seed, dtype):
    """The oracle's per-tensor quantize against FlashInfer's fp4_quantize with the same
    encode scale. The E4M3 block scales must agree byte for byte (the scale rule E4M3(amax/6 x
    g) with round-to-nearest and saturation). FlashInfer's default path takes approximate
    reciprocals, so a packed value may land one E2M1 step away where x * r sits at a rounding
    midpoint: fewer than 1% of bytes may differ, by one step, with the same sign."""
    require_cuda()
    flashinfer = _flashinfer()
    from nvfp4_block_scaled_10_b200 import workloads
    x = workloads.per_token(M, K, seed=seed).to(dtype)
    odt = orc.BF16 if dtype == torch.bfloat16 else orc.FP16
    bits = x.view(torch.int16).numpy().view(np.uint16)
    g = orc.global_scale(bits, odt)
    q_o, sf_o, _ = orc.quantize(bits, odt, g=g)
    q_f, sf_f = flashinfer.fp4_quantize(x.cuda(), torch.tensor([g], device="cuda"), 16, False,
                                        is_sf_swizzled_layout=False)
    torch.cuda.synchronize()
    qf = q_f.view(torch.uint8).cpu().numpy().reshape(M, K // 2)
    sff = sf_f.view(torch.uint8).cpu().numpy().reshape(-1)[:M * (K // 16)].reshape(M, K // 16)
    assert np.array_equal(sff, sf_o)
    steps = _e2m1_steps(qf, q_o)
    assert steps.max() <= 1
    assert np.count_nonzero(steps) < 0.01 * qf.size
