"""The oracle's 128x4 and 8x4 scale layouts against FlashInfer's fp4_quantize, the library
routine behind "feature: add fp4 mm using trtllm backend" (FlashInfer PR #1355), which
writes both layouts. FlashInfer quantizes the same input three times (linear, 128x4, 8x4
scales); the oracle's swizzle of FlashInfer's own linear scales must reproduce its swizzled
bytes exactly, padding included. Only the byte permutation is compared, so the two
quantizers' arithmetic does not enter. No kernel of this library runs here."""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.helpers import require_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K", [(40, 512), (130, 320), (17, 64), (256, 1024)])
def test_scale_layouts_match_flashinfer(M, K):
    require_cuda()
    flashinfer = pytest.importorskip("flashinfer")
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
