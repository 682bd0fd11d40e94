"""Writes flashinfer_sf_layouts.txt: FlashInfer's own scale bytes for a few small, ragged
shapes, in the linear, 128x4 and 8x4 layouts of "feature: add fp4 mm using trtllm backend"
(FlashInfer PR #1355, the PR that introduced the two swizzled layouts).

Only FlashInfer runs here (fp4_quantize on a CUDA device; the input is drawn by a seeded
torch CPU generator): no code of this repository's library or oracle is called, so the
stored bytes are an outside reference for the layouts. The CPU test
tests/test_oracle_layout_gemm.py::test_flashinfer_sf_layout_bytes checks that the oracle's
swizzle of the stored linear scales gives the stored 128x4 and 8x4 bytes, padding included.

    python tests/golden/make_flashinfer_sf_layouts.py [output path]
"""
import sys

import torch

SHAPES = [(17, 64), (9, 96), (130, 320)]  # rows and K: ragged rows, and C = K/16 = 6 ragged


def main(path):
    import flashinfer

    lines = ["# FlashInfer " + flashinfer.__version__ + " fp4_quantize scale bytes (hex), written by",
             "# make_flashinfer_sf_layouts.py. One record per shape: 'shape M K', then the",
             "# linear [M, K/16] scales, the 128x4 buffer and the 8x4 buffer, each on one line."]
    for M, K in SHAPES:
        g = torch.Generator().manual_seed(M * 1000 + K)
        # block magnitudes over several binades so that many scale codes occur
        x = torch.randn(M, K, generator=g) * torch.exp(
            2 * torch.randn(M, K // 16, generator=g)).repeat_interleave(16, dim=1)
        x = x.to(torch.bfloat16).cuda()
        gs = torch.tensor([2688.0 / x.float().abs().max().item()], device="cuda")
        try:
            _, lin = flashinfer.fp4_quantize(x, gs, 16, False, is_sf_swizzled_layout=False)
            _, s128 = flashinfer.fp4_quantize(x, gs, 16, False, is_sf_swizzled_layout=True,
                                              is_sf_8x4_layout=False)
            _, s84 = flashinfer.fp4_quantize(x, gs, 16, False, is_sf_swizzled_layout=True,
                                             is_sf_8x4_layout=True)
        except Exception as e:  # a shape FlashInfer does not take is left out, said so
            lines.append(f"# shape {M} {K} not taken by fp4_quantize: {type(e).__name__}")
            continue
        torch.cuda.synchronize()
        lin = lin.view(torch.uint8).cpu().reshape(-1)[:M * (K // 16)]
        lines.append(f"shape {M} {K}")
        for t in (lin, s128.view(torch.uint8).cpu().reshape(-1), s84.view(torch.uint8).cpu().reshape(-1)):
            lines.append(bytes(t.tolist()).hex())
    with open(path, "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main(sys.argv[1] if len(sys.argv) > 1 else __file__.replace("make_flashinfer_sf_layouts.py",
                                                                 "flashinfer_sf_layouts.txt"))
