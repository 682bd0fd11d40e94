"""The GEMM's bounded waits, made to run out on purpose (no fault, no hang).

Every barrier wait in the GEMM kernels gives up after a wall-time limit, reports bit 1 in
the caller's dev_status word and lets the kernel leave through its normal teardown, so a
kernel whose data never arrives cannot hang the GPU ("Building Custom TensorRT-LLM Plugins
for Low-Latency FP8 Inference at Scale", "Production Pitfalls & Hard Lessons"). The test
hooks of include/nvfp4_testing.h shorten the limit to 1 ms and make one CTA's producer stop
issuing copies at a chosen ring position: its consumers then wait on a barrier nothing will
complete, with no copy in flight. The test checks that the call reports the timeout within
milliseconds, that no guard band around the outputs was touched, that the other CTAs'
outputs are correct, and that the next call -- with the workspace zero-filled again, as the
header asks after any dev_status error -- is correct against the oracle."""
import time

import numpy as np
import pytest
import torch

import oracle as orc
from nvfp4_block_scaled_10_b200 import workloads
from tests.helpers import Guarded, check_guards, gemm_close, guarded, require_cuda

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed):
    a = workloads.random_bytes((M, K // 2), seed)
    w = workloads.random_bytes((N, K // 2), seed + 1)
    sa = workloads.random_bytes((M, K // 16), seed + 2, 0x28, 0x48)
    sw = workloads.random_bytes((N, K // 16), seed + 3, 0x28, 0x48)
    return a, sa, 3.5, w, sw, 250.0


@pytest.mark.parametrize("ring_position", [0, 1])
def test_withheld_stage_times_out_then_next_call_is_correct(ring_position):
    nv = require_cuda()
    L = nv.lib()
    # N = 20480: 160 weight tiles over 148 CTAs, so CTA 0 first runs one K-step of a split
    # tile (ring position 0), then its whole tile 0 (positions 1..4). Withholding position 0
    # stops it inside the split tile; position 1 inside its whole tile.
    M, N, K = 8, 20480, 1024
    a, sa, ga, w, sw, gw = _operands(M, N, K, seed=4242)
    _, ref = orc.gemm(a, sa, ga, w, sw, gw, want_f64=True)
    d = dict(a_q=torch.from_numpy(a).cuda(),
             a_sf=torch.from_numpy(orc.swizzle(sa, orc.L128x4)).cuda(),
             a_g=torch.tensor([ga], dtype=torch.float32, device="cuda"),
             w_q=torch.from_numpy(w).cuda(),
             w_sf=torch.from_numpy(orc.swizzle(sw, orc.L128x4)).cuda(),
             w_g=torch.tensor([gw], dtype=torch.float32, device="cuda"))
    g_out = guarded((M, N), torch.float16)
    g_ws = Guarded(nv.nvfp4_gemm_workspace_bytes(M, N, K), fill=0)
    g_st = Guarded(4, fill=0)
    out = g_out.view(torch.float16, (M, N))
    status = g_st.view(torch.int32)
    torch.cuda.synchronize()
    try:
        assert L.nvfp4_testing_set_wait_limit(1_000_000) == nv.OK  # 1 ms
        assert L.nvfp4_testing_withhold_stage(0, ring_position) == nv.OK
        t0 = time.perf_counter()
        nv.nvfp4_gemm(**d, out=out, workspace=g_ws.view(), dev_status=status)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        L.nvfp4_testing_withhold_stage(-1, -1)
        L.nvfp4_testing_set_wait_limit(0)
    assert status.item() & 1, "the withheld stage was not reported as a timeout"
    assert elapsed < 1.0, f"gave up after {elapsed:.3f} s (limit 1 ms per wait)"
    check_guards(out=g_out, workspace=g_ws, dev_status=g_st)
    got = out.cpu().view(torch.int16).numpy().view(np.uint16)
    if ring_position == 1:
        # only CTA 0's whole tile (output columns 0..127) is missing; every other CTA
        # finished normally, the split tile CTA 0 had already contributed to included
        gemm_close(got[:, 128:], ref[:, 128:])

    # the documented recovery: zero the workspace after a call that set dev_status; the
    # next call on the same stream and buffers is then complete and correct
    g_ws.view().zero_()
    status.zero_()
    nv.nvfp4_gemm(**d, out=out, workspace=g_ws.view(), dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    check_guards(out=g_out, workspace=g_ws, dev_status=g_st)
    gemm_close(out.cpu().view(torch.int16).numpy().view(np.uint16), ref)
