"""nvfp4_global_scale_noalloc: the global scale for callers that cannot allocate device
memory at the call site (an engine's enqueue() handed only tensor pointers, a fixed memory
plan that forbids per-call cudaMalloc/cudaFree). Its reduction scratch is a static array
inside the library, so the call takes no workspace.

The GPU test calls the new entry point through the C ABI and checks it against the
workspace-taking nvfp4_global_scale and against the oracle's global scale (bit-identical g,
the tolerance every global-scale test here uses) on consecutive calls, the second smaller
than the first so stale partials from the first call would show. This file sorts last so a stop-at-first-failure run has already
run everything else."""
import ctypes

import pytest
import torch

import nvfp4_block_scaled_10_b200 as nv
import oracle as orc
from nvfp4_block_scaled_10_b200 import workloads


def _c(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_rejects_inputs_beyond_its_scratch():
    from nvfp4_block_scaled_10_b200 import build

    build.build()
    L = nv.lib()
    p = ctypes.c_void_p(0x10000)  # aligned stand-in: the size check fails before any CUDA call
    # 2^28 elements is the limit; one more row of 16 elements is over it
    assert L.nvfp4_global_scale_noalloc(p, 0, (1 << 24) + 1, 16, 16, p, None) == nv.ERR_SCRATCH_LIMIT
    assert L.nvfp4_global_scale_noalloc(p, 0, 1 << 20, 512, 512, p, None) == nv.ERR_SCRATCH_LIMIT
    assert L.nvfp4_global_scale_noalloc(p, 0, 4, 24, 24, p, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_status_str(nv.ERR_SCRATCH_LIMIT) == b"NVFP4_ERR_SCRATCH_LIMIT"


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.fail("GPU test needs a CUDA device")
    from nvfp4_block_scaled_10_b200 import build

    build.build()
    L = nv.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [
        (workloads.per_token(4096, 7168, seed=21), 0),   # many CTAs: 448 partials
        (workloads.normal((16, 512), 1.0, seed=22), 0),  # one CTA, after the big call
        (workloads.with_outliers((333, 1040), seed=23, dtype=torch.float16), 1),
        (workloads.normal((1, 16), 3.0, seed=24), 0),
    ]
    for x_host, dtype in cases:
        x = x_host.to(dev)
        M, K = x.shape
        g_ref = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
        g_new = torch.full((1,), -2.0, dtype=torch.float32, device=dev)
        ws_bytes = max(L.nvfp4_global_scale_workspace_bytes(M, K), 16)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        assert L.nvfp4_global_scale(_c(x), dtype, M, K, K, _c(g_ref), _c(ws), ws_bytes, stream) == nv.OK
        assert L.nvfp4_global_scale_noalloc(_c(x), dtype, M, K, K, _c(g_new), stream) == nv.OK
        torch.cuda.synchronize()
        assert g_new.item() == g_ref.item(), (M, K, g_new.item(), g_ref.item())
        g_orc = orc.global_scale(workloads.bits16(x_host), orc.BF16 if dtype == 0 else orc.FP16)
        assert g_new.item() == g_orc, (M, K, g_new.item(), g_orc)
        assert g_new.item() > 0
