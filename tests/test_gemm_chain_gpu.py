"""Calls enqueued back to back on one stream, with no synchronisation between them.

The GEMM kernels (the small-M stream-K kernel and the CTA-pair kernel) are launched as
programmatic dependents of the kernel before them: they may start while that kernel
finishes and prefetch the weights of their first ring pass into L2, and they wait for it
(griddepcontrol.wait) before any load of an input or any write. Each chain here has calls that read the previous call's output, share
one workspace, or rewrite a buffer the previous call used. Every result must equal, bit for
bit, the result of the same call made alone between two synchronisations (the kernels are
deterministic), eagerly and replayed from a CUDA graph; the alone results of the first link
are checked against the oracle too.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from nvfp4_block_scaled_10_b200 import workloads
from tests.helpers import gemm_close, host_bytes, require_cuda

pytestmark = pytest.mark.gpu


def _weights(N, K, seed):
    """Weights quantized by the oracle on the host: (q, 128x4 scales, g) on the device, and
    the oracle's own (q, linear scales, g)."""
    wb = workloads.bits16(workloads.normal((N, K), std=0.05, seed=seed))
    gw = orc.global_scale(wb)
    wq, wsf, _ = orc.quantize(wb, g=gw)
    dev = (torch.from_numpy(wq).cuda(), torch.from_numpy(orc.swizzle(wsf, orc.L128x4)).cuda(),
           torch.tensor([gw], dtype=torch.float32, device="cuda"))
    return dev, (wq, wsf, gw)


class _Layers:
    """x -> quantize (per tensor) -> GEMM 1 -> quantize (per token) -> GEMM 2.

    The intermediate buffers and the GEMM workspace are shared by every pass; each pass
    writes its own final output."""

    def __init__(self, nv, M, K1, N1, N2, seed):
        self.nv = nv
        self.w1, self.w1_host = _weights(N1, K1, seed)
        self.w2, _ = _weights(N2, N1, seed + 1)
        dev = "cuda"
        self.g1 = torch.empty(1, dtype=torch.float32, device=dev)
        self.q1 = torch.empty(M, K1 // 2, dtype=torch.uint8, device=dev)
        self.sf1 = torch.empty(nv.nvfp4_sf_bytes(M, K1), dtype=torch.uint8, device=dev)
        self.y1 = torch.empty(M, N1, dtype=torch.float16, device=dev)
        self.g2 = torch.empty(M, dtype=torch.float32, device=dev)
        self.q2 = torch.empty(M, N1 // 2, dtype=torch.uint8, device=dev)
        self.sf2 = torch.empty(nv.nvfp4_sf_bytes(M, N1), dtype=torch.uint8, device=dev)
        ws = max(nv.nvfp4_gemm_workspace_bytes(M, N1, K1), nv.nvfp4_gemm_workspace_bytes(M, N2, N1))
        self.ws = torch.zeros(max(ws, 16), dtype=torch.uint8, device=dev)
        self.gs_ws = torch.empty(max(nv.nvfp4_global_scale_workspace_bytes(M, K1), 16),
                                 dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def run(self, x, y2, y1_copy=None, sync=False):
        nv = self.nv

        def step():
            if sync:
                torch.cuda.synchronize()

        nv.nvfp4_global_scale(x, self.g1, workspace=self.gs_ws)
        step()
        nv.nvfp4_quantize(x, self.g1, q=self.q1, sf=self.sf1)
        step()
        nv.nvfp4_gemm(self.q1, self.sf1, self.g1, *self.w1, out=self.y1, workspace=self.ws,
                      dev_status=self.status)
        step()
        if y1_copy is not None:
            y1_copy.copy_(self.y1)
            step()
        nv.nvfp4_quantize(self.y1, self.g2, per_token=True, q=self.q2, sf=self.sf2)
        step()
        nv.nvfp4_gemm(self.q2, self.sf2, self.g2, *self.w2, out=y2, workspace=self.ws,
                      dev_status=self.status, per_token_a=True)
        step()


def _chain_case(M, K1, N1, N2, seed, passes=4, graph=False):
    nv = require_cuda()
    L = _Layers(nv, M, K1, N1, N2, seed)
    xs = [workloads.normal((M, K1), seed=seed + 10 + i).cuda() for i in range(passes)]
    # alone: a synchronisation between every two calls
    want2, want1 = [], []
    for x in xs:
        y2 = torch.empty(M, N2, dtype=torch.float16, device="cuda")
        y1 = torch.empty(M, N1, dtype=torch.float16, device="cuda")
        L.run(x, y2, y1_copy=y1, sync=True)
        torch.cuda.synchronize()
        want2.append(host_bytes(y2))
        want1.append(host_bytes(y1))
    assert L.status.item() == 0
    # chained: all passes enqueued at once
    got2 = [torch.full((M, N2), float("nan"), dtype=torch.float16, device="cuda") for _ in xs]
    got1 = [torch.full((M, N1), float("nan"), dtype=torch.float16, device="cuda") for _ in xs]
    torch.cuda.synchronize()
    if graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for x, y2, y1 in zip(xs, got2, got1):
                    L.run(x, y2, y1_copy=y1)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        for t in got2 + got1:
            t.fill_(float("nan"))
        torch.cuda.synchronize()
        g.replay()
    else:
        for x, y2, y1 in zip(xs, got2, got1):
            L.run(x, y2, y1_copy=y1)
    torch.cuda.synchronize()
    assert L.status.item() == 0
    for i in range(passes):
        np.testing.assert_array_equal(host_bytes(got1[i]), want1[i], err_msg=f"pass {i}, GEMM 1")
        np.testing.assert_array_equal(host_bytes(got2[i]), want2[i], err_msg=f"pass {i}, GEMM 2")
    # the first link against the oracle, which quantizes x itself (the GPU quantize is
    # bit-exact against it in the quantize tests)
    x0 = workloads.bits16(xs[0].cpu())
    ga = orc.global_scale(x0)
    aq, sa, _ = orc.quantize(x0, g=ga)
    _, ref = orc.gemm(aq, sa, ga, *L.w1_host, want_f64=True)
    gemm_close(want1[0].view(np.uint16).reshape(M, N1), ref)


@pytest.mark.parametrize("M", [8, 32])
def test_decode_chain(M):
    """Swap-AB stream-K kernels, split tiles sharing one workspace across the two GEMMs."""
    _chain_case(M, K1=2048, N1=4096, N2=2560, seed=300 + M)


def test_decode_chain_graph():
    _chain_case(32, K1=2048, N1=4096, N2=2560, seed=400, graph=True)


def test_pair_chain():
    """CTA-pair kernels (M >= 256), ragged N."""
    _chain_case(512, K1=1024, N1=1280, N2=776, seed=500, passes=3)


def test_pair_chain_graph():
    _chain_case(512, K1=1024, N1=1280, N2=776, seed=600, passes=3, graph=True)


def test_act_f32_chain():
    """Split kernel and GEMM pairs back to back in one workspace; 40 rows = two chunks."""
    nv = require_cuda()
    M, N, K = 40, 2304, 1024
    (wq, wsf, _), _ = _weights(N, K, 700)
    w_scale = torch.tensor([0.75], dtype=torch.float32, device="cuda")
    ws = torch.zeros(nv.nvfp4_gemm_act_f32_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ins = []
    for i in range(4):
        aq = torch.from_numpy(workloads.random_bytes((M, K // 2), 710 + i)).cuda()
        # fp32 scales over several binades, different in every call
        rng = np.random.default_rng(720 + i)
        sf32 = np.float32(2.0 ** rng.uniform(-12, 0, (M, K // 16)) * rng.uniform(1, 2, (M, K // 16)))
        ins.append((aq, torch.from_numpy(sf32).cuda()))
    want = []
    for aq, sf32 in ins:
        out = torch.empty(M, N, dtype=torch.float16, device="cuda")
        nv.nvfp4_gemm_act_f32(aq, sf32, wq, wsf, w_scale, out=out, workspace=ws, dev_status=status)
        torch.cuda.synchronize()
        want.append(host_bytes(out))
    got = [torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda") for _ in ins]
    torch.cuda.synchronize()
    for (aq, sf32), out in zip(ins, got):
        nv.nvfp4_gemm_act_f32(aq, sf32, wq, wsf, w_scale, out=out, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for i, out in enumerate(got):
        np.testing.assert_array_equal(host_bytes(out), want[i], err_msg=f"call {i}")


def test_gemm_after_torch_writer():
    """The GEMM's inputs rewritten by torch elementwise kernels right before each call."""
    nv = require_cuda()
    M, N, K = 32, 3072, 2048
    (wq, wsf, gw), _ = _weights(N, K, 800)
    srcs = []
    for i in range(4):
        xb = workloads.bits16(workloads.normal((M, K), seed=810 + i))
        g = orc.global_scale(xb)
        q, sf, _ = orc.quantize(xb, g=g)
        srcs.append((torch.from_numpy(q).cuda(), torch.from_numpy(orc.swizzle(sf, orc.L128x4)).cuda(),
                     torch.tensor([g], dtype=torch.float32, device="cuda")))
    torch.cuda.synchronize()
    q_buf, sf_buf = torch.empty_like(srcs[0][0]), torch.empty_like(srcs[0][1])
    g_buf = torch.empty_like(srcs[0][2])
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    want = [host_bytes(nv.nvfp4_gemm(q, sf, g, wq, wsf, gw)) for q, sf, g in srcs]
    torch.cuda.synchronize()
    got = []
    for q, sf, g in srcs:
        torch.bitwise_xor(q, 0, out=q_buf)
        torch.bitwise_xor(sf, 0, out=sf_buf)
        torch.mul(g, 1.0, out=g_buf)
        got.append(nv.nvfp4_gemm(q_buf, sf_buf, g_buf, wq, wsf, gw, workspace=ws))
    torch.cuda.synchronize()
    for i, out in enumerate(got):
        np.testing.assert_array_equal(host_bytes(out), want[i], err_msg=f"call {i}")


@pytest.mark.parametrize("M", [32, 512])
def test_gemm_after_weight_writer(M):
    """The weights rewritten on the GPU by the quantize kernel right before each call (the
    GEMM prefetches its first weight tiles while that kernel may still run)."""
    nv = require_cuda()
    N, K = 1280, 2048
    xb = workloads.bits16(workloads.normal((M, K), seed=900 + M))
    ga = orc.global_scale(xb)
    aq, asf, _ = orc.quantize(xb, g=ga)
    a_dev = (torch.from_numpy(aq).cuda(), torch.from_numpy(orc.swizzle(asf, orc.L128x4)).cuda(),
             torch.tensor([ga], dtype=torch.float32, device="cuda"))
    ws_ = [workloads.normal((N, K), std=0.05, seed=910 + i).cuda() for i in range(4)]
    wq = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    wsf = torch.empty(nv.nvfp4_sf_bytes(N, K), dtype=torch.uint8, device="cuda")
    gw = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(nv.nvfp4_gemm_workspace_bytes(M, N, K), 16), dtype=torch.uint8, device="cuda")
    want = []
    for w in ws_:
        nv.nvfp4_global_scale(w, gw)
        nv.nvfp4_quantize(w, gw, q=wq, sf=wsf)
        torch.cuda.synchronize()
        want.append(host_bytes(nv.nvfp4_gemm(*a_dev, wq, wsf, gw, workspace=ws)))
        torch.cuda.synchronize()
    got = []
    for w in ws_:
        nv.nvfp4_global_scale(w, gw)
        nv.nvfp4_quantize(w, gw, q=wq, sf=wsf)
        got.append(nv.nvfp4_gemm(*a_dev, wq, wsf, gw, workspace=ws))
    torch.cuda.synchronize()
    for i, out in enumerate(got):
        np.testing.assert_array_equal(host_bytes(out), want[i], err_msg=f"call {i}")
