"""GPU parity of the block-scaled FP4 GEMM against the oracle (fp64 sum, one fp16 rounding).

Tolerance (normwise and elementwise, see helpers.gemm_close and GEMM_RTOL). Small shapes
cover swap-AB decode tiles, ragged M/N/K tails and both activation-scale layouts; the decode
and prefill workloads are compared in full, every output element against the oracle. Every
output, workspace and status word carries canary guard bands (helpers.Guarded) that must be
untouched after the launch."""
import numpy as np
import pytest
import torch

import oracle as orc
from nvfp4_block_scaled_10_b200 import workloads
from tests.helpers import (GEMM_RTOL, Guarded, check_guards, gemm_close, gemm_close_act_f32,
                           guarded, host_bytes, require_cuda)

pytestmark = pytest.mark.gpu


def _random_operands(M, N, K, seed):
    a = workloads.random_bytes((M, K // 2), seed)
    w = workloads.random_bytes((N, K // 2), seed + 1)
    sa = workloads.random_bytes((M, K // 16), seed + 2, 0x28, 0x48)
    sw = workloads.random_bytes((N, K // 16), seed + 3, 0x28, 0x48)
    return a, sa, 3.5, w, sw, 250.0


def _quantized_operands(a_bf16, w_bf16):
    ab, wb = workloads.bits16(a_bf16), workloads.bits16(w_bf16)
    ga = orc.global_scale(ab)
    gw = orc.global_scale(wb)
    a, sa, _ = orc.quantize(ab, g=ga)
    w, sw, _ = orc.quantize(wb, g=gw)
    return a, sa, ga, w, sw, gw


def _to_device(nv, a, sa, ga, w, sw, gw, a_layout):
    return dict(
        a_q=torch.from_numpy(a).cuda(),
        a_sf=torch.from_numpy(orc.swizzle(sa, a_layout)).cuda(),
        a_g=torch.tensor([ga], dtype=torch.float32, device="cuda"),
        w_q=torch.from_numpy(w).cuda(),
        w_sf=torch.from_numpy(orc.swizzle(sw, orc.L128x4)).cuda(),
        w_g=torch.tensor([gw], dtype=torch.float32, device="cuda"),
        a_layout=a_layout,
    )


def _run(nv, ops, a_layout, per_token_a=False):
    """One GEMM call with guard bands around the output, the workspace and the status word;
    returns the fp16 output bits."""
    dev = _to_device(nv, *ops, a_layout)
    M, N, K = dev["a_q"].shape[0], dev["w_q"].shape[0], 2 * dev["a_q"].shape[1]
    if per_token_a:
        dev["a_g"] = torch.from_numpy(np.ascontiguousarray(ops[2], dtype=np.float32)).cuda()
    g_out = guarded((M, N), torch.float16)
    ws_bytes = nv.nvfp4_gemm_workspace_bytes(M, N, K)
    g_ws = Guarded(ws_bytes, fill=0) if ws_bytes else None
    g_st = Guarded(4, fill=0)
    out = nv.nvfp4_gemm(**dev, out=g_out.view(torch.float16, (M, N)),
                        workspace=None if g_ws is None else g_ws.view(),
                        dev_status=g_st.view(torch.int32), per_token_a=per_token_a)
    torch.cuda.synchronize()
    assert g_st.view(torch.int32).item() == 0
    check_guards(out=g_out, workspace=g_ws, dev_status=g_st)
    return out.cpu().view(torch.int16).numpy().view(np.uint16)


def _ref_by_rows(aq, sa, ga, wq, ws, gw, rows=2048):
    """The oracle's fp64 sums for the whole output, computed over chunks of activation rows
    so that host memory stays bounded (each chunk is the oracle's GEMM of those rows)."""
    M = aq.shape[0]
    parts = []
    for r0 in range(0, M, rows):
        _, ref = orc.gemm(aq[r0:r0 + rows], sa[r0:r0 + rows], ga, wq, ws, gw, want_f64=True)
        parts.append(ref)
    return np.concatenate(parts, axis=0)


def _ref_by_cols(aq, sa, ga, wq, ws, gw, cols=7168):
    """Same over chunks of weight rows (output columns)."""
    N = wq.shape[0]
    parts = []
    for c0 in range(0, N, cols):
        _, ref = orc.gemm(aq, sa, ga, wq[c0:c0 + cols], ws[c0:c0 + cols], gw, want_f64=True)
        parts.append(ref)
    return np.concatenate(parts, axis=1)


# M <= 32: swap-AB tiles; 33..255: single-CTA 128 x 256 tiles; M >= 256: CTA-pair 256 x 256
# tiles (ragged M, N and K tails, and more tiles than resident pairs so the accumulator is
# reused).
SMALL = [(1, 256, 512), (8, 256, 512), (16, 256, 512), (32, 512, 1024), (3, 136, 64),
         (33, 256, 512), (128, 256, 256), (130, 520, 320), (256, 1024, 2048), (300, 264, 4096),
         (520, 776, 320), (4096, 2560, 512), (2000, 5000, 320), (1536, 4608, 512),
         (2048, 3072, 1024),
         (2, 20480, 1024), (32, 4096, 3072), (17, 1032, 8192)]


@pytest.mark.parametrize("M,N,K", SMALL)
def test_gemm_parity_small(M, N, K):
    nv = require_cuda()
    ops = _random_operands(M, N, K, seed=M * 1000 + N + K)
    _, ref = orc.gemm(*ops, want_f64=True)
    layouts = [orc.L128x4, orc.L8x4] if M <= 32 else [orc.L128x4]
    for layout in layouts:
        got = _run(nv, ops, layout)
        gemm_close(got, ref)


def test_gemm_small_m_workspace_contract():
    """M <= 32 needs the split-K workspace; a smaller one is refused before any launch."""
    nv = require_cuda()
    import ctypes
    L = nv.lib()
    M, N, K = 8, 28672, 8192
    need = L.nvfp4_gemm_workspace_bytes(M, N, K)
    assert need >= (N // 128) * 128 * 32 * 4
    assert L.nvfp4_gemm_workspace_bytes(33, N, K) == 0
    ops = _random_operands(M, 256, 512, seed=5)
    dev = _to_device(nv, *ops, orc.L128x4)
    out = torch.empty(M, 256, dtype=torch.float16, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = L.nvfp4_gemm(p(dev["a_q"]), p(dev["a_sf"]), orc.L128x4, p(dev["a_g"]), p(dev["w_q"]),
                      p(dev["w_sf"]), p(dev["w_g"]), p(out), M, 256, 512, p(small), 16, None,
                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == nv.ERR_INVALID_ARG


def test_gemm_tiny_workload():
    """A [16,512] ~N(0,1), W [256,512] ~N(0,0.02) quantized by the oracle; both layouts."""
    nv = require_cuda()
    a, w = workloads.tiny()
    ops = _quantized_operands(a, w)
    _, ref = orc.gemm(*ops, want_f64=True)
    for layout in (orc.L128x4, orc.L8x4):
        gemm_close(_run(nv, ops, layout), ref)


@pytest.fixture(scope="module")
def decode_weights():
    _, w = workloads.decode(1)
    wb = workloads.bits16(w)
    gw = orc.global_scale(wb)
    wq, ws, _ = orc.quantize(wb, g=gw)
    return wq, ws, gw


@pytest.mark.parametrize("M", [1, 8, 32])
def test_gemm_decode_workload(decode_weights, M):
    """W NVFP4 [28672, 8192], A NVFP4 [M, 8192]; both activation-scale layouts; every output
    element (all 28672 columns) against the oracle."""
    nv = require_cuda()
    wq, ws, gw = decode_weights
    a_bf16, _ = workloads.decode(M, N=16, K=8192)  # the activation draw of this workload
    ab = workloads.bits16(a_bf16)
    ga = orc.global_scale(ab)
    aq, sa, _ = orc.quantize(ab, g=ga)
    ref = _ref_by_cols(aq, sa, ga, wq, ws, gw)
    for layout in (orc.L128x4, orc.L8x4):
        got = _run(nv, (aq, sa, ga, wq, ws, gw), layout)
        gemm_close(got, ref)


def test_gemm_prefill_workload():
    """A, W NVFP4 [8192, 8192] from bf16 N(0,1) / N(0,0.02): every one of the 8192 x 8192
    outputs against the oracle (its fp64 product taken over 2048-row chunks)."""
    nv = require_cuda()
    a, w = workloads.prefill()
    ops = _quantized_operands(a, w)
    got = _run(nv, ops, orc.L128x4)
    ref = _ref_by_rows(*ops)
    gemm_close(got, ref)


@pytest.mark.parametrize("M,N,K", [(8, 512, 1024), (32, 20480, 1024), (100, 520, 512),
                                   (300, 264, 1024), (1024, 1024, 2048), (2048, 3072, 1024)])
def test_gemm_per_token_activation_scales(M, N, K):
    """Activation quantized per token (one g per row, as nvfp4_quantize(per_token=True)
    writes), weights per tensor: nvfp4_gemm_per_token against the oracle GEMM with row
    scales. Shapes reach the decode (M <= 32), single-CTA and CTA-pair kernels."""
    nv = require_cuda()
    a = workloads.per_token(M, K, seed=M + K)
    w = workloads.normal((N, K), 0.02, seed=N + 3)
    ab, wb = workloads.bits16(a), workloads.bits16(w)
    a_q, a_sf, g_rows = orc.quantize(ab, per_token=True)
    gw = orc.global_scale(wb)
    w_q, w_sf, _ = orc.quantize(wb, g=gw)
    _, ref = orc.gemm(a_q, a_sf, g_rows, w_q, w_sf, gw, want_f64=True)
    layouts = [orc.L128x4, orc.L8x4] if M <= 32 else [orc.L128x4]
    for layout in layouts:
        got = _run(nv, (a_q, a_sf, g_rows, w_q, w_sf, gw), layout, per_token_a=True)
        gemm_close(got, ref)


def test_per_token_quantize_then_gemm_pipeline():
    """The whole per-token path on the GPU (quantize with per-row g, then the GEMM with those
    row scales) against the same two steps in the oracle, from the same bf16 inputs."""
    nv = require_cuda()
    M, N, K = 384, 768, 2048
    a = workloads.per_token(M, K, seed=77)
    w = workloads.normal((N, K), 0.02, seed=78)
    ab, wb = workloads.bits16(a), workloads.bits16(w)
    a_q, a_sf, g_rows = orc.quantize(ab, per_token=True)
    gw = orc.global_scale(wb)
    w_q, w_sf, _ = orc.quantize(wb, g=gw)
    _, ref = orc.gemm(a_q, a_sf, g_rows, w_q, w_sf, gw, want_f64=True)
    ad, wd = a.cuda(), w.cuda()
    aq_d, asf_d, ag_d = nv.nvfp4_quantize(ad, per_token=True, sf_layout=nv.SF_128x4)
    gw_d = nv.nvfp4_global_scale(wd)
    wq_d, wsf_d, _ = nv.nvfp4_quantize(wd, gw_d, sf_layout=nv.SF_128x4)
    out = nv.nvfp4_gemm(aq_d, asf_d, ag_d, wq_d, wsf_d, gw_d, per_token_a=True)
    torch.cuda.synchronize()
    gemm_close(out.cpu().view(torch.int16).numpy().view(np.uint16), ref)


# ------------------------------------------------------------------ fp32 activation scales

def _e4m3_f64(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def _act_f32_scales(kind, M, K, seed):
    rng = np.random.default_rng(seed)
    if kind == "product":  # E4M3 block scale x fp32 dequantization scale, as DequantizeLinear
        codes = rng.integers(0x10, 0x7F, (M, K // 16), dtype=np.uint8)
        return np.float32(_e4m3_f64(codes) * np.float64(np.float32(1.0 / 37.0)))
    if kind == "wide":  # every block its own binade over 2^-22 .. 2^2, some zeros (the
        # largest kept small enough that the fp16 result stays finite)
        s = np.float32(2.0 ** rng.uniform(-22, 1, (M, K // 16)) * rng.uniform(1, 2, (M, K // 16)))
        s[rng.random(s.shape) < 0.05] = 0.0
        return s
    raise ValueError(kind)


def _run_act_f32(nv, a, sa32, w, sw, w_scale):
    M, N, K = a.shape[0], w.shape[0], 2 * a.shape[1]
    g_out = guarded((M, N), torch.float16)
    g_ws = Guarded(nv.nvfp4_gemm_act_f32_workspace_bytes(M, N, K), fill=0)
    g_st = Guarded(4, fill=0)
    out = nv.nvfp4_gemm_act_f32(torch.from_numpy(a).cuda(),
                                torch.from_numpy(np.ascontiguousarray(sa32)).cuda(),
                                torch.from_numpy(w).cuda(),
                                torch.from_numpy(orc.swizzle(sw, orc.L128x4)).cuda(),
                                torch.tensor([w_scale], dtype=torch.float32, device="cuda"),
                                out=g_out.view(torch.float16, (M, N)), workspace=g_ws.view(),
                                dev_status=g_st.view(torch.int32))
    torch.cuda.synchronize()
    check_guards(out=g_out, workspace=g_ws, dev_status=g_st)
    return out.cpu().view(torch.int16).numpy().view(np.uint16), g_st.view(torch.int32).item()


# M <= 32 one split kernel and one GEMM launch; M > 32 that pair per 32 rows (ragged last
# chunk); K = 64 a single MMA K step; K up to 32768 (the plane words live in the workspace,
# so K has no shared-memory limit).
ACT_F32 = [(1, 256, 512), (5, 136, 64), (32, 512, 1024), (33, 256, 512), (80, 1032, 2048),
           (17, 1032, 8192), (8, 264, 16384), (2, 520, 32768)]


@pytest.mark.parametrize("kind", ["product", "wide"])
@pytest.mark.parametrize("M,N,K", ACT_F32)
def test_gemm_act_f32_parity(M, N, K, kind):
    nv = require_cuda()
    seed = M * 31 + N + K
    a = workloads.random_bytes((M, K // 2), seed)
    w = workloads.random_bytes((N, K // 2), seed + 1)
    sw = workloads.random_bytes((N, K // 16), seed + 3, 0x28, 0x48)
    sa32 = _act_f32_scales(kind, M, K, seed + 2)
    w_scale = float(np.float32(1.0 / 250.0))
    _, ref = orc.gemm_act_f32(a, sa32, w, sw, w_scale, want_f64=True)
    got, status = _run_act_f32(nv, a, sa32, w, sw, w_scale)
    assert status == 0
    gemm_close_act_f32(got, ref)


def test_gemm_act_f32_zero_rows_and_blocks():
    """A row whose scales are all zero gives zeros (the split's row factor is then zero)."""
    nv = require_cuda()
    M, N, K = 6, 264, 1024
    a = workloads.random_bytes((M, K // 2), 3)
    w = workloads.random_bytes((N, K // 2), 4)
    sw = workloads.random_bytes((N, K // 16), 5, 0x28, 0x48)
    sa32 = _act_f32_scales("product", M, K, 6)
    sa32[2] = 0.0
    sa32[4, ::3] = 0.0
    _, ref = orc.gemm_act_f32(a, sa32, w, sw, 0.5, want_f64=True)
    got, status = _run_act_f32(nv, a, sa32, w, sw, 0.5)
    assert status == 0
    assert (got[2].view(np.float16) == 0).all()
    gemm_close_act_f32(got, ref)


def test_gemm_act_f32_bad_scales_flagged():
    """Negative, NaN and infinite activation scales are flagged in dev_status (value 2) and
    their blocks count as zero; the rest of the result is unaffected."""
    nv = require_cuda()
    M, N, K = 4, 136, 512
    a = workloads.random_bytes((M, K // 2), 13)
    w = workloads.random_bytes((N, K // 2), 14)
    sw = workloads.random_bytes((N, K // 16), 15, 0x28, 0x48)
    sa32 = _act_f32_scales("product", M, K, 16)
    bad = sa32.copy()
    bad[0, 3] = -1.0
    bad[1, 0] = np.nan
    bad[3, 31] = np.inf
    clean = sa32.copy()
    clean[0, 3] = clean[1, 0] = clean[3, 31] = 0.0
    _, ref = orc.gemm_act_f32(a, clean, w, sw, 1.0, want_f64=True)
    got, status = _run_act_f32(nv, a, bad, w, sw, 1.0)
    assert status == 2
    gemm_close_act_f32(got, ref)


def test_gemm_act_f32_graph_replay_matches_eager():
    """The split kernel and the GEMM it launches as a programmatic dependent, captured in a
    CUDA graph (two 32-row chunks, so four kernels): every replay, with new activation
    scales copied in between, equals an eager call bit for bit and the oracle."""
    nv = require_cuda()
    M, N, K = 40, 1032, 2048
    a = workloads.random_bytes((M, K // 2), 901)
    w = workloads.random_bytes((N, K // 2), 902)
    sw = workloads.random_bytes((N, K // 16), 903, 0x28, 0x48)
    w_scale = float(np.float32(1.0 / 250.0))
    sets = [_act_f32_scales(kind, M, K, 904 + i) for i, kind in enumerate(["product", "wide"])]
    a_d, w_d = torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda()
    sw_d = torch.from_numpy(orc.swizzle(sw, orc.L128x4)).cuda()
    wsc = torch.tensor([w_scale], dtype=torch.float32, device="cuda")
    sa_d = torch.from_numpy(np.ascontiguousarray(sets[0])).cuda()
    out = torch.empty(M, N, dtype=torch.float16, device="cuda")
    ws = torch.zeros(nv.nvfp4_gemm_act_f32_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        nv.nvfp4_gemm_act_f32(a_d, sa_d, w_d, sw_d, wsc, out=out, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        nv.nvfp4_gemm_act_f32(a_d, sa_d, w_d, sw_d, wsc, out=out, workspace=ws, dev_status=status)
    for sa in sets + sets[:1]:
        sa_d.copy_(torch.from_numpy(np.ascontiguousarray(sa)))
        graph.replay()
        torch.cuda.synchronize()
        replayed = out.cpu().view(torch.int16).numpy().view(np.uint16).copy()
        eager = nv.nvfp4_gemm_act_f32(a_d, sa_d, w_d, sw_d, wsc, workspace=ws, dev_status=status)
        torch.cuda.synchronize()
        assert np.array_equal(replayed, eager.cpu().view(torch.int16).numpy().view(np.uint16))
        _, ref = orc.gemm_act_f32(a, sa, w, sw, w_scale, want_f64=True)
        gemm_close_act_f32(replayed, ref)
    assert status.item() == 0
    del graph


@pytest.mark.parametrize("M", [1, 32])
def test_gemm_act_f32_decode_workload(decode_weights, M):
    """The decode workload (W NVFP4 [28672, 8192]) under the fp32 activation contract: the
    activation quantized by the oracle, its scales handed over as E4M3 value x fp32(1/ga) and
    the weight scale as fp32(1/gw); every output element against the oracle."""
    nv = require_cuda()
    wq, ws, gw = decode_weights
    a_bf16, _ = workloads.decode(M, N=16, K=8192)
    ab = workloads.bits16(a_bf16)
    ga = orc.global_scale(ab)
    aq, sa, _ = orc.quantize(ab, g=ga)
    sa32 = np.float32(_e4m3_f64(sa) * np.float64(np.float32(1.0 / ga)))
    w_scale = float(np.float32(1.0 / gw))
    parts = []
    for c0 in range(0, wq.shape[0], 7168):
        _, r = orc.gemm_act_f32(aq, sa32, wq[c0:c0 + 7168], ws[c0:c0 + 7168], w_scale,
                                want_f64=True)
        parts.append(r)
    ref = np.concatenate(parts, axis=1)
    got, status = _run_act_f32(nv, aq, sa32, wq, ws, w_scale)
    assert status == 0
    gemm_close_act_f32(got, ref)


# ------------------------------------------------------------------ exact special case

@pytest.mark.parametrize("M,N,K", [(8, 1032, 512), (100, 520, 512), (512, 1024, 512),
                                   (2048, 3072, 512)])
def test_gemm_bit_exact_when_accumulation_is_exact(M, N, K):
    """With block scales in {1/2, 1, 2} and unit global scales every product is a multiple of
    1/16 below 2^8, so every partial sum of K = 512 terms is exact in fp32 whatever the
    accumulation order, and alpha = 1: the kernels' fp16 output must equal the oracle's single
    rounding of the exact sum bit for bit. Shapes reach the decode (split-K), single-CTA and
    CTA-pair kernels."""
    nv = require_cuda()
    rng = np.random.default_rng(M + N)
    a = workloads.random_bytes((M, K // 2), M + 1)
    w = workloads.random_bytes((N, K // 2), N + 2)
    codes = np.array([0x30, 0x38, 0x40], np.uint8)  # E4M3 0.5, 1, 2
    sa = codes[rng.integers(0, 3, (M, K // 16))]
    sw = codes[rng.integers(0, 3, (N, K // 16))]
    ref = orc.gemm(a, sa, 1.0, w, sw, 1.0)
    layouts = [orc.L128x4, orc.L8x4] if M <= 32 else [orc.L128x4]
    for layout in layouts:
        got = _run(nv, (a, sa, 1.0, w, sw, 1.0), layout)
        assert np.array_equal(got, ref), f"{np.count_nonzero(got != ref)} outputs differ"


# ------------------------------------------------------------------ row-parallel (tp) GEMM

@pytest.mark.parametrize("M,N,K", [(8, 1032, 2048), (300, 520, 2048)])
def test_row_parallel_shards_on_one_gpu(M, N, K):
    """The two K shards' GEMMs (decode and single-CTA kernels) on one GPU, each against the
    oracle's GEMM of that shard, and their fp16 sum (what the AllReduce computes) against the
    oracle's row-parallel reading, within the two partials' tolerances plus one fp16 rounding.
    No collective runs here."""
    nv = require_cuda()
    from nvfp4_block_scaled_10_b200 import tp
    ops = _random_operands(M, N, K, seed=M + N + K + 7)
    a, sa, ga, w, sw, gw = ops
    d = _to_device(nv, *ops, orc.L128x4)
    outs, bound = [], 0.0
    for r in range(2):
        out = nv.nvfp4_gemm(tp.shard_packed(d["a_q"], r, 2),
                            tp.shard_scales(d["a_sf"], M, K, nv.SF_128x4, r, 2), d["a_g"],
                            tp.shard_packed(d["w_q"], r, 2),
                            tp.shard_scales(d["w_sf"], N, K, nv.SF_128x4, r, 2), d["w_g"])
        k0, k1 = tp.k_shard_bounds(K, r, 2)
        _, ref_r = orc.gemm(a[:, k0 // 2:k1 // 2], sa[:, k0 // 16:k1 // 16], ga,
                            w[:, k0 // 2:k1 // 2], sw[:, k0 // 16:k1 // 16], gw, want_f64=True)
        torch.cuda.synchronize()
        gemm_close(out.cpu().view(torch.int16).numpy().view(np.uint16), ref_r)
        outs.append(out)
        bound = bound + GEMM_RTOL * np.abs(ref_r) + GEMM_RTOL * np.sqrt(np.mean(ref_r ** 2))
    got = (outs[0] + outs[1]).cpu().view(torch.int16).numpy().view(np.uint16)
    want = orc.gemm_row_parallel(*ops, tp=2).view(np.float16).astype(np.float64)
    diff = np.abs(got.view(np.float16).astype(np.float64) - want)
    assert np.all(diff <= bound + 2.0 ** -11 * np.abs(want))


def test_row_parallel_nccl_one_rank():
    """The row-parallel call through NCCL with a single rank equals the plain GEMM."""
    nv = require_cuda()
    import socket

    import torch.distributed as dist

    from nvfp4_block_scaled_10_b200 import tp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        d = _to_device(nv, *_random_operands(8, 520, 1024, seed=91), orc.L128x4)
        ref = nv.nvfp4_gemm(**d)
        got = tp.row_parallel_gemm(**d)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
    finally:
        dist.destroy_process_group()


# ------------------------------------------------------------------ split-K workspace reuse

def test_workspace_reused_across_calls_stays_zero():
    """One zero-filled workspace serves consecutive small-M calls of different shapes (each
    against the oracle); the tiles' last arrivers hand it back zero-filled every time."""
    nv = require_cuda()
    # (8, 19072, 1024): 149 weight tiles, so one tile is left over after a whole tile per
    # CTA and its K-steps are cut over a few CTAs only
    shapes = [(8, 20480, 1024), (32, 4096, 3072), (1, 20480, 8192), (17, 1032, 8192),
              (8, 19072, 1024), (32, 4096, 3072)]
    ws = torch.zeros(max(nv.nvfp4_gemm_workspace_bytes(*s) for s in shapes), dtype=torch.uint8,
                     device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, (M, N, K) in enumerate(shapes):
        ops = _random_operands(M, N, K, seed=600 + i)
        _, ref = orc.gemm(*ops, want_f64=True)
        d = _to_device(nv, *ops, orc.L8x4 if i % 2 else orc.L128x4)
        out = nv.nvfp4_gemm(**d, workspace=ws, dev_status=status)
        torch.cuda.synchronize()
        gemm_close(out.cpu().view(torch.int16).numpy().view(np.uint16), ref)
        assert status.item() == 0
    # the counters sit at the front, in a region sized by the workspace length alone
    region = 16 * (ws.numel() // 65536 + 1)
    assert int(ws[:region].count_nonzero().item()) == 0


def test_workspace_not_zero_is_flagged():
    """A workspace whose tile counters are not zero on entry is reported (dev_status bit 4),
    and the same workspace zero-filled again gives the right result."""
    nv = require_cuda()
    M, N, K = 8, 20480, 1024
    ops = _random_operands(M, N, K, seed=77)
    _, ref = orc.gemm(*ops, want_f64=True)
    d = _to_device(nv, *ops, orc.L128x4)
    ws = torch.full((nv.nvfp4_gemm_workspace_bytes(M, N, K),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_gemm(**d, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() & 4
    ws.zero_()
    status.zero_()
    out = nv.nvfp4_gemm(**d, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    gemm_close(out.cpu().view(torch.int16).numpy().view(np.uint16), ref)
