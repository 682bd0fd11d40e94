"""bench.py host logic on CPU: the algorithmic byte and FLOP counts every roofline fraction
divides by, against the counts worked out from the workload shapes (one read of each input,
one write of each output, scales at one byte per 16 elements in their padded layout)."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_per_token_bytes(bench):
    a = bench.algorithmic("per_token", M=8192, K=7168)
    # X bf16 read; Q 4 bits per element; 8192 x 448 scales (no padding); one fp32 g per row
    assert a["read"] == 8192 * 7168 * 2 == 117_440_512
    assert a["written"] == 29_360_128 + 3_670_016 + 32_768
    assert a["bytes"] == 150_503_424


def test_swiglu_bytes(bench):
    nh = 4096 * 14336
    a = bench.algorithmic("swiglu", M=4096, H=14336)
    assert a["read"] == 4 * nh and a["written"] == nh // 2 + nh // 16
    assert a["bytes"] == 267_911_168  # 4.5625 NH
    f = bench.algorithmic("swiglu_fp8", M=4096, H=14336)
    assert f["bytes"] == 5 * nh  # 4NH read, NH written


def test_scale_padding_counts(bench):
    # 100 rows pad to 128 in 128x4; K/16 = 36 columns pad to 36 (already a multiple of 4)
    a = bench.algorithmic("per_token", M=100, K=576)
    assert a["written"] == 100 * 288 + 128 * 36 + 100 * 4


@pytest.mark.parametrize("M,layout,sa", [(32, "128x4", 128 * 512), (32, "8x4", 32 * 512),
                                         (1, "8x4", 8 * 512), (8, "128x4", 128 * 512)])
def test_decode_bytes(bench, M, layout, sa):
    N, K = 28672, 8192
    a = bench.algorithmic("decode", M=M, N=N, K=K, a_layout=layout)
    w = N * K // 2 + N * K // 16  # packed weights and their 128x4 scales (N a multiple of 128)
    assert a["read"] == w + M * K // 2 + sa
    assert a["written"] == 2 * M * N
    assert a["flops"] == 2 * M * N * K


def test_decode_f32_and_prefill(bench):
    a = bench.algorithmic("decode_f32", M=32, N=28672, K=8192)
    assert a["read"] == 28672 * 4096 + 28672 * 512 + 32 * 4096 + 32 * 512 * 4
    p = bench.algorithmic("prefill", M=8192, N=8192, K=8192)
    assert p["flops"] == 2 * 8192 ** 3 == 1_099_511_627_776


def test_workload_config_shared_by_both_arms(bench):
    """Both arms print the same workload keys; the GEMM ones carry the shapes they run."""
    import types
    args = types.SimpleNamespace(m=32, a_layout="128x4")
    for wl in ("per_token", "swiglu", "swiglu_fp8"):
        assert "workload" in bench.workload_config(wl, args)
    shapes = {"decode": (32, 28672, 8192), "decode_f32": (32, 28672, 8192),
              "prefill": (8192, 8192, 8192), "tiny": (16, 256, 512)}
    for wl, mnk in shapes.items():
        c = bench.workload_config(wl, args)
        assert (c["M"], c["N"], c["K"]) == mnk
    assert bench.workload_config("decode_f32", args)["a_scales"] == "fp32 [M, K/16]"


def test_cpu_baseline_repeats_the_sample(bench):
    """The single-thread oracle baseline repeats its bounded sample until the time budget
    has run and scales the value by the repetitions (the tiny GEMM, a few ms per run)."""
    import types
    args = types.SimpleNamespace(cpu_rows=2048, m=32, a_layout="128x4", no_all_cores=True,
                                 cpu_seconds=0.2)
    r = bench.cpu_baseline("tiny", args)
    reps = int(r["sample"].rsplit(", ", 1)[1].split()[0])
    assert reps >= 1 and r["seconds"] >= 0.2
    assert r["kind"] == "oracle" and r["unit"] == "TFLOP/s" and r["value"] > 0
