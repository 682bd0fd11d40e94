"""Shared helpers for the GPU parity tests (no method arithmetic here)."""
import json
import os

import numpy as np
import pytest
import torch

# GEMM tolerances (normwise and elementwise, see gemm_close), tightened from 1e-3 to what
# the measurements allow. The fp16 rounding of the output alone moves a result by up to
# 2^-11 = 4.88e-4 of its magnitude; the fp32 accumulation on the tensor cores adds far less.
# Measured on B200 over every GEMM comparison of the GPU tests (55 with E4M3 activation
# scales, the full 8192^3 prefill and 32 x 28672 decode outputs among them): normwise errors
# up to 4.51e-4, elementwise ratios up to 4.23e-4, and every output within one fp16 step of
# the oracle's correctly rounded result (at most 0.036% of a comparison's outputs one step
# away). So: rtol 5e-4, at most one fp16 step, at most 1% of outputs one step away (a biased
# final rounding, e.g. toward zero, would move far more than 1%).
GEMM_RTOL = 5e-4
GEMM_MAX_ULP = 1
GEMM_MAX_OFF_FRAC = 0.01
# fp32 activation scales: each block scale is carried as rho * (v1 + v2 + v3), three E4M3
# codes under one fp32 row factor, which moves a product by about 1e-4 of itself, so
# outputs near zero can sit many fp16 steps from the correctly rounded sum while the error
# stays a small fraction of rms(ref). Measured over 23 comparisons: normwise up to 4.42e-4,
# elementwise up to 4.35e-4. rtol 6e-4, no fp16-step criterion.
GEMM_RTOL_ACT_F32 = 6e-4


def require_cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU test needs a CUDA device (run with -m 'not gpu' on CPU machines)")
    import nvfp4_block_scaled_10_b200 as nv
    from nvfp4_block_scaled_10_b200 import build

    build.build()
    nv.lib()
    return nv


def to_dev_bits(bits: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """np.uint16 patterns -> device tensor of `dtype` (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dtype)
    return t.cuda()


def host_bytes(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.uint8).numpy().reshape(-1)


def assert_bytes_equal(got: np.ndarray, want: np.ndarray, what: str):
    got = np.asarray(got).reshape(-1)
    want = np.asarray(want).reshape(-1)
    assert got.size == want.size, (what, got.size, want.size)
    bad = np.nonzero(got != want)[0]
    if bad.size:
        i = bad[:8]
        raise AssertionError(f"{what}: {bad.size} of {got.size} bytes differ; first at {i}: "
                             f"got {got[i]} want {want[i]}")


def _f16_order(bits: np.ndarray) -> np.ndarray:
    """fp16 bit patterns -> integers in the order of their values (adjacent values differ
    by 1; +0 and -0 both map to 0)."""
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


ULP_FLOOR = 1.0 / 64  # fp16-step check only where |ref| >= ULP_FLOOR * rms(ref)


def gemm_errors(got16: np.ndarray, ref64: np.ndarray) -> dict:
    """Error figures of a GEMM output against the oracle's fp64 sums: the normwise error
    max|d - ref| / max|ref|, the smallest rtol the elementwise bound accepts
    (max |d - ref| / (|ref| + rms(ref))), and the distance in fp16 steps from the oracle's
    correctly rounded fp16 result, over all outputs and over those with |ref| >=
    ULP_FLOOR * rms(ref) (near zero, the fp32 accumulation error of a cancelling sum can
    exceed an fp16 step of the small result)."""
    got = got16.view(np.float16).astype(np.float64)
    diff = np.abs(got - ref64)
    scale = np.abs(ref64).max()
    rms = np.sqrt(np.mean(ref64 ** 2))
    from oracle import f64_to_f16
    want16 = f64_to_f16(ref64.reshape(-1)).reshape(ref64.shape)
    steps = np.abs(_f16_order(got16.view(np.uint16)) - _f16_order(want16))
    big = np.abs(ref64) >= ULP_FLOOR * rms
    sb = steps[big]
    return {"norm": float(diff.max() / max(scale, 1e-300)),
            "elem": float((diff / (np.abs(ref64) + rms + 1e-300)).max()),
            "ulp_max": int(steps.max()) if steps.size else 0,
            "ulp_frac": float(np.count_nonzero(steps) / max(steps.size, 1)),
            "ulp_max_big": int(sb.max()) if sb.size else 0,
            "ulp_frac_big": float(np.count_nonzero(sb) / max(sb.size, 1)),
            "n": int(ref64.size)}


def _record(errs: dict):
    path = os.environ.get("NVFP4_GEMM_ERR_LOG")
    if path:
        test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
        with open(path, "a") as f:
            f.write(json.dumps({"test": test, **errs}) + "\n")


def gemm_close(got16: np.ndarray, ref64: np.ndarray, rtol: float = GEMM_RTOL,
               max_ulp: int | None = GEMM_MAX_ULP, max_off_frac: float | None = GEMM_MAX_OFF_FRAC):
    """GEMM tolerance: normwise max|d - ref| / max|ref| <= rtol and, per element,
    |d - ref| <= rtol * |ref| + rtol * rms(ref) (the fp16 output rounding alone is 2^-11
    relative, and near-zero outputs need the rms term). With max_ulp set, every output with
    |ref| >= ULP_FLOOR * rms(ref) must also lie within max_ulp fp16 steps of the oracle's
    correctly rounded fp16 result (the fp32 accumulation moves such a sum far less than one
    fp16 step, so only sums next to a rounding boundary land on the neighbouring value), and
    at most max_off_frac of those outputs may differ from it at all."""
    got = got16.view(np.float16).astype(np.float64)
    assert np.isfinite(got).all(), "non-finite GEMM output"
    errs = gemm_errors(got16, ref64)
    _record(errs)
    diff = np.abs(got - ref64)
    rms = np.sqrt(np.mean(ref64 ** 2))
    bound = rtol * np.abs(ref64) + rtol * rms
    bad = np.nonzero(diff > bound)
    assert errs["norm"] <= rtol, f"normwise error {errs['norm']:.3e} > {rtol}"
    assert bad[0].size == 0, (f"{bad[0].size} elements outside tolerance, e.g. got "
                              f"{got[bad][:4]} want {ref64[bad][:4]}")
    if max_ulp is not None:
        assert errs["ulp_max_big"] <= max_ulp, f"{errs['ulp_max_big']} fp16 steps from the oracle"
    if max_off_frac is not None:
        assert errs["ulp_frac_big"] <= max_off_frac, \
            f"{errs['ulp_frac_big']:.3%} of outputs differ from the oracle's fp16 rounding"
    return errs["norm"]


def gemm_close_act_f32(got16: np.ndarray, ref64: np.ndarray):
    """gemm_close with the fp32-activation-scale tolerance (no fp16-step criterion)."""
    return gemm_close(got16, ref64, GEMM_RTOL_ACT_F32, max_ulp=None, max_off_frac=None)


# ------------------------------------------------------------------ guard bands

GUARD_BYTES = 4096
CANARY = 0xA5


class Guarded:
    """A device buffer of `nbytes` with GUARD_BYTES canary bytes before and after it.

    compute-sanitizer is not available to these tests, so out-of-bounds writes are caught
    this way: a kernel that writes past either end of an output changes a canary byte, and
    check() fails. The body starts GUARD_BYTES into the allocation, so it keeps the
    allocation's alignment. `fill` is the body's initial byte (a canary too, unless a zero-
    filled workspace is wanted)."""

    def __init__(self, nbytes: int, fill: int = CANARY, device="cuda"):
        self.n = int(nbytes)
        self.raw = torch.full((self.n + 2 * GUARD_BYTES,), CANARY, dtype=torch.uint8, device=device)
        self.body = self.raw[GUARD_BYTES:GUARD_BYTES + self.n]
        if fill != CANARY:
            self.body.fill_(fill)

    def view(self, dtype=torch.uint8, shape=None) -> torch.Tensor:
        t = self.body.view(dtype)
        return t if shape is None else t.view(*shape)

    def check(self, what: str = "buffer"):
        head = self.raw[:GUARD_BYTES].cpu().numpy()
        tail = self.raw[GUARD_BYTES + self.n:].cpu().numpy()
        for name, band in (("before", head), ("after", tail)):
            bad = np.nonzero(band != CANARY)[0]
            if bad.size:
                raise AssertionError(f"{what}: {bad.size} guard bytes {name} the buffer were "
                                     f"written (first at offset {bad[0]})")


def guarded(shape, dtype=torch.uint8, fill: int = CANARY) -> Guarded:
    """Guarded buffer sized for a tensor of `shape` and `dtype`."""
    n = int(np.prod(shape)) * torch.empty(0, dtype=dtype).element_size()
    return Guarded(n, fill)


def check_guards(**bufs):
    for name, g in bufs.items():
        if g is not None:
            g.check(name)
