"""Shared helpers for the GPU parity tests (no method arithmetic here)."""
import numpy as np
import pytest
import torch


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


def gemm_close(got16: np.ndarray, ref64: np.ndarray, rtol: float = 1e-3):
    """GEMM tolerance: normwise max|d - ref| / max|ref| <= rtol and, per element,
    |d - ref| <= rtol * |ref| + rtol * rms(ref) (the fp16 output rounding alone is 2^-11
    relative, and near-zero outputs need the rms term)."""
    got = got16.view(np.float16).astype(np.float64)
    assert np.isfinite(got).all(), "non-finite GEMM output"
    diff = np.abs(got - ref64)
    scale = np.abs(ref64).max()
    rms = np.sqrt(np.mean(ref64 ** 2))
    norm_err = diff.max() / max(scale, 1e-300)
    bound = rtol * np.abs(ref64) + rtol * rms
    bad = np.nonzero(diff > bound)
    assert norm_err <= rtol, f"normwise error {norm_err:.3e} > {rtol}"
    assert bad[0].size == 0, (f"{bad[0].size} elements outside tolerance, e.g. got "
                              f"{got[bad][:4]} want {ref64[bad][:4]}")
    return norm_err
