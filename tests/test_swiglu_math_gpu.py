"""silu(gate) of the fused SwiGLU kernel for every possible 16-bit gate.

The kernel divides gate by den = 1 + e(-gate) with a reciprocal approximation and one FMA
correction instead of the general IEEE division sequence. For 16-bit inputs the gate takes
only 2^16 values per type, so the whole domain is checked here: the device arithmetic
(compiled from the same header as the kernel) against the oracle's silu, bit for bit
(NaN against NaN)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle as orc
from tests.helpers import require_cuda

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "nvfp4_block_scaled_10_b200", "csrc")


@pytest.fixture(scope="module")
def silu_lib(tmp_path_factory):
    require_cuda()
    so = str(tmp_path_factory.mktemp("silu") / "libsilu_all.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", "-I", CSRC, "-o", so,
                    os.path.join(HERE, "native", "silu_all.cu")], check=True)
    lib = ctypes.CDLL(so)
    lib.silu_all.restype = ctypes.c_int
    lib.silu_all.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
    return lib


@pytest.mark.parametrize("form", [0, 1, 2])
@pytest.mark.parametrize("dtype", [orc.BF16, orc.FP16])
def test_silu_every_gate_matches_oracle(silu_lib, dtype, form):
    # the kernel picks a form per block from the block's largest |gate| (NaN skipped):
    # form 0 (no exp clamp, no infinite-dividend select) for |gate| <= 87, form 1 (clamp)
    # for other finite gates, form 2 (clamp and select) when a gate is infinite. Each form
    # is checked on every gate it can meet, NaN included.
    bits = np.arange(1 << 16, dtype=np.uint16)
    if dtype == orc.BF16:
        gate = (bits.astype(np.uint32) << 16).view(np.float32)
    else:
        gate = orc.f16_to_f32(bits)
    if form == 0:
        keep = np.isnan(gate) | (np.abs(gate) <= 87.0)
    elif form == 1:
        keep = ~np.isinf(gate)
    else:
        keep = np.ones(gate.shape, bool)
    bits, gate = bits[keep], gate[keep]
    out = np.empty(bits.size, np.float32)
    rc = silu_lib.silu_all(bits.ctypes.data, int(dtype), bits.size, out.ctypes.data, int(form))
    assert rc == 0, f"CUDA error {rc}"
    ref = orc.silu32(gate)
    both_nan = np.isnan(out) & np.isnan(ref)
    bad = (out.view(np.uint32) != ref.view(np.uint32)) & ~both_nan
    idx = np.nonzero(bad)[0]
    assert idx.size == 0, (f"{idx.size} gates differ, e.g. bits {bits[idx[:5]]}: "
                           f"{out[idx[:5]]} vs {ref[idx[:5]]}")
