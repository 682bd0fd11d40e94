"""The C ABI without a GPU: the library loads, exports every declared symbol, and its host
logic (buffer sizes, argument checks) behaves as include/nvfp4.h states. No call here
reaches a CUDA API: every argument check fails before the device is touched."""
import ctypes
import os
import re

import pytest

import nvfp4_block_scaled_10_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


TESTING_HEADER = os.path.join(ROOT, "include", "nvfp4_testing.h")


def _declared_symbols(header=HEADER):
    text = open(header).read()
    return sorted(set(re.findall(r"^NVFP4_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def L():
    from nvfp4_block_scaled_10_b200 import build

    build.build()
    return nv.lib()


def test_header_declares_the_boundary():
    syms = _declared_symbols()
    assert syms == sorted(nv.SIGNATURES), syms


def test_library_exports_every_declared_symbol(L):
    for name in _declared_symbols() + _declared_symbols(TESTING_HEADER):
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_testing_header_declares_the_hooks(L):
    assert _declared_symbols(TESTING_HEADER) == sorted(nv.TESTING_SIGNATURES)
    # host-only setters: defaults restored, out-of-range positions refused
    assert L.nvfp4_testing_set_wait_limit(0) == nv.OK
    assert L.nvfp4_testing_withhold_stage(-1, -1) == nv.OK
    assert L.nvfp4_testing_withhold_stage(0, 1 << 40) == nv.ERR_INVALID_ARG


def test_status_strings(L):
    assert L.nvfp4_status_str(0) == b"NVFP4_OK"
    assert L.nvfp4_status_str(5) == b"NVFP4_ERR_TIMEOUT"
    assert L.nvfp4_status_str(99) == b"NVFP4_ERR_UNKNOWN"


@pytest.mark.parametrize("rows,k,layout", [(16, 512, 1), (16, 512, 2), (8192, 7168, 1),
                                           (1, 8192, 2), (130, 112, 1), (7, 16, 0), (0, 64, 1)])
def test_sf_bytes_matches_oracle(L, orc, rows, k, layout):
    assert L.nvfp4_sf_bytes(rows, k, layout) == orc.sf_bytes(layout, rows, k // 16)


def test_sf_bytes_rejects(L):
    assert L.nvfp4_sf_bytes(4, 24, 1) == -1
    assert L.nvfp4_sf_bytes(4, 32, 7) == -1
    assert L.nvfp4_sf_bytes(-1, 32, 1) == -1


def test_workspace_sizes(L):
    assert L.nvfp4_gemm_workspace_bytes(8192, 8192, 8192) == 0
    n = L.nvfp4_global_scale_workspace_bytes(8192, 7168)
    assert n % 4 == 0 and 4 <= n <= 8 * 160 * 4
    assert L.nvfp4_global_scale_workspace_bytes(1, 16) == 4


P16 = ctypes.c_void_p(0x10000)   # aligned stand-in pointers: never dereferenced, because
P_ODD = ctypes.c_void_p(0x10008)  # every call below fails its argument check first


def test_quantize_argument_checks(L):
    q = L.nvfp4_quantize
    assert q(P16, 0, 4, 24, 24, P16, 0, P16, P16, 1, None) == nv.ERR_INVALID_ARG   # K % 16
    assert q(P16, 2, 4, 32, 32, P16, 0, P16, P16, 1, None) == nv.ERR_INVALID_ARG   # dtype
    assert q(P16, 0, 4, 32, 16, P16, 0, P16, P16, 1, None) == nv.ERR_INVALID_ARG   # ldx < K
    assert q(P16, 0, 4, 32, 32, P16, 0, P16, P16, 9, None) == nv.ERR_INVALID_ARG   # layout
    assert q(P16, 0, 4, 32, 32, P16, 2, P16, P16, 1, None) == nv.ERR_INVALID_ARG   # per_token
    assert q(P_ODD, 0, 4, 32, 32, P16, 0, P16, P16, 1, None) == nv.ERR_MISALIGNED  # x
    assert q(P16, 0, 4, 32, 36, P16, 0, P16, P16, 1, None) == nv.ERR_MISALIGNED    # ldx % 8
    assert q(P16, 0, 4, 32, 32, P16, 0, P_ODD, P16, 1, None) == nv.ERR_MISALIGNED  # q
    assert q(P16, 0, 4, 32, 32, None, 0, P16, P16, 1, None) == nv.ERR_INVALID_ARG  # g
    assert q(P16, 0, 0, 32, 32, None, 0, None, None, 1, None) == nv.OK             # empty


def test_swiglu_argument_checks(L):
    f = L.swiglu_nvfp4_quantize
    assert f(P16, 0, 4, 24, 48, P16, P16, P16, 1, None) == nv.ERR_INVALID_ARG   # H % 16
    assert f(P16, 0, 4, 32, 48, P16, P16, P16, 1, None) == nv.ERR_INVALID_ARG   # ldx < 2H
    assert f(P_ODD, 0, 4, 32, 64, P16, P16, P16, 1, None) == nv.ERR_MISALIGNED
    assert f(P16, 0, 0, 32, 64, None, None, None, 1, None) == nv.OK


@pytest.mark.parametrize("entry", ["nvfp4_gemm", "nvfp4_gemm_per_token"])
def test_gemm_argument_checks(L, entry):
    g = getattr(L, entry)
    a = (P16, P16, 1, P16, P16, P16, P16, P16)
    assert g(*a, 16, 256, 96, None, 0, None, None) == nv.ERR_INVALID_ARG        # K % 64
    assert g(*a, 16, 250, 512, None, 0, None, None) == nv.ERR_INVALID_ARG       # N % 8
    assert g(P16, P16, 0, P16, P16, P16, P16, P16, 16, 256, 512, None, 0, None, None) == \
        nv.ERR_INVALID_ARG                                                       # linear A scales
    assert g(P16, P16, 2, P16, P16, P16, P16, P16, 64, 256, 512, None, 0, None, None) == \
        nv.ERR_UNSUPPORTED                                                       # 8x4 with M > 32
    assert g(P_ODD, P16, 1, P16, P16, P16, P16, P16, 16, 256, 512, None, 0, None, None) == \
        nv.ERR_MISALIGNED
    assert g(*a, 0, 256, 512, None, 0, None, None) == nv.OK                      # empty


def test_global_scale_and_swizzle_argument_checks(L):
    assert L.nvfp4_global_scale(P16, 0, 4, 24, 24, P16, P16, 64, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_global_scale(P16, 0, 4, 32, 32, None, P16, 64, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_sf_swizzle(P16, P16, 4, 4, 5, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_sf_unswizzle(P16, P16, 0, 4, 1, None) == nv.OK


def test_swiglu_fp8_argument_checks(L):
    f = L.swiglu_fp8_quantize
    assert f(P16, 0, 4, 24, 48, P16, P16, None) == nv.ERR_INVALID_ARG    # H % 16
    assert f(P16, 0, 4, 32, 48, P16, P16, None) == nv.ERR_INVALID_ARG    # ldx < 2H
    assert f(P16, 2, 4, 32, 64, P16, P16, None) == nv.ERR_INVALID_ARG    # dtype
    assert f(P_ODD, 0, 4, 32, 64, P16, P16, None) == nv.ERR_MISALIGNED   # x
    assert f(P16, 0, 4, 32, 64, None, P16, None) == nv.ERR_INVALID_ARG   # scale
    assert f(P16, 0, 4, 32, 64, P16, P_ODD, None) == nv.ERR_MISALIGNED   # q
    assert f(P16, 0, 0, 32, 64, None, None, None) == nv.OK               # empty


def test_gemm_act_f32_argument_checks(L):
    g = L.nvfp4_gemm_act_f32
    a = (P16, P16, P16, P16, P16, P16)  # a_q, a_sf32, w_q, w_sf, w_scale, out
    assert g(*a, 16, 256, 96, None, 0, None, None) == nv.ERR_INVALID_ARG      # K % 64
    assert g(*a, 16, 250, 512, None, 0, None, None) == nv.ERR_INVALID_ARG     # N % 8
    assert g(P16, None, P16, P16, P16, P16, 16, 256, 512, None, 0, None, None) == \
        nv.ERR_INVALID_ARG                                                     # a_sf32
    assert g(P16, P_ODD, P16, P16, P16, P16, 16, 256, 512, None, 0, None, None) == \
        nv.ERR_MISALIGNED                                                      # a_sf32
    assert g(P16, P16, P16, P16, ctypes.c_void_p(0x10002), P16, 16, 256, 512, None, 0, None,
             None) == nv.ERR_MISALIGNED                                        # w_scale
    assert g(*a, 0, 256, 512, None, 0, None, None) == nv.OK                    # empty


def test_missing_library_fails_loudly(monkeypatch):
    """No fallback: without the built library every entry point raises, on a GPU machine too."""
    import torch

    monkeypatch.setattr(nv, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libnvfp4.so"))
    monkeypatch.setattr(nv, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        nv.lib()
    x = torch.zeros(4, 32, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError, match="not built"):
        nv.nvfp4_quantize(x, torch.ones(1))


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "nvfp4.h"

int main(void) {
  /* host-only entry points: sizes, status strings and argument checks (no device touched) */
  long long a = (long long)nvfp4_sf_bytes(200, 96, NVFP4_SF_128x4);  /* 256 rows x 8 columns */
  long long b = (long long)nvfp4_sf_bytes(9, 64, NVFP4_SF_8x4);      /* 16 rows x 4 columns */
  int bad = nvfp4_quantize(NULL, NVFP4_IN_BF16, 1, 17, 17, NULL, 0, NULL, NULL, NVFP4_SF_128x4, NULL);
  printf("%lld %lld %d %s\n", a, b, bad, nvfp4_status_str(bad));
  return strcmp(nvfp4_status_str(NVFP4_OK), "NVFP4_OK") != 0;
}
"""


def test_plain_c_client_compiles_links_and_runs(L, tmp_path):
    """The boundary used from C: the header compiles as pedantic C99 and a program linked
    against libnvfp4.so gets the documented sizes and argument errors."""
    import subprocess

    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(nv.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-l:libnvfp4.so", "-Wl,-rpath," + libdir]
    build = subprocess.run(cmd, capture_output=True, text=True, timeout=120)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    assert run.stdout.split() == [str(256 * 8), str(16 * 4), "1", "NVFP4_ERR_INVALID_ARG"]
