"""NVFP4 block-scaled quantization and block-scaled FP4 GEMM for B200 (sm_100a).

Thin Python binding over the C ABI of ``libnvfp4.so`` (declared in ``include/nvfp4.h``).
Functions carry the C names; they only marshal torch tensors (device memory, the current
stream) into pointers and sizes and raise on a non-zero status. Every step runs in the
library's CUDA kernels; there is no other implementation behind these names, and the
library must be built (``python -m nvfp4_block_scaled_10_b200.build``) or calls raise.

Tensors: activations bf16/fp16 [M, K] (row stride may exceed K); packed E2M1 operands
uint8 [rows, K/2]; scale buffers uint8 of ``nvfp4_sf_bytes`` bytes; global scales fp32.
"""
from __future__ import annotations

import ctypes
import os

import torch

SF_LINEAR, SF_128x4, SF_8x4 = 0, 1, 2
IN_BF16, IN_FP16 = 0, 1

OK, ERR_INVALID_ARG, ERR_MISALIGNED, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_SCRATCH_LIMIT = range(7)

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4.so")

# every symbol include/nvfp4.h declares, with its ctypes signature
_i64, _sz, _vp, _i32 = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int
SIGNATURES = {
    "nvfp4_status_str": (ctypes.c_char_p, [_i32]),
    "nvfp4_sf_bytes": (_i64, [_i64, _i64, _i32]),
    "nvfp4_global_scale_workspace_bytes": (_sz, [_i64, _i64]),
    "nvfp4_global_scale": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _vp, _sz, _vp]),
    "nvfp4_global_scale_noalloc": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _vp]),
    "nvfp4_quantize": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _i32, _vp]),
    "swiglu_nvfp4_quantize": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _i32, _vp]),
    "swiglu_fp8_quantize": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _vp, _vp]),
    "nvfp4_sf_swizzle": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp]),
    "nvfp4_sf_unswizzle": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp]),
    "nvfp4_gemm_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "nvfp4_gemm": (_i32, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz,
                          _vp, _vp]),
    "nvfp4_gemm_per_token": (_i32, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                    _vp, _sz, _vp, _vp]),
    "nvfp4_gemm_act_f32_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "nvfp4_gemm_act_f32": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz, _vp,
                                  _vp]),
}

# test hooks declared in include/nvfp4_testing.h (they change no result; see that header)
TESTING_SIGNATURES = {
    "nvfp4_testing_set_wait_limit": (_i32, [ctypes.c_uint64]),
    "nvfp4_testing_withhold_stage": (_i32, [_i32, _i64]),
}

_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().nvfp4_status_str(status).decode()} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded libnvfp4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libnvfp4.so is not built ({LIB_PATH}); run "
                               "`python -m nvfp4_block_scaled_10_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in {**SIGNATURES, **TESTING_SIGNATURES}.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != OK:
        raise Nvfp4Error(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return IN_BF16
    if t.dtype == torch.float16:
        return IN_FP16
    raise TypeError(f"activations must be bf16 or fp16, got {t.dtype}")


def _rows_ld(x: torch.Tensor):
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit inner stride")
    return x.shape[0], x.shape[1], x.stride(0)


def nvfp4_sf_bytes(rows: int, k: int, layout: int = SF_128x4) -> int:
    n = lib().nvfp4_sf_bytes(rows, k, layout)
    if n < 0:
        raise ValueError(f"invalid scale-buffer request rows={rows} k={k} layout={layout}")
    return n


def nvfp4_global_scale_workspace_bytes(M: int, K: int) -> int:
    return lib().nvfp4_global_scale_workspace_bytes(M, K)


def nvfp4_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return lib().nvfp4_gemm_workspace_bytes(M, N, K)


def nvfp4_global_scale(x: torch.Tensor, g_out: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """g = 448*6 / max|x| over the tensor, as a device fp32 [1]."""
    M, K, ldx = _rows_ld(x)
    if g_out is None:
        g_out = torch.empty(1, dtype=torch.float32, device=x.device)
    nbytes = nvfp4_global_scale_workspace_bytes(M, K)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _check(lib().nvfp4_global_scale(_ptr(x), _dtype_code(x), M, K, ldx, _ptr(g_out),
                                    _ptr(workspace), workspace.numel(), _stream(stream)),
           "nvfp4_global_scale")
    return g_out


def nvfp4_global_scale_noalloc(x: torch.Tensor, g_out: torch.Tensor, stream=None) -> torch.Tensor:
    """Same g as nvfp4_global_scale, reduction scratch inside the library (no workspace).

    For callers that cannot allocate at the call site; `g_out` (device fp32 [1]) is theirs.
    Inputs above 2^28 elements raise (NVFP4_ERR_SCRATCH_LIMIT).
    """
    M, K, ldx = _rows_ld(x)
    _check(lib().nvfp4_global_scale_noalloc(_ptr(x), _dtype_code(x), M, K, ldx, _ptr(g_out),
                                            _stream(stream)), "nvfp4_global_scale_noalloc")
    return g_out


def nvfp4_quantize(x: torch.Tensor, g: torch.Tensor | None = None, per_token: bool = False,
                   sf_layout: int = SF_128x4, q: torch.Tensor | None = None,
                   sf: torch.Tensor | None = None, stream=None):
    """Quantize x [M, K] -> (q uint8 [M, K/2], sf uint8 [nvfp4_sf_bytes], g fp32).

    per_token=False: `g` (device fp32 [1]) is the per-tensor encode scale.
    per_token=True: g [M] is written (allocated when None).
    """
    M, K, ldx = _rows_ld(x)
    dev = x.device
    if per_token and g is None:
        g = torch.empty(M, dtype=torch.float32, device=dev)
    if g is None:
        raise ValueError("per-tensor quantize needs g")
    if q is None:
        q = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty(nvfp4_sf_bytes(M, K, sf_layout), dtype=torch.uint8, device=dev)
    _check(lib().nvfp4_quantize(_ptr(x), _dtype_code(x), M, K, ldx, _ptr(g), int(per_token),
                                _ptr(q), _ptr(sf), sf_layout, _stream(stream)), "nvfp4_quantize")
    return q, sf, g


def swiglu_nvfp4_quantize(x: torch.Tensor, g: torch.Tensor, sf_layout: int = SF_128x4,
                          q: torch.Tensor | None = None, sf: torch.Tensor | None = None,
                          stream=None):
    """Fused silu(gate) * up -> NVFP4 for x [M, 2H] = [gate | up]; returns (q [M,H/2], sf)."""
    M, H2, ldx = _rows_ld(x)
    H = H2 // 2
    dev = x.device
    if q is None:
        q = torch.empty(M, H // 2, dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty(nvfp4_sf_bytes(M, H, sf_layout), dtype=torch.uint8, device=dev)
    _check(lib().swiglu_nvfp4_quantize(_ptr(x), _dtype_code(x), M, H, ldx, _ptr(g), _ptr(q),
                                       _ptr(sf), sf_layout, _stream(stream)),
           "swiglu_nvfp4_quantize")
    return q, sf


def swiglu_fp8_quantize(x: torch.Tensor, scale: torch.Tensor, q: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """Fused silu(gate) * up -> FP8 E4M3 (saturating) for x [M, 2H] = [gate | up]; returns
    q uint8 [M, H] (E4M3 bit patterns). scale: device fp32 [1], multiplies y."""
    M, H2, ldx = _rows_ld(x)
    H = H2 // 2
    if q is None:
        q = torch.empty(M, H, dtype=torch.uint8, device=x.device)
    _check(lib().swiglu_fp8_quantize(_ptr(x), _dtype_code(x), M, H, ldx, _ptr(scale), _ptr(q),
                                     _stream(stream)), "swiglu_fp8_quantize")
    return q


def nvfp4_sf_swizzle(lin: torch.Tensor, layout: int = SF_128x4, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Linear [R, C] scale codes -> layout buffer (padding zeroed)."""
    R, C = lin.shape
    if out is None:
        out = torch.empty(nvfp4_sf_bytes(R, 16 * C, layout), dtype=torch.uint8, device=lin.device)
    _check(lib().nvfp4_sf_swizzle(_ptr(lin.contiguous()), _ptr(out), R, C, layout,
                                  _stream(stream)), "nvfp4_sf_swizzle")
    return out


def nvfp4_sf_unswizzle(buf: torch.Tensor, R: int, C: int, layout: int = SF_128x4,
                       out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Layout buffer -> linear [R, C] scale codes."""
    if out is None:
        out = torch.empty(R, C, dtype=torch.uint8, device=buf.device)
    _check(lib().nvfp4_sf_unswizzle(_ptr(buf), _ptr(out), R, C, layout, _stream(stream)),
           "nvfp4_sf_unswizzle")
    return out


def nvfp4_gemm(a_q: torch.Tensor, a_sf: torch.Tensor, a_g: torch.Tensor, w_q: torch.Tensor,
               w_sf: torch.Tensor, w_g: torch.Tensor, a_layout: int = SF_128x4,
               out: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, per_token_a: bool = False,
               stream=None) -> torch.Tensor:
    """out[M, N] fp16 = dequant(a_q) @ dequant(w_q)^T (K = 2 * a_q.shape[1]).

    per_token_a: a_g is fp32 [M], one encode scale per activation row (the g that
    nvfp4_quantize(per_token=True) writes); otherwise a_g is fp32 [1].
    """
    M, K2 = a_q.shape
    N = w_q.shape[0]
    K = 2 * K2
    if out is None:
        out = torch.empty(M, N, dtype=torch.float16, device=a_q.device)
    nbytes = nvfp4_gemm_workspace_bytes(M, N, K)
    if workspace is None and nbytes > 0:
        workspace = torch.zeros(nbytes, dtype=torch.uint8, device=a_q.device)  # zero on first use
    if per_token_a and a_g.numel() != M:
        raise ValueError(f"per_token_a needs a_g with M = {M} elements, got {a_g.numel()}")
    fn = lib().nvfp4_gemm_per_token if per_token_a else lib().nvfp4_gemm
    _check(fn(_ptr(a_q), _ptr(a_sf), a_layout, _ptr(a_g), _ptr(w_q), _ptr(w_sf), _ptr(w_g),
              _ptr(out), M, N, K, _ptr(workspace), 0 if workspace is None else workspace.numel(),
              _ptr(dev_status), _stream(stream)),
           "nvfp4_gemm_per_token" if per_token_a else "nvfp4_gemm")
    return out


def nvfp4_gemm_act_f32_workspace_bytes(M: int, N: int, K: int) -> int:
    return lib().nvfp4_gemm_act_f32_workspace_bytes(M, N, K)


def nvfp4_gemm_act_f32(a_q: torch.Tensor, a_sf32: torch.Tensor, w_q: torch.Tensor,
                       w_sf: torch.Tensor, w_scale: torch.Tensor, out: torch.Tensor | None = None,
                       dev_status: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[M, N] fp16 under the fp32 activation-scale contract: a_sf32 fp32 [M, K/16] (or
    [M, 1, K/16]) combined activation scales, w_scale fp32 [1] multiplying the weight."""
    M, K2 = a_q.shape
    N = w_q.shape[0]
    K = 2 * K2
    if a_sf32.dtype != torch.float32 or a_sf32.numel() != M * (K // 16) or not a_sf32.is_contiguous():
        raise ValueError("a_sf32 must be a contiguous fp32 tensor of M x K/16 scales")
    if out is None:
        out = torch.empty(M, N, dtype=torch.float16, device=a_q.device)
    nbytes = nvfp4_gemm_act_f32_workspace_bytes(M, N, K)
    if workspace is None and nbytes > 0:
        workspace = torch.zeros(nbytes, dtype=torch.uint8, device=a_q.device)  # zero on first use
    _check(lib().nvfp4_gemm_act_f32(_ptr(a_q), _ptr(a_sf32), _ptr(w_q), _ptr(w_sf), _ptr(w_scale),
                                    _ptr(out), M, N, K, _ptr(workspace),
                                    0 if workspace is None else workspace.numel(),
                                    _ptr(dev_status), _stream(stream)),
           "nvfp4_gemm_act_f32")
    return out
