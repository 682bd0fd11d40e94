"""CPU oracle for the NVFP4 quantize + block-scaled FP4 GEMM path.

TEST INFRASTRUCTURE ONLY: the library (``nvfp4_block_scaled_10_b200``) never imports
this package. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm use it.

The arithmetic lives in ``nvfp4_oracle.c`` (plain loops, fp32 quantize math with one
IEEE rounding per operation, fp64 GEMM sum). This module only compiles it with gcc,
loads it with ctypes and marshals numpy arrays. Every function cites the passage it
follows in the C source.

Layouts: ``LINEAR = 0``, ``L128x4 = 1``, ``L8x4 = 2``. Input dtypes: ``BF16 = 0``,
``FP16 = 1`` (raw 16-bit patterns held in ``np.uint16`` arrays).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

LINEAR, L128x4, L8x4 = 0, 1, 2
BF16, FP16 = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", _SRC, "-o", tmp, "-lm",
        ])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        i64, f32, f64, vp, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        sigs = {
            "orc_bf16_to_f32": (f32, [ctypes.c_uint16]),
            "orc_f16_to_f32": (f32, [ctypes.c_uint16]),
            "orc_e2m1_value": (f64, [i32]),
            "orc_e2m1_encode": (i32, [f32]),
            "orc_e4m3_value": (f64, [i32]),
            "orc_e4m3_encode": (i32, [f32]),
            "orc_f64_to_f16": (ctypes.c_uint16, [f64]),
            "orc_exp": (f32, [f32]),
            "orc_silu": (f32, [f32]),
            "orc_swiglu_elem": (f32, [f32, f32]),
            "orc_global_scale": (f32, [f32]),
            "orc_amax": (f32, [vp, i32, i64, i64, i64]),
            "orc_quantize_block": (None, [vp, f32, vp, vp]),
            "orc_quantize": (None, [vp, i32, i64, i64, i64, vp, i32, vp, vp]),
            "orc_swiglu": (None, [vp, i32, i64, i64, i64, vp]),
            "orc_swiglu_quantize": (None, [vp, i32, i64, i64, i64, f32, vp, vp]),
            "orc_swiglu_amax": (f32, [vp, i32, i64, i64, i64]),
            "orc_sf_rows_padded": (i64, [i32, i64]),
            "orc_sf_cols_padded": (i64, [i32, i64]),
            "orc_sf_bytes": (i64, [i32, i64, i64]),
            "orc_sf_offset": (i64, [i32, i64, i64, i64, i64]),
            "orc_sf_swizzle": (None, [vp, i64, i64, i32, vp]),
            "orc_sf_unswizzle": (None, [vp, i64, i64, i32, vp]),
            "orc_gemm": (None, [vp, vp, f32, vp, vp, f32, i64, i64, i64, vp, vp]),
            "orc_dequantize": (None, [vp, vp, f32, i64, i64, vp]),
            "orc_dequantize_rows": (None, [vp, vp, vp, i64, i64, vp]),
            "orc_swiglu_fp8": (None, [vp, i32, i64, i64, i64, f32, vp]),
            "orc_e4m3_encode_signed_array": (None, [vp, i64, vp]),
            "orc_e2m1_encode_array": (None, [vp, i64, vp]),
            "orc_e4m3_encode_array": (None, [vp, i64, vp]),
            "orc_exp_array": (None, [vp, i64, vp]),
            "orc_silu_array": (None, [vp, i64, vp]),
            "orc_f64_to_f16_array": (None, [vp, i64, vp]),
            "orc_f16_to_f32_array": (None, [vp, i64, vp]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------------------- codecs

def e2m1_value(code: int) -> float:
    """OCP MX E2M1 value of a 4-bit code."""
    return lib().orc_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    """OCP OFP8 E4M3 value of an 8-bit code (NaN for 0x7F / 0xFF)."""
    return lib().orc_e4m3_value(int(code))


def e2m1_encode(y) -> np.ndarray:
    """E2M1 round-to-nearest-even with saturation, sign kept (array in, uint8 codes out)."""
    y = _c(np.atleast_1d(y), np.float32)
    out = np.empty(y.shape, np.uint8)
    lib().orc_e2m1_encode_array(_p(y), y.size, _p(out))
    return out


def e4m3_encode(s) -> np.ndarray:
    """E4M3 round-to-nearest-even with saturation to 448 (non-negative input)."""
    s = _c(np.atleast_1d(s), np.float32)
    out = np.empty(s.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(s), s.size, _p(out))
    return out


def f64_to_f16(v) -> np.ndarray:
    """fp64 -> IEEE binary16 bits, round to nearest even, overflow to inf."""
    v = _c(np.atleast_1d(v), np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().orc_f64_to_f16_array(_p(v), v.size, _p(out))
    return out


def f16_to_f32(h) -> np.ndarray:
    h = _c(np.atleast_1d(h), np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().orc_f16_to_f32_array(_p(h), h.size, _p(out))
    return out


def exp32(x) -> np.ndarray:
    """Project-defined fp32 exponential used by SwiGLU (clamp, Cody-Waite, Taylor-7)."""
    x = _c(np.atleast_1d(x), np.float32)
    out = np.empty(x.shape, np.float32)
    lib().orc_exp_array(_p(x), x.size, _p(out))
    return out


def silu32(x) -> np.ndarray:
    """silu(v) = v / (1 + e(-v)) in fp32."""
    x = _c(np.atleast_1d(x), np.float32)
    out = np.empty(x.shape, np.float32)
    lib().orc_silu_array(_p(x), x.size, _p(out))
    return out


# ----------------------------------------------------------------------------- scales

def global_scale_from_amax(amax: float) -> float:
    """g = 448*6/amax (1 when amax == 0, clamped to FLT_MAX)."""
    return float(np.float32(lib().orc_global_scale(float(np.float32(amax)))))


def amax(x_bits: np.ndarray, dtype: int = BF16) -> float:
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    return float(np.float32(lib().orc_amax(_p(x), dtype, M, K, K)))


def global_scale(x_bits: np.ndarray, dtype: int = BF16) -> float:
    """Per-tensor global encode scale of X: g = 448*6 / max|x|."""
    return global_scale_from_amax(amax(x_bits, dtype))


# ----------------------------------------------------------------------------- quantize

def quantize_block(x16, g: float):
    """One 16-element block -> (E4M3 scale code, 16 unpacked E2M1 codes)."""
    x = _c(x16, np.float32)
    assert x.size == 16
    s = np.zeros(1, np.uint8)
    q = np.zeros(16, np.uint8)
    lib().orc_quantize_block(_p(x), float(np.float32(g)), _p(s), _p(q))
    return int(s[0]), q


def quantize(x_bits: np.ndarray, dtype: int = BF16, g=None, per_token: bool = False):
    """Quantize X [M,K] (raw 16-bit patterns).

    Returns (q [M,K/2] uint8 packed, sf [M,K/16] uint8 linear E4M3 codes, g) where g is
    a float32 array: [1] as given (per-tensor) or [M] computed (per-token).
    """
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    assert K % 16 == 0
    q = np.zeros((M, K // 2), np.uint8)
    sf = np.zeros((M, K // 16), np.uint8)
    if per_token:
        gv = np.zeros(M, np.float32)
    else:
        gv = np.array([g], dtype=np.float32)
    lib().orc_quantize(_p(x), dtype, M, K, K, _p(gv), 1 if per_token else 0, _p(q), _p(sf))
    return q, sf, gv


def swiglu(x_bits: np.ndarray, dtype: int = BF16) -> np.ndarray:
    """Y = silu(gate) * up in fp32 for X [M, 2H] = [gate | up]."""
    x = _c(x_bits, np.uint16)
    M, H2 = x.shape
    H = H2 // 2
    y = np.zeros((M, H), np.float32)
    lib().orc_swiglu(_p(x), dtype, M, H, H2, _p(y))
    return y


def swiglu_amax(x_bits: np.ndarray, dtype: int = BF16) -> float:
    x = _c(x_bits, np.uint16)
    M, H2 = x.shape
    return float(np.float32(lib().orc_swiglu_amax(_p(x), dtype, M, H2 // 2, H2)))


def e4m3_encode_signed(v) -> np.ndarray:
    """Signed saturating FP8 E4M3 codes of fp32 values (NaN -> 0x7F)."""
    vv = _c(np.atleast_1d(v), np.float32)
    out = np.empty(vv.shape, np.uint8)
    lib().orc_e4m3_encode_signed_array(_p(vv), vv.size, _p(out))
    return out


def swiglu_fp8(x_bits: np.ndarray, scale: float, dtype: int = BF16) -> np.ndarray:
    """Fused SwiGLU + FP8 E4M3: q [M, H] = E4M3_sat(fl(silu(gate) * up) * scale)."""
    x = _c(x_bits, np.uint16)
    M, H2 = x.shape
    H = H2 // 2
    q = np.zeros((M, H), np.uint8)
    lib().orc_swiglu_fp8(_p(x), dtype, M, H, H2, float(np.float32(scale)), _p(q))
    return q


def swiglu_quantize(x_bits: np.ndarray, g: float, dtype: int = BF16):
    """Fused SwiGLU + NVFP4 quantize with per-tensor g -> (q [M,H/2], sf [M,H/16] linear)."""
    x = _c(x_bits, np.uint16)
    M, H2 = x.shape
    H = H2 // 2
    assert H % 16 == 0
    q = np.zeros((M, H // 2), np.uint8)
    sf = np.zeros((M, H // 16), np.uint8)
    lib().orc_swiglu_quantize(_p(x), dtype, M, H, H2, float(np.float32(g)), _p(q), _p(sf))
    return q, sf


# ----------------------------------------------------------------------------- layouts

def sf_bytes(layout: int, R: int, C: int) -> int:
    return int(lib().orc_sf_bytes(layout, R, C))


def sf_offset(layout: int, r: int, c: int, R: int, C: int) -> int:
    return int(lib().orc_sf_offset(layout, r, c, R, C))


def swizzle(sf_lin: np.ndarray, layout: int) -> np.ndarray:
    """Linear [R,C] scale codes -> the layout's padded byte buffer (padding zero)."""
    s = _c(sf_lin, np.uint8)
    R, C = s.shape
    out = np.full(sf_bytes(layout, R, C), 0xAA, np.uint8)
    lib().orc_sf_swizzle(_p(s), R, C, layout, _p(out))
    return out


def unswizzle(buf: np.ndarray, R: int, C: int, layout: int) -> np.ndarray:
    b = _c(buf, np.uint8).reshape(-1)
    assert b.size >= sf_bytes(layout, R, C)
    lin = np.zeros((R, C), np.uint8)
    lib().orc_sf_unswizzle(_p(b), R, C, layout, _p(lin))
    return lin


# ----------------------------------------------------------------------------- GEMM

def dequantize(q, sf_lin, g) -> np.ndarray:
    """fp64 values E2M1(q) * E4M3(s) / g of a packed operand [rows, K/2]."""
    qq = _c(q, np.uint8)
    ss = _c(sf_lin, np.uint8)
    rows, K2 = qq.shape
    K = 2 * K2
    assert ss.shape == (rows, K // 16)
    out = np.zeros((rows, K), np.float64)
    lib().orc_dequantize(_p(qq), _p(ss), float(np.float32(g)), rows, K, _p(out))
    return out


def dequantize_rows(q, sf_lin, g_rows) -> np.ndarray:
    """fp64 values E2M1(q) * E4M3(s) / g[r] of a packed operand [rows, K/2] quantized with
    one encode scale per row."""
    qq = _c(q, np.uint8)
    ss = _c(sf_lin, np.uint8)
    gg = _c(np.asarray(g_rows, dtype=np.float32).reshape(-1), np.float32)
    rows, K2 = qq.shape
    K = 2 * K2
    assert ss.shape == (rows, K // 16) and gg.shape == (rows,)
    out = np.zeros((rows, K), np.float64)
    lib().orc_dequantize_rows(_p(qq), _p(ss), _p(gg), rows, K, _p(out))
    return out


def gemm(a_q, a_sf_lin, a_g, w_q, w_sf_lin, w_g, want_f64: bool = False):
    """D = fp16_rn(deq(A) @ deq(W)^T): dequantization in the C oracle, the fp64 product by
    numpy's matmul (a library step), one rounding to fp16 by the C oracle.

    a_q [M,K/2], a_sf_lin [M,K/16], w_q [N,K/2], w_sf_lin [N,K/16]; w_g is a scalar; a_g is a
    scalar or, for an activation quantized per token, an array of M row scales.
    Returns fp16 bits [M,N] (uint16), plus the fp64 sums when want_f64.
    """
    if np.ndim(a_g) > 0 and np.size(a_g) == np.shape(a_q)[0] and np.size(a_g) > 1:
        da = dequantize_rows(a_q, a_sf_lin, a_g)
    else:
        da = dequantize(a_q, a_sf_lin, float(np.asarray(a_g).reshape(-1)[0]))
    dw = dequantize(w_q, w_sf_lin, w_g)
    out64 = np.matmul(da, dw.T)
    out16 = f64_to_f16(out64.reshape(-1)).reshape(out64.shape)
    return (out16, out64) if want_f64 else out16


def gemm_loops(a_q, a_sf_lin, a_g, w_q, w_sf_lin, w_g, want_f64: bool = False):
    """The same GEMM as three plain loops in C (fp64 sum in k order); for tiny shapes."""
    a = _c(a_q, np.uint8)
    w = _c(w_q, np.uint8)
    sa = _c(a_sf_lin, np.uint8)
    sw = _c(w_sf_lin, np.uint8)
    M, K2 = a.shape
    N = w.shape[0]
    K = K2 * 2
    assert w.shape[1] == K2 and sa.shape == (M, K // 16) and sw.shape == (N, K // 16)
    out16 = np.zeros((M, N), np.uint16)
    out64 = np.zeros((M, N), np.float64) if want_f64 else None
    lib().orc_gemm(_p(a), _p(sa), float(np.float32(a_g)), _p(w), _p(sw), float(np.float32(w_g)),
                   M, N, K, _p(out16), _p(out64) if want_f64 else None)
    return (out16, out64) if want_f64 else out16


def gemm_act_f32(a_q, a_sf32, w_q, w_sf_lin, w_scale, want_f64: bool = False):
    """The GEMM under the activation contract of "Fused Nvfp4 GEMM All Reduce Plugin"
    (TensorRT-Edge-LLM C++ API, inputs [1] activation_scale FP32 [B,1,K/16] and [4]
    weight_f32_scale): the activation's block scales arrive as combined fp32 values, and the
    weight's scalar fp32 scale multiplies, as a DequantizeLinear scale does:
        D = fp16_rn( sum_k E2M1(a[m,k]) * sa32[m,k/16] * E2M1(w[n,k]) * E4M3(sw[n,k/16]) * w_scale ).
    E2M1 values come from the dequantizer with unit scales (code 0x38 is 1.0); each product
    is exact in fp64; the sum by numpy's matmul; one rounding to fp16.
    a_q [M,K/2], a_sf32 fp32 [M,K/16] (or [M,1,K/16]), w_q [N,K/2], w_sf_lin [N,K/16]."""
    qa = _c(a_q, np.uint8)
    M, K2 = qa.shape
    K = 2 * K2
    s32 = np.asarray(a_sf32, dtype=np.float32).reshape(M, K // 16).astype(np.float64)
    e2m1_a = dequantize(qa, np.full((M, K // 16), 0x38, np.uint8), 1.0)
    da = e2m1_a * np.repeat(s32, 16, axis=1)
    dw = dequantize(w_q, w_sf_lin, 1.0) * float(np.float32(w_scale))
    out64 = np.matmul(da, dw.T)
    out16 = f64_to_f16(out64.reshape(-1)).reshape(out64.shape)
    return (out16, out64) if want_f64 else out16


def gemm_row_parallel(a_q, a_sf_lin, a_g, w_q, w_sf_lin, w_g, tp: int = 2,
                      want_f64: bool = False):
    """Row-parallel GEMM of "Fused Nvfp4 GEMM All Reduce Plugin" (TensorRT-Edge-LLM C++ API,
    tp_size 2): K is split into tp equal shards; rank r's local output is the GEMM over its
    shard rounded to fp16 (the plugin's rank-local FP16 [B,N]); the AllReduce sums the tp fp16
    outputs (fp64 sum, one rounding to fp16 -- for two ranks the correctly rounded sum).
    Returns fp16 bits [M,N], plus the fp64 sum of the unrounded partials when want_f64."""
    qa, qw = _c(a_q, np.uint8), _c(w_q, np.uint8)
    K = 2 * qa.shape[1]
    assert K % (64 * tp) == 0, "each shard must hold whole 64-element MMA steps"
    ks = K // tp
    parts16, sum64 = [], 0.0
    for r in range(tp):
        b0, b1, c0, c1 = r * ks // 2, (r + 1) * ks // 2, r * ks // 16, (r + 1) * ks // 16
        p16, p64 = gemm(qa[:, b0:b1], np.asarray(a_sf_lin)[:, c0:c1], a_g, qw[:, b0:b1],
                        np.asarray(w_sf_lin)[:, c0:c1], w_g, want_f64=True)
        parts16.append(p16.view(np.float16).astype(np.float64))
        sum64 = sum64 + p64
    total = parts16[0]
    for p in parts16[1:]:
        total = total + p
    out16 = f64_to_f16(total.reshape(-1)).reshape(total.shape)
    return (out16, sum64) if want_f64 else out16


# ----------------------------------------------------------------------------- traffic

def swiglu_quant_traffic_as_printed(N: int, H: int):
    """The SwiGLU + FP8 byte counts exactly as the SwiGLU/FP8 plugin write-up's steps print
    them ("The Cost of Non-Fused Quantization"): unfused = 8NH + 2NH + 2NH + NH,
    fused = 8NH + NH. Returns (unfused, fused, reduction)."""
    unfused = 8 * N * H + 2 * N * H + 2 * N * H + 1 * N * H
    fused = 8 * N * H + 1 * N * H
    return unfused, fused, 1.0 - fused / unfused


def swiglu_quant_traffic_from_shapes(N: int, H: int, out: str = "fp8"):
    """The same counts recomputed from the stated shapes (X is [N, 2H] bf16 = 4NH bytes).

    out='fp8': unfused = X + Y_w(bf16) + Y_r(bf16) + Q(fp8) = 4+2+2+1 = 9NH, fused = 5NH.
    out='nvfp4': fused = X + Q(NH/2) + scales(NH/16) = 4.5625 NH (unfused adds Y twice).
    Returns (unfused, fused) in bytes.
    """
    x_bytes = N * 2 * H * 2
    y_bf16 = N * H * 2
    if out == "fp8":
        q = N * H
    elif out == "nvfp4":
        q = N * H // 2 + N * H // 16
    else:
        raise ValueError(out)
    return x_bytes + 2 * y_bf16 + q, x_bytes + q
