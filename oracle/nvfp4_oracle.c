/*
 * nvfp4_oracle.c -- plain CPU oracle for the NVFP4 quantize + block-scaled FP4 GEMM path.
 *
 * TEST INFRASTRUCTURE ONLY. The library under nvfp4_block_scaled_10_b200/ never includes,
 * links, loads or calls anything in oracle/. Only tests/, __graft_entry__.smoke() and
 * bench.py's CPU-baseline / reference arm use it. The two share no code, header, table or
 * constant generator.
 *
 * Style: plain loops, no blocking, no vector tricks. Codecs are searches over the decoded
 * value grid (never bit manipulation of the encoded form). Quantize arithmetic is fp32 with
 * one IEEE round-to-nearest-even per operation, exactly as written (compile with
 * -ffp-contract=off, never -ffast-math). The GEMM sums in fp64.
 *
 * Sources (the pages define the operations but not the number formats):
 *  - E2M1 element format and the 16-element E4M3-scaled NVFP4 block: OCP Microscaling
 *    Formats (MX) v1.0, FP4 E2M1; NVIDIA NVFP4 (block of 16, UE4M3 scale, fp32 global scale).
 *  - E4M3 scale format: OCP 8-bit Floating Point Specification (OFP8), E4M3.
 *  - Block quantize (per-16 amax -> E4M3 scale -> exact division -> E2M1):
 *    "perf: optimize per-token nvfp4 quantization kernel" (FlashInfer PR #3237), review of
 *    quantization_utils.cuh (cvt_warp_fp16_to_fp4 / cvt_warp_fp16_to_fp4_with_vec_max and
 *    the exact, non-fast-math path).
 *  - Per-token global scale with the row read once: the same PR, description and
 *    invokeNvfp4QuantAndPerTokenScale.
 *  - 128x4 / 8x4 swizzled scale layouts: the same PR (get_sf_out_offset_128x4 /
 *    get_sf_out_offset_8x4) and "feature: add fp4 mm using trtllm backend" (FlashInfer PR
 *    #1355), description item 1. The byte order is the public cuBLAS block-scaling-factor
 *    layout (128x4) and its 8-row analogue (8x4, a reading).
 *  - Fused SwiGLU + quantize: "Building Custom TensorRT-LLM Plugins for Low-Latency FP8
 *    Inference at Scale", sections "The Cost of Non-Fused Quantization" and "Fusing the
 *    Kernel in CUDA" (SwiGLU in fp32 registers, Y never written).
 *  - GEMM contract ([B,K] FP4 activation, [N,K/16] FP8 weight scale, scalar FP32 global
 *    weight scale, FP16 [B,N] result): "Fused Nvfp4 GEMM All Reduce Plugin"
 *    (TensorRT-Edge-LLM C++ API), input/output tensor list.
 *
 * Parity pins live in tests/test_oracle_*.py. The 8x4 byte order (orc_sf_offset, layout 2)
 * is a reading, since the pages name the layout without its bytes. On CPU it is checked
 * against a second formulation of the same reading and for bijection; on the GPU both
 * swizzled layouts are checked against FlashInfer's fp4_quantize, the library of "feature:
 * add fp4 mm using trtllm backend" (tests/test_layout_library_gpu.py).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_SF_LINEAR 0
#define ORC_SF_128x4 1
#define ORC_SF_8x4 2

#define ORC_IN_BF16 0
#define ORC_IN_FP16 1

/* ------------------------------------------------------------------------------------ */
/* Input element types -> fp32 (both conversions are exact).                            */
/* ------------------------------------------------------------------------------------ */

/* bfloat16 is the top 16 bits of an IEEE binary32. */
float orc_bf16_to_f32(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* IEEE binary16: 1 sign, 5 exponent bits (bias 15), 10 mantissa bits. */
float orc_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
  } else if (e == 31) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
  }
  return (float)(sign ? -v : v);
}

static float load_elem(const uint16_t *x, int dtype, int64_t idx) {
  return dtype == ORC_IN_BF16 ? orc_bf16_to_f32(x[idx]) : orc_f16_to_f32(x[idx]);
}

/* ------------------------------------------------------------------------------------ */
/* E2M1 (OCP MX FP4): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN.  */
/* ------------------------------------------------------------------------------------ */

/* Value of a 4-bit code (bit 3 = sign). Exponent field 0 is subnormal: 0.5 * m. */
double orc_e2m1_value(int code) {
  int sign = (code >> 3) & 1;
  int e = (code >> 1) & 3;
  int m = code & 1;
  double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return sign ? -mag : mag;
}

/*
 * Round y to the nearest E2M1 value, ties to the even code (mantissa bit 0), with
 * saturation (|y| >= 6 -> 6, infinity included). The sign bit is kept, so a negative y
 * that rounds to zero gives -0 (code 0x8).
 */
int orc_e2m1_encode(float y) {
  int sign = signbit(y) ? 1 : 0;
  double a = fabs((double)y);
  int best = 7;
  if (!(a >= 6.0)) {
    double best_d = INFINITY;
    for (int c = 0; c < 8; ++c) {
      double d = fabs(a - orc_e2m1_value(c));
      if (d < best_d || (d == best_d && (c & 1) == 0)) {
        best = c;
        best_d = d;
      }
    }
  }
  return (sign << 3) | best;
}

/* ------------------------------------------------------------------------------------ */
/* E4M3 (OCP OFP8): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; S.1111.111 = NaN,  */
/* no infinities, largest finite 448 (0x7E).                                             */
/* ------------------------------------------------------------------------------------ */

double orc_e4m3_value(int code) {
  int sign = (code >> 7) & 1;
  int e = (code >> 3) & 15;
  int m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    mag = ldexp((double)m, -9); /* subnormal: (m/8) * 2^-6 */
  else
    mag = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  return sign ? -mag : mag;
}

/*
 * Encode a non-negative scale s as E4M3: nearest finite value, ties to the even code,
 * saturating (s >= 448, +inf included, -> 0x7E). Block scales are never negative; a NaN
 * input (never produced by the quantizer) maps to 0x7F.
 */
int orc_e4m3_encode(float s) {
  double a = (double)s;
  if (a != a) return 0x7F;
  if (a >= 448.0) return 0x7E;
  int best = 0;
  double best_d = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double d = fabs(a - orc_e4m3_value(c));
    if (d < best_d || (d == best_d && (c & 1) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return best;
}

/* ------------------------------------------------------------------------------------ */
/* fp64 -> IEEE binary16, round to nearest even, overflow to +-inf.                      */
/* ------------------------------------------------------------------------------------ */

uint16_t orc_f64_to_f16(double v) {
  uint16_t sign = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (a != a) return 0x7E00;
  if (a == 0.0) return sign;
  if (a >= 65520.0) return sign | 0x7C00; /* 65504 plus half its ulp (16) rounds to inf */
  /* Binade exponent e with 2^e <= a < 2^(e+1); below 2^-14 the spacing stays 2^-24. */
  int ex;
  frexp(a, &ex);
  int e = ex - 1;
  if (e < -14) e = -14;
  double q = ldexp(a, 10 - e); /* a / ulp, exact (power-of-two scaling) */
  double fl = floor(q);
  double rem = q - fl;
  double k = fl;
  if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) == 1.0)) k = fl + 1.0;
  /* k in [0, 2048]; k == 2048 carries into the next exponent, k < 1024 only when e == -14
     (subnormal): the exponent/mantissa sum below covers every case. */
  uint32_t bits = ((uint32_t)(e + 15) << 10) + (uint32_t)k - 1024u;
  return (uint16_t)(sign | bits);
}

/* ------------------------------------------------------------------------------------ */
/* Project-defined fp32 exponential e(x) used by SwiGLU.                                 */
/*                                                                                        */
/* The pages fix SwiGLU to fp32 registers but not an exp; bit-exact quantized output      */
/* needs one exact definition on both sides. Written from the mathematics:                */
/*   x clamped to [-87, 88] (keeps 2^k a normal number),                                  */
/*   k = the integer nearest the exact product x * fl(log2 e), ties to even (the product  */
/*       of two fp32 values is exact in double, so it is formed there and rounded once),  */
/*   f = x - k*ln2 with ln2 split hi/lo (Cody & Waite, "Software Manual for the           */
/*       Elementary Functions", 1980): hi = 0x3F317200 has 15 significant bits, so k*hi  */
/*       is exact for |k| <= 127,                                                         */
/*   p = degree-7 Taylor polynomial of e^f (coefficients 1/n! rounded to fp32), Horner    */
/*       with fused multiply-add,                                                         */
/*   e(x) = p * 2^k.                                                                      */
/* Every step is one IEEE fp32 operation with round-to-nearest-even.                      */
/* ------------------------------------------------------------------------------------ */

static const float ORC_LOG2E = 0x1.715476p+0f;   /* fp32(1/ln 2) */
static const float ORC_LN2_HI = 0x1.62e4p-1f;    /* 0.693145751953125 */
static const float ORC_LN2_LO = 0x1.7f7d1cp-20f; /* fp32(ln 2 - hi) */
static const float ORC_INV_FACT[8] = {
    1.0f,            /* 1/0! */
    1.0f,            /* 1/1! */
    0x1.0p-1f,       /* 1/2! */
    0x1.555556p-3f,  /* 1/3! */
    0x1.555556p-5f,  /* 1/4! */
    0x1.111112p-7f,  /* 1/5! */
    0x1.6c16c2p-10f, /* 1/6! */
    0x1.a01a02p-13f, /* 1/7! */
};

float orc_exp(float x) {
  if (x < -87.0f) x = -87.0f;
  if (x > 88.0f) x = 88.0f;
  double z = (double)x * (double)ORC_LOG2E; /* exact: 24 x 24 significant bits */
  float k = (float)rint(z);                  /* default rounding: to nearest, ties to even */
  float f = fmaf(-k, ORC_LN2_HI, x);
  f = fmaf(-k, ORC_LN2_LO, f);
  float p = ORC_INV_FACT[7];
  for (int n = 6; n >= 0; --n) p = fmaf(p, f, ORC_INV_FACT[n]);
  float two_k = ldexpf(1.0f, (int)k); /* exact: -126 <= k <= 127 */
  return p * two_k;
}

/* silu(v) = v * sigmoid(v) = v / (1 + e(-v)): one fp32 add and one IEEE division. */
float orc_silu(float v) { return v / (1.0f + orc_exp(-v)); }

/* y = silu(gate) * up, kept in fp32 (never rounded to bf16). */
float orc_swiglu_elem(float gate, float up) { return orc_silu(gate) * up; }

/* ------------------------------------------------------------------------------------ */
/* Scales.                                                                               */
/* ------------------------------------------------------------------------------------ */

/*
 * Global encode scale g = 448 * 6 / amax (E4M3 max times E2M1 max over the amax), so the
 * block that holds amax gets block scale 448. amax == 0 gives g = 1; an overflowing
 * quotient (amax below ~7.9e-36) is clamped to FLT_MAX so g stays finite.
 */
float orc_global_scale(float amax) {
  if (amax == 0.0f) return 1.0f;
  float g = 2688.0f / amax;
  if (g > FLT_MAX) g = FLT_MAX;
  return g;
}

float orc_amax(const uint16_t *x, int dtype, int64_t M, int64_t K, int64_t ldx) {
  float amax = 0.0f;
  for (int64_t r = 0; r < M; ++r)
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(load_elem(x, dtype, r * ldx + k));
      if (a > amax) amax = a;
    }
  return amax;
}

/*
 * Quantize one block of 16 fp32 values with global scale g:
 *   amax_b = max |x_i|
 *   s      = (amax_b / 6) * g             (two fp32 ops)
 *   s_enc  = E4M3(s),  s_dec = value(s_enc)
 *   r      = g / s_dec   (exact IEEE division; 0 when s_dec == 0; clamped to FLT_MAX)
 *   q_i    = E2M1(x_i * r)
 * Codes are returned unpacked, one per byte.
 */
void orc_quantize_block(const float *x16, float g, uint8_t *s_enc_out, uint8_t *q16) {
  float amax_b = 0.0f;
  for (int i = 0; i < 16; ++i) {
    float a = fabsf(x16[i]);
    if (a > amax_b) amax_b = a;
  }
  float s = (amax_b / 6.0f) * g;
  int s_enc = orc_e4m3_encode(s);
  float s_dec = (float)orc_e4m3_value(s_enc);
  float r = (s_dec == 0.0f) ? 0.0f : g / s_dec;
  if (r > FLT_MAX) r = FLT_MAX;
  for (int i = 0; i < 16; ++i) {
    float y = x16[i] * r;
    q16[i] = (uint8_t)orc_e2m1_encode(y);
  }
  *s_enc_out = (uint8_t)s_enc;
}

/* Packing: byte j of a row holds element 2j in its low nibble and 2j+1 in its high nibble. */
static void pack_row(const uint8_t *codes, int64_t K, uint8_t *q) {
  for (int64_t j = 0; j < K / 2; ++j)
    q[j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
}

/*
 * Quantize X [M,K] (row stride ldx elements). per_token == 0: g[0] is read.
 * per_token == 1: g[r] = global_scale(max_k |x[r,k]|) is written for every row.
 * q: [M, K/2] packed bytes (row stride K/2). sf: [M, K/16] linear E4M3 codes.
 */
void orc_quantize(const uint16_t *x, int dtype, int64_t M, int64_t K, int64_t ldx, float *g,
                  int per_token, uint8_t *q, uint8_t *sf) {
  float xb[16];
  uint8_t codes[16];
  for (int64_t r = 0; r < M; ++r) {
    float gr;
    if (per_token) {
      gr = orc_global_scale(orc_amax(x + r * ldx, dtype, 1, K, ldx));
      g[r] = gr;
    } else {
      gr = g[0];
    }
    for (int64_t b = 0; b < K / 16; ++b) {
      for (int i = 0; i < 16; ++i) xb[i] = load_elem(x, dtype, r * ldx + b * 16 + i);
      orc_quantize_block(xb, gr, &sf[r * (K / 16) + b], codes);
      pack_row(codes, 16, &q[r * (K / 2) + b * 8]);
    }
  }
}

/* Y = silu(gate) * up for X [M, 2H] = [gate | up] (row stride ldx), fp32 out [M, H]. */
void orc_swiglu(const uint16_t *x, int dtype, int64_t M, int64_t H, int64_t ldx, float *y) {
  for (int64_t r = 0; r < M; ++r)
    for (int64_t h = 0; h < H; ++h)
      y[r * H + h] =
          orc_swiglu_elem(load_elem(x, dtype, r * ldx + h), load_elem(x, dtype, r * ldx + H + h));
}

/* Fused SwiGLU + quantize with a given per-tensor g: Y is formed per block, never stored. */
void orc_swiglu_quantize(const uint16_t *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                         float g, uint8_t *q, uint8_t *sf) {
  float yb[16];
  uint8_t codes[16];
  for (int64_t r = 0; r < M; ++r)
    for (int64_t b = 0; b < H / 16; ++b) {
      for (int i = 0; i < 16; ++i) {
        int64_t h = b * 16 + i;
        yb[i] = orc_swiglu_elem(load_elem(x, dtype, r * ldx + h),
                                load_elem(x, dtype, r * ldx + H + h));
      }
      orc_quantize_block(yb, g, &sf[r * (H / 16) + b], codes);
      pack_row(codes, 16, &q[r * (H / 2) + b * 8]);
    }
}

/*
 * FP8 E4M3 with sign (OCP OFP8 E4M3): NaN -> 0x7F; otherwise the sign bit (bit 7, kept for
 * -0 and for negatives that round to zero) and the saturating magnitude code of |v|, round
 * to nearest even, |v| >= 448 (infinity included) -> 448.
 */
int orc_e4m3_encode_signed(float v) {
  if (v != v) return 0x7F;
  const int sign = signbit(v) ? 0x80 : 0;
  return sign | orc_e4m3_encode(fabsf(v));
}

/*
 * Fused SwiGLU + FP8 E4M3 quantize ("Building Custom TensorRT-LLM Plugins for Low-Latency FP8
 * Inference at Scale", "Fusing the Kernel in CUDA": SwiGLU in fp32, the quantization scale
 * applied, saturation to +-448): q[r, h] = E4M3(fl(y[r, h] * scale)), y = silu(gate) * up in
 * fp32, q [M, H] row-major. The scale multiplies, as the NVFP4 encode scales do here.
 */
void orc_swiglu_fp8(const uint16_t *x, int dtype, int64_t M, int64_t H, int64_t ldx, float scale,
                    uint8_t *q) {
  for (int64_t r = 0; r < M; ++r)
    for (int64_t h = 0; h < H; ++h) {
      const float y =
          orc_swiglu_elem(load_elem(x, dtype, r * ldx + h), load_elem(x, dtype, r * ldx + H + h));
      q[r * H + h] = (uint8_t)orc_e4m3_encode_signed(y * scale);
    }
}

void orc_e4m3_encode_signed_array(const float *v, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)orc_e4m3_encode_signed(v[i]);
}

/* amax of Y = silu(gate) * up (used to pick the per-tensor g for the fused kernel). */
float orc_swiglu_amax(const uint16_t *x, int dtype, int64_t M, int64_t H, int64_t ldx) {
  float amax = 0.0f;
  for (int64_t r = 0; r < M; ++r)
    for (int64_t h = 0; h < H; ++h) {
      float a = fabsf(orc_swiglu_elem(load_elem(x, dtype, r * ldx + h),
                                      load_elem(x, dtype, r * ldx + H + h)));
      if (a > amax) amax = a;
    }
  return amax;
}

/* ------------------------------------------------------------------------------------ */
/* Scale-factor layouts.                                                                  */
/*   linear: [R, C], offset r*C + c.                                                      */
/*   128x4 : R' = ceil(R/128)*128, C' = ceil(C/4)*4; 512-byte atoms of 128 rows x 4       */
/*           columns; within an atom row r%32 strides 16 B, row group (r/32)%4 strides    */
/*           4 B, column c%4 strides 1 B; atoms ordered row-block major, then c/4.        */
/*   8x4   : R' = ceil(R/8)*8, C' = ceil(C/4)*4; 32-byte atoms of 8 rows x 4 columns;     */
/*           row r%8 strides 4 B, column c%4 strides 1 B; atoms row-block major.          */
/* Padding bytes (r >= R or c >= C) are zero.                                            */
/* ------------------------------------------------------------------------------------ */

static int64_t ceil_to(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

int64_t orc_sf_rows_padded(int layout, int64_t R) {
  if (layout == ORC_SF_128x4) return ceil_to(R, 128);
  if (layout == ORC_SF_8x4) return ceil_to(R, 8);
  return R;
}

int64_t orc_sf_cols_padded(int layout, int64_t C) {
  if (layout == ORC_SF_LINEAR) return C;
  return ceil_to(C, 4);
}

int64_t orc_sf_bytes(int layout, int64_t R, int64_t C) {
  return orc_sf_rows_padded(layout, R) * orc_sf_cols_padded(layout, C);
}

int64_t orc_sf_offset(int layout, int64_t r, int64_t c, int64_t R, int64_t C) {
  int64_t Cp = orc_sf_cols_padded(layout, C);
  (void)R;
  if (layout == ORC_SF_128x4) {
    int64_t atom = (r / 128) * (Cp / 4) + (c / 4);
    return atom * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4);
  }
  if (layout == ORC_SF_8x4) {
    int64_t atom = (r / 8) * (Cp / 4) + (c / 4);
    return atom * 32 + (r % 8) * 4 + (c % 4);
  }
  return r * C + c;
}

/* lin [R, C] -> out (orc_sf_bytes bytes), padding zeroed. */
void orc_sf_swizzle(const uint8_t *lin, int64_t R, int64_t C, int layout, uint8_t *out) {
  int64_t Rp = orc_sf_rows_padded(layout, R), Cp = orc_sf_cols_padded(layout, C);
  for (int64_t r = 0; r < Rp; ++r)
    for (int64_t c = 0; c < Cp; ++c) {
      uint8_t v = (r < R && c < C) ? lin[r * C + c] : 0;
      out[orc_sf_offset(layout, r, c, R, C)] = v;
    }
}

/* in (orc_sf_bytes bytes) -> lin [R, C]. */
void orc_sf_unswizzle(const uint8_t *in, int64_t R, int64_t C, int layout, uint8_t *lin) {
  for (int64_t r = 0; r < R; ++r)
    for (int64_t c = 0; c < C; ++c) lin[r * C + c] = in[orc_sf_offset(layout, r, c, R, C)];
}

/* ------------------------------------------------------------------------------------ */
/* Dequantized GEMM.                                                                      */
/*   deq(a)[m,k] = E2M1(a[m,k]) * E4M3(sa[m,k/16]) / ga                                   */
/*   deq(w)[n,k] = E2M1(w[n,k]) * E4M3(sw[n,k/16]) / gw                                   */
/*   D[m,n]      = fp16_rn( sum_k deq(a)[m,k] * deq(w)[n,k] )   (sum in fp64)             */
/* a: [M, K/2] packed, sa: [M, K/16] linear; w: [N, K/2] packed, sw: [N, K/16] linear.    */
/* out16 [M, N] fp16 bits (row stride N); out64 (optional) the fp64 sums.                 */
/* ------------------------------------------------------------------------------------ */

static double elem_value(const uint8_t *packed_row, int64_t k) {
  uint8_t byte = packed_row[k / 2];
  int code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
  return orc_e2m1_value(code);
}

void orc_gemm(const uint8_t *a, const uint8_t *sa, float ga, const uint8_t *w, const uint8_t *sw,
              float gw, int64_t M, int64_t N, int64_t K, uint16_t *out16, double *out64) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double da = elem_value(a + m * (K / 2), k) * orc_e4m3_value(sa[m * (K / 16) + k / 16]) /
                    (double)ga;
        double dw = elem_value(w + n * (K / 2), k) * orc_e4m3_value(sw[n * (K / 16) + k / 16]) /
                    (double)gw;
        acc += da * dw;
      }
      if (out64) out64[m * N + n] = acc;
      if (out16) out16[m * N + n] = orc_f64_to_f16(acc);
    }
}

/*
 * Dequantize a packed operand: out[r, k] = E2M1(q[r, k]) * E4M3(s[r, k/16]) / g in fp64
 * (the same expression the loop GEMM above uses for each factor).
 */
void orc_dequantize(const uint8_t *q, const uint8_t *s, float g, int64_t rows, int64_t K,
                    double *out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k)
      out[r * K + k] =
          elem_value(q + r * (K / 2), k) * orc_e4m3_value(s[r * (K / 16) + k / 16]) / (double)g;
}

/*
 * The same with one encode scale per row (an operand quantized per token): out[r, k] =
 * E2M1(q[r, k]) * E4M3(s[r, k/16]) / g[r].
 */
void orc_dequantize_rows(const uint8_t *q, const uint8_t *s, const float *g, int64_t rows,
                         int64_t K, double *out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k)
      out[r * K + k] = elem_value(q + r * (K / 2), k) * orc_e4m3_value(s[r * (K / 16) + k / 16]) /
                       (double)g[r];
}

/* ------------------------------------------------------------------------------------ */
/* Array helpers for the pin tests (elementwise loops over the scalar definitions).       */
/* ------------------------------------------------------------------------------------ */

void orc_e2m1_encode_array(const float *y, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)orc_e2m1_encode(y[i]);
}

void orc_e4m3_encode_array(const float *s, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)orc_e4m3_encode(s[i]);
}

void orc_exp_array(const float *x, int64_t n, float *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_exp(x[i]);
}

void orc_silu_array(const float *x, int64_t n, float *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_silu(x[i]);
}

void orc_f64_to_f16_array(const double *v, int64_t n, uint16_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_f64_to_f16(v[i]);
}

void orc_f16_to_f32_array(const uint16_t *h, int64_t n, float *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_f16_to_f32(h[i]);
}
