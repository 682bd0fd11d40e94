// quantize.cu -- NVFP4 quantization kernels for sm_100a (memory-bound, CUDA cores).
//
//  * global amax -> per-tensor encode scale g (two launches, partial maxima in workspace)
//  * streaming quantize: one thread owns one 16-element block (one 32-byte load), given g
//    per tensor or per row
//  * per-token quantize: one row per CTA at a time held in registers (the next row streams
//    into the registers as they free), row amax -> g_row, then the blocks of the row are
//    quantized from the same registers, so X is read from HBM once (rows longer than
//    32768 elements take a two-pass path that reads X twice)
//  * fused SwiGLU + quantize: y = silu(gate) * up formed in registers, never stored
//  * scale-layout swizzle / unswizzle
//
// Block math (exact path of the per-token NVFP4 quantize PR, FlashInfer #3237): amax_b;
// s = (amax_b / 6) * g; E4M3 with saturation; r = g / s_dec by IEEE division; q = E2M1(x*r).
// All fp32 steps use the explicit round-to-nearest intrinsics so no FMA contraction or
// approximate division can change a bit.
#include <cfloat>
#include <cstdint>

#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"
#include "swiglu_math.cuh"

namespace nvfp4 {

// Sticky error word of the quantize kernels (bit kDevErrTimeout: a bounded wait gave up).
__device__ int g_device_error = 0;

int *device_error_symbol() {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return static_cast<int *>(p);
}

// ------------------------------------------------------------------------------ helpers

__device__ __forceinline__ float global_scale_from_amax(float amax) {
  if (amax == 0.0f) return 1.0f;
  return fminf(__fdiv_rn(2688.0f, amax), FLT_MAX);
}

// Byte offset of scale (r, c) in the given layout; Cp = padded column count.
__device__ __forceinline__ int64_t sf_offset(int layout, int64_t r, int64_t c, int64_t C,
                                             int64_t Cp) {
  if (layout == kSf128x4) {
    const int64_t atom = (r >> 7) * (Cp >> 2) + (c >> 2);
    return (atom << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (c & 3);
  }
  if (layout == kSf8x4) {
    const int64_t atom = (r >> 3) * (Cp >> 2) + (c >> 2);
    return (atom << 5) + ((r & 7) << 2) + (c & 3);
  }
  return r * C + c;
}

// fl(x / 6) for x >= 0 (a block maximum), the IEEE quotient, without the general division
// sequence: q0 = fl(x * fl(1/6)), rem = x - 6*q0 by one FMA, q1 = q0 + rem*fl(1/6) by one
// FMA. An exhaustive check over every fp32 bit pattern with a clear sign bit finds q1
// equal to the IEEE quotient for +0 and every finite x >= 2^-125 (NaN and infinity keep
// q0, which is then the quotient too); for 0 < x < 2^-125 the quotient is subnormal and the
// IEEE division is used.
__device__ __forceinline__ float div6_rn(float x) {
  if (x > 0.0f && x < 0x1p-125f) return __fdiv_rn(x, 6.0f);
  constexpr float kSixth = 0x1.555556p-3f;  // fl(1/6)
  const float q0 = __fmul_rn(x, kSixth);
  const float rem = __fmaf_rn(-q0, 6.0f, x);
  const float q1 = __fmaf_rn(rem, kSixth, q0);
  return (rem == rem) ? q1 : q0;
}

// E4M3 block scale of a block with maximum magnitude `amax` under encode scale g:
// s = (amax / 6) * g (two IEEE roundings), saturating E4M3 code.
__device__ __forceinline__ uint32_t block_scale_code(float amax, float g) {
  return cvt_e4m3(__fmul_rn(div6_rn(amax), g));
}

// Per-row reciprocal table for one warp: lane k (1..15) holds fl(g / k), lane 0 holds 0.
// Every finite E4M3 value is k * 2^E with an integer k in 0..15 (k = 8 + mantissa for a
// normal code with E = exponent - 10, k = mantissa with E = -9 for a subnormal code), so
// g / value = fl(g / k) * 2^-E exactly whenever the product is a normal float, and an
// overflow of the product is exactly an overflow of the quotient. For every g that
// global_scale_from_amax yields from a bf16 or fp16 maximum the products are normal; an
// exhaustive check over those g and all 127 codes finds the table equal to the division.
__device__ __forceinline__ float row_recip_lane(float g) {
  const int k = static_cast<int>(lane_id());
  return (k == 0 || k > 15) ? 0.0f : __fdiv_rn(g, static_cast<float>(k));
}

// r = g / value(code) from the warp's row table (all 32 lanes must call it together).
__device__ __forceinline__ float row_recip(uint32_t code, float lane_tab) {
  const uint32_t e = code >> 3, m = code & 7u;
  const int k = static_cast<int>(e ? (8u | m) : m);
  const float t = __shfl_sync(0xffffffffu, lane_tab, k);
  const float p2 = __uint_as_float((137u - (e ? e : 1u)) << 23);  // 2^(10 - max(e, 1))
  return fminf(__fmul_rn(t, p2), FLT_MAX);
}

// r = g / value(code) (IEEE division), 0 for a zero scale, clamped to FLT_MAX.
__device__ __forceinline__ float block_recip(uint32_t code, float g) {
  const float s_dec = e4m3_to_f32(code);
  return (s_dec == 0.0f) ? 0.0f : fminf(__fdiv_rn(g, s_dec), FLT_MAX);
}

// Packs E2M1(x_i * r) for the 16 elements of 8 packed 16-bit words (element 2j in the low
// nibble of byte j).
template <int DTYPE>
__device__ __forceinline__ uint64_t quant_packed16(const uint32_t (&w)[8], float r) {
  float y[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float lo, hi;
    unpack2<DTYPE>(w[i], lo, hi);
    mul2_rn(lo, hi, r, y[2 * i], y[2 * i + 1]);
  }
  const uint32_t a = e2m1x8_from_pairs(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
  const uint32_t b = e2m1x8_from_pairs(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
  return (static_cast<uint64_t>(b) << 32) | a;
}

// Same for 16 fp32 values.
__device__ __forceinline__ uint64_t quant_f32x16(const float (&x)[16], float r) {
  float y[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) mul2_rn(x[2 * i], x[2 * i + 1], r, y[2 * i], y[2 * i + 1]);
  const uint32_t a = e2m1x8_from_pairs(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
  const uint32_t b = e2m1x8_from_pairs(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
  return (static_cast<uint64_t>(b) << 32) | a;
}

// Per-CTA table of r for every finite E4M3 scale code under one encode scale g
// (128 entries; entry 0x7F is never indexed: codes come from a saturating conversion).
__device__ __forceinline__ void fill_recip_table(float *table, float g) {
  for (int c = threadIdx.x; c < 128; c += blockDim.x) table[c] = (c == 0x7F) ? 0.0f : block_recip(c, g);
}

// Byte offset of row r's scale for column c = 0 (the per-row part of sf_offset).
__device__ __forceinline__ int64_t sf_row_base(int layout, int64_t r, int64_t C, int64_t Cp) {
  if (layout == kSf128x4) return ((r >> 7) * (Cp >> 2) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2);
  if (layout == kSf8x4) return ((r >> 3) * (Cp >> 2) << 5) + ((r & 7) << 2);
  return r * C;
}

// Column part of sf_offset (add to sf_row_base).
__device__ __forceinline__ int64_t sf_col_off(int layout, int64_t c) {
  if (layout == kSf128x4) return ((c >> 2) << 9) + (c & 3);
  if (layout == kSf8x4) return ((c >> 2) << 5) + (c & 3);
  return c;
}

template <int DTYPE>
__device__ __forceinline__ void unpack16(const uint32_t (&w)[8], float (&y)[16]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) unpack2<DTYPE>(w[i], y[2 * i], y[2 * i + 1]);
}

// Writes zeros into the padding of a scale buffer: rows [M, Rp) x [0, Cp) and
// rows [0, M) x [C, Cp). Grid-strided over all threads of the launch.
__device__ void zero_sf_padding(uint8_t *sf, int layout, int64_t M, int64_t C, int64_t Rp,
                                int64_t Cp) {
  const int64_t row_pad = (Rp - M) * Cp;
  const int64_t col_pad = M * (Cp - C);
  const int64_t total = row_pad + col_pad;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; p < total;
       p += stride) {
    int64_t r, c;
    if (p < row_pad) {
      r = M + p / Cp;
      c = p % Cp;
    } else {
      const int64_t p2 = p - row_pad;
      r = p2 / (Cp - C);
      c = C + p2 % (Cp - C);
    }
    sf[sf_offset(layout, r, c, C, Cp)] = 0;
  }
}

// Block-level max over all threads (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ float block_max(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  __syncthreads();  // `red` may still be read from a previous call
  if (lane_id() == 0) red[warp] = v;
  __syncthreads();
  float m = 0.0f;
  for (int w = 0; w < nwarps; ++w) m = fmaxf(m, red[w]);
  return m;
}

// ------------------------------------------------------------------------------ amax

template <int DTYPE, bool V8>
__global__ void __launch_bounds__(256) amax_partial_kernel(const uint16_t *__restrict__ x,
                                                          int64_t M, int64_t K, int64_t ldx,
                                                          float *__restrict__ partial) {
  __shared__ float red[32];
  const int64_t C = K / 16;
  const int64_t nblk = M * C;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float m = 0.0f;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nblk;
       b += stride) {
    const int64_t r = b / C, c = b - r * C;
    uint32_t w[8];
    ld_block16<V8>(x + r * ldx + c * 16, w);
    float y[16];
    unpack16<DTYPE>(w, y);
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(y[i]));
  }
  m = block_max(m, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = m;
}

__global__ void __launch_bounds__(1024) amax_finalize_kernel(const float *__restrict__ partial,
                                                            int n, float *__restrict__ g_out) {
  __shared__ float red[32];
  float m = 0.0f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, partial[i]);
  m = block_max(m, red);
  if (threadIdx.x == 0) g_out[0] = global_scale_from_amax(m);
}

// ------------------------------------------------------------------------------ streaming

// Row-major streaming quantize: CTA b handles rows b, b + gridDim.x, ...; thread t owns
// blocks t, t + blockDim.x, ... of each row (one 32-byte block per load), UNROLL blocks in
// flight per thread. g_per_row == 0: g[0] for every row (r from a per-CTA table of all E4M3
// codes); == 1: g[r] (r by division).
template <int DTYPE, int UNROLL, bool V8>
__global__ void __launch_bounds__(256) quant_stream_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, const float *__restrict__ g,
    int g_per_row, uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int layout, int64_t Rp,
    int64_t Cp) {
  __shared__ float rtab[128];
  const int C = static_cast<int>(K / 16);
  const float g0 = g_per_row ? 0.0f : g[0];
  if (!g_per_row) fill_recip_table(rtab, g0);
  __syncthreads();
  const int step = blockDim.x * UNROLL;
  for (int64_t r = blockIdx.x; r < M; r += gridDim.x) {
    const uint16_t *xrow = x + r * ldx;
    uint8_t *qrow = q + r * (K / 2);
    uint8_t *sfrow = sf + sf_row_base(layout, r, C, Cp);
    const float gr = g_per_row ? g[r] : g0;
    for (int c0 = threadIdx.x; c0 < C; c0 += step) {
      uint32_t w[UNROLL][8];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int c = c0 + u * blockDim.x;
        if (c < C) ld_block16<V8>(xrow + c * 16, w[u]);
      }
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int c = c0 + u * blockDim.x;
        if (c < C) {
          const float amax = amax16_packed<DTYPE>(w[u]);
          const uint32_t s = block_scale_code(amax, gr);
          const float rr = g_per_row ? block_recip(s, gr) : rtab[s];
          st_cs_u64(qrow + c * 8, quant_packed16<DTYPE>(w[u], rr));
          sfrow[sf_col_off(layout, c)] = static_cast<uint8_t>(s);
        }
      }
    }
  }
  zero_sf_padding(sf, layout, M, C, Rp, Cp);
}

// Row amax -> g[r] (two-pass per-token path for rows too long to stage on chip).
template <int DTYPE, bool V8>
__global__ void __launch_bounds__(256) row_scale_kernel(const uint16_t *__restrict__ x, int64_t M,
                                                       int64_t K, int64_t ldx,
                                                       float *__restrict__ g) {
  __shared__ float red[32];
  const int64_t C = K / 16;
  for (int64_t r = blockIdx.x; r < M; r += gridDim.x) {
    float m = 0.0f;
    for (int64_t c = threadIdx.x; c < C; c += blockDim.x) {
      uint32_t w[8];
      ld_block16<V8>(x + r * ldx + c * 16, w);
      float y[16];
      unpack16<DTYPE>(w, y);
#pragma unroll
      for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(y[i]));
    }
    m = block_max(m, red);
    if (threadIdx.x == 0) g[r] = global_scale_from_amax(m);
  }
}

// ------------------------------------------------------------------------------ per-token

// Persistent, one row per CTA at a time: CTA b handles rows b, b + gridDim.x, ... Thread t
// owns blocks t + i * NT (i < BPT) of a row and holds them in registers, so the row is read
// from HBM once: block maxima from registers, one CTA barrier for the row maximum, then the
// blocks are quantized from the same registers. As soon as block i of the current row has
// been quantized, block i of the CTA's next row is loaded into the registers it occupied,
// so the next row streams in while the rest of this one is being quantized. (Staging the
// rows in shared memory by bulk copies with a deeper ring measured slower than this on
// 8192 x 7168 bf16 rows.)
template <int DTYPE, int BPT>
__device__ __forceinline__ void load_row_blocks(const uint16_t *xrow, int C, int nt, bool v8,
                                                uint32_t (&w)[BPT][8]) {
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    const int c = static_cast<int>(threadIdx.x) + i * nt;
    if (c < C) {
      if (v8) ld_block16<true>(xrow + c * 16, w[i]);
      else ld_block16<false>(xrow + c * 16, w[i]);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) w[i][k] = 0u;  // zero blocks: amax 0, scale code 0
    }
  }
}

template <int DTYPE, int BPT, int NT, int MINB>
__global__ void __launch_bounds__(NT, MINB) quant_pertoken_regs_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float *__restrict__ g,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int layout, int64_t Rp, int64_t Cp,
    bool v8) {
  __shared__ float red[2][NT / 32];
  const int C = static_cast<int>(K / 16);
  const int warp = threadIdx.x >> 5;

  uint32_t w[BPT][8];
  int64_t r = blockIdx.x;
  const int64_t step = gridDim.x;
  if (r < M) load_row_blocks<DTYPE, BPT>(x + r * ldx, C, NT, v8, w);
  zero_sf_padding(sf, layout, M, C, Rp, Cp);

  for (uint32_t j = 0; r < M; r += step, ++j) {
    float bam[BPT];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      bam[i] = amax16_packed<DTYPE>(w[i]);
      m = fmaxf(m, bam[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    // red is double-buffered by row parity: row j + 2 writes this half only after every
    // thread has passed row j + 1's barrier, i.e. after all reads of row j's partials.
    if (lane_id() == 0) red[j & 1][warp] = m;
    __syncthreads();
    float amax = red[j & 1][0];
#pragma unroll
    for (int w2 = 1; w2 < NT / 32; ++w2) amax = fmaxf(amax, red[j & 1][w2]);
    const float gr = global_scale_from_amax(amax);
    if (threadIdx.x == 0) g[r] = gr;
    const float tab = row_recip_lane(gr);

    uint8_t *qrow = q + r * (K / 2);
    uint8_t *sfrow = sf + sf_row_base(layout, r, C, Cp);
    const int64_t rn = r + step;
    const uint16_t *xn = x + rn * ldx;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int c = static_cast<int>(threadIdx.x) + i * NT;
      // out-of-row slots carry zero blocks (code 0) and still join the table shuffle
      const uint32_t s = block_scale_code(bam[i], gr);
      const float rr = row_recip(s, tab);
      if (c < C) {
        st_cs_u64(qrow + c * 8, quant_packed16<DTYPE>(w[i], rr));
        sfrow[sf_col_off(layout, c)] = static_cast<uint8_t>(s);
        if (rn < M) {
          if (v8) ld_block16<true>(xn + c * 16, w[i]);
          else ld_block16<false>(xn + c * 16, w[i]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------ SwiGLU

// SiLU table for bfloat16 gates. silu(gate) depends on the 16-bit gate alone, so each CTA of
// the fused SwiGLU kernels first evaluates it once for every bf16 gate with 2^-26 <= |gate| <
// 2^7 (biased exponents 101..133, both signs: 8448 values, 33 KB of shared memory) with the
// same arithmetic as the per-element path (silu_pair_neg, whose forms agree bit for bit on
// every gate), and then looks silu up instead of evaluating the exponential and the division
// per element. A block takes the table path when all 16 gates are numbers inside that range
// (a NaN-propagating packed maximum and a packed minimum of |gate| decide it); any other block
// (zeros, tiny, huge, infinite or NaN gates) evaluates silu per element as before.
constexpr uint32_t kSiluTabLo = 0x3280u;  // bf16 magnitude bits of 2^-26
constexpr uint32_t kSiluTabHi = 0x4300u;  // bf16 magnitude bits of 2^7 (first value past the table)
constexpr uint32_t kSiluTabHalf = kSiluTabHi - kSiluTabLo;  // 4224 entries per sign
constexpr int kSiluTabEntries = 2 * kSiluTabHalf;            // positive gates, then negative
constexpr int kSiluTabBytes = kSiluTabEntries * 4;

// Fills the table (all threads of the CTA; the caller synchronises before any lookup).
__device__ __forceinline__ void build_silu_table(float *tab) {
  for (int j = 2 * static_cast<int>(threadIdx.x); j < kSiluTabEntries; j += 2 * blockDim.x) {
    // entries j and j + 1 hold the same sign (kSiluTabHalf is even)
    const uint32_t mag = kSiluTabLo + static_cast<uint32_t>(j) % kSiluTabHalf;
    const uint32_t sign = j < static_cast<int>(kSiluTabHalf) ? 0u : 0x80000000u;
    // silu_pair_neg takes -gate; a bf16 pattern is the upper half of its fp32 value
    const F2 v{__uint_as_float((mag << 16) ^ sign ^ 0x80000000u),
               __uint_as_float(((mag + 1u) << 16) ^ sign ^ 0x80000000u)};
    const F2 sv = silu_pair_neg<true, false>(v);
    tab[j] = sv.x;
    tab[j + 1] = sv.y;
  }
}

// True when every one of the 16 bf16 gates of a block is a number with 2^-26 <= |gate| < 2^7.
__device__ __forceinline__ bool silu_table_covers(const uint32_t (&w)[8]) {
  uint32_t hi0 = w[0], hi1 = w[1], lo0 = w[0], lo1 = w[1];
#pragma unroll
  for (int i = 2; i < 8; i += 2) {
    asm("max.NaN.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(hi0) : "r"(w[i]));
    asm("max.NaN.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(hi1) : "r"(w[i + 1]));
    asm("min.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(lo0) : "r"(w[i]));
    asm("min.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(lo1) : "r"(w[i + 1]));
  }
  asm("max.NaN.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(hi0) : "r"(hi1));
  asm("min.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(lo0) : "r"(lo1));
  // clear the signs xorsign left; a NaN magnitude compares above kSiluTabHi too
  const uint32_t hmax = hi0 & 0x7FFF7FFFu, hmin = lo0 & 0x7FFF7FFFu;
  return max(hmax & 0xFFFFu, hmax >> 16) < kSiluTabHi && min(hmin & 0xFFFFu, hmin >> 16) >= kSiluTabLo;
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// y = silu(gate) * up for one block from the table (silu_table_covers(wg) must hold; tab is
// the table's shared-memory address). Returns max |y|. For a packed pair of gates the two
// table indices come out of one 32-bit computation with 16-bit lanes: idx = magnitude -
// kSiluTabLo, plus kSiluTabHalf for a negative gate, i.e. bits - kSiluTabLo - sign * (0x8000 -
// kSiluTabHalf); no lane borrows from or carries into the other for gates in the table.
__device__ __forceinline__ float swiglu_block16_tab(const uint32_t (&wg)[8], const uint32_t (&wu)[8],
                                                    uint32_t tab, float (&y)[16]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t s2 = (wg[i] >> 15) & 0x00010001u;
    const uint32_t idx2 = wg[i] - (kSiluTabLo | (kSiluTabLo << 16)) - s2 * (0x8000u - kSiluTabHalf);
    const uint32_t off2 = idx2 << 2;  // byte offsets, each below 2^16
    const F2 sv{lds_f32(tab + (off2 & 0xFFFFu)), lds_f32(tab + (off2 >> 16))};
    F2 up;
    unpack2<0>(wu[i], up.x, up.y);
    const F2 v = mul2f_rn(sv, up);
    y[2 * i] = v.x;
    y[2 * i + 1] = v.y;
    amax = fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y)));
  }
  return amax;
}

// y = silu(gate) * up for the 16 elements of one block (8 packed words of each half);
// returns max |y|.
template <int DTYPE, bool CLAMP, bool SAFE>
__device__ __forceinline__ float swiglu_block16(const uint32_t (&wg)[8], const uint32_t (&wu)[8],
                                                float (&y)[16]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    F2 up;
    unpack2<DTYPE>(wu[i], up.x, up.y);
    const F2 v = mul2f_rn(silu_pair_neg<CLAMP, SAFE>(unpack2_neg<DTYPE>(wg[i])), up);
    y[2 * i] = v.x;
    y[2 * i + 1] = v.y;
    amax = fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y)));
  }
  return amax;
}

// Persistent: the work items are (row, chunk) pairs, a chunk being NT * UNROLL consecutive
// output blocks of a row, dealt round-robin to the CTAs (the row count of the workloads is
// not a multiple of the grid, so whole rows would leave a long tail). Thread t owns blocks
// t + u * NT (u < UNROLL) of the chunk; gate and up are loaded as two 32-byte blocks each.
// Once y of block u is formed, block u of the CTA's next item is loaded into the registers
// it held, so the next item streams in while this one is quantized. Per block the packed
// maximum |gate| picks the cheapest silu form that is exact for it.
template <int DTYPE, int UNROLL, bool V8>
__device__ __forceinline__ void load_swiglu_item(const uint16_t *x, int64_t ldx, int64_t H, int C,
                                                 int64_t r, int c0, int nt, uint32_t (&wg)[UNROLL][8],
                                                 uint32_t (&wu)[UNROLL][8]) {
  const uint16_t *grow = x + r * ldx;
#pragma unroll
  for (int u = 0; u < UNROLL; ++u) {
    const int c = c0 + u * nt;
    if (c < C) {
      ld_block16<V8>(grow + c * 16, wg[u]);
      ld_block16<V8>(grow + H + c * 16, wu[u]);
    }
  }
}

template <int DTYPE, int UNROLL, bool V8, int NT, int MINB>
__global__ void __launch_bounds__(NT, MINB) swiglu_quant_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t H, int64_t ldx, const float *__restrict__ g,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int layout, int64_t Rp, int64_t Cp,
    int chunks_per_row) {
  __shared__ float rtab[128];
  extern __shared__ float silu_tab[];  // bf16 input: the SiLU table (kSiluTabBytes)
  const int C = static_cast<int>(H / 16);
  const float g0 = g[0];
  // item = blockIdx.x + k * gridDim.x as (row r, chunk ch), advanced without a division
  const int64_t step_r = gridDim.x / chunks_per_row;
  const int step_ch = static_cast<int>(gridDim.x % chunks_per_row);
  int64_t r = blockIdx.x / chunks_per_row;
  int ch = static_cast<int>(blockIdx.x % chunks_per_row);
  uint32_t wg[UNROLL][8], wu[UNROLL][8];
  if (r < M) load_swiglu_item<DTYPE, UNROLL, V8>(x, ldx, H, C, r, ch * (NT * UNROLL) + threadIdx.x, NT, wg, wu);
  fill_recip_table(rtab, g0);
  if constexpr (DTYPE == 0) build_silu_table(silu_tab);  // while the first item's loads fly
  const uint32_t tab = smem_u32(silu_tab);
  __syncthreads();
  while (r < M) {
    int64_t rn = r + step_r;
    int chn = ch + step_ch;
    if (chn >= chunks_per_row) {
      chn -= chunks_per_row;
      ++rn;
    }
    const int c0 = ch * (NT * UNROLL) + static_cast<int>(threadIdx.x);
    const int c0n = chn * (NT * UNROLL) + static_cast<int>(threadIdx.x);
    const uint16_t *gnext = x + rn * ldx;
    uint8_t *qrow = q + r * (H / 2);
    uint8_t *sfrow = sf + sf_row_base(layout, r, C, Cp);
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int c = c0 + u * NT;
      float y[16];
      float amax = 0.0f;
      if (c < C) {
        if (DTYPE == 0 && silu_table_covers(wg[u])) {
          amax = swiglu_block16_tab(wg[u], wu[u], tab, y);
        } else {
          // the packed maximum skips NaN: it exceeds 87 only for a gate beyond the exp clamp
          // and is infinite only for an infinite gate
          const float gmax = amax16_packed<DTYPE>(wg[u]);
          if (gmax <= 87.0f) amax = swiglu_block16<DTYPE, false, false>(wg[u], wu[u], y);
          else if (gmax != INFINITY) amax = swiglu_block16<DTYPE, true, false>(wg[u], wu[u], y);
          else amax = swiglu_block16<DTYPE, true, true>(wg[u], wu[u], y);
        }
      }
      const int cn = c0n + u * NT;
      if (rn < M && cn < C) {
        ld_block16<V8>(gnext + cn * 16, wg[u]);
        ld_block16<V8>(gnext + H + cn * 16, wu[u]);
      }
      if (c < C) {
        const uint32_t s = block_scale_code(amax, g0);
        st_cs_u64(qrow + c * 8, quant_f32x16(y, rtab[s]));
        sfrow[sf_col_off(layout, c)] = static_cast<uint8_t>(s);
      }
    }
    r = rn;
    ch = chn;
  }
  zero_sf_padding(sf, layout, M, C, Rp, Cp);
}

// Fused SwiGLU + FP8 E4M3, the write-up's own kernel ("Building Custom TensorRT-LLM Plugins for
// Low-Latency FP8 Inference at Scale", "Fusing the Kernel in CUDA"): q = E4M3(fl(y * scale)),
// saturating at +-448, y = silu(gate) * up in fp32 exactly as in the NVFP4 variant; q is
// [M, H] row-major, one 16-byte store per 16-element block. Same work items and rolling
// next-item loads as swiglu_quant_kernel.
template <int DTYPE, int UNROLL, bool V8, int NT, int MINB>
__global__ void __launch_bounds__(NT, MINB) swiglu_fp8_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t H, int64_t ldx,
    const float *__restrict__ scale, uint8_t *__restrict__ q, int chunks_per_row) {
  extern __shared__ float silu_tab[];  // bf16 input: the SiLU table (kSiluTabBytes)
  const int C = static_cast<int>(H / 16);
  const float sc = scale[0];
  const int64_t step_r = gridDim.x / chunks_per_row;
  const int step_ch = static_cast<int>(gridDim.x % chunks_per_row);
  int64_t r = blockIdx.x / chunks_per_row;
  int ch = static_cast<int>(blockIdx.x % chunks_per_row);
  uint32_t wg[UNROLL][8], wu[UNROLL][8];
  if (r < M) load_swiglu_item<DTYPE, UNROLL, V8>(x, ldx, H, C, r, ch * (NT * UNROLL) + threadIdx.x, NT, wg, wu);
  if constexpr (DTYPE == 0) {
    build_silu_table(silu_tab);  // while the first item's loads fly
    __syncthreads();
  }
  const uint32_t tab = smem_u32(silu_tab);
  while (r < M) {
    int64_t rn = r + step_r;
    int chn = ch + step_ch;
    if (chn >= chunks_per_row) {
      chn -= chunks_per_row;
      ++rn;
    }
    const int c0 = ch * (NT * UNROLL) + static_cast<int>(threadIdx.x);
    const int c0n = chn * (NT * UNROLL) + static_cast<int>(threadIdx.x);
    const uint16_t *gnext = x + rn * ldx;
    uint8_t *qrow = q + r * H;
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int c = c0 + u * NT;
      float y[16];
      if (c < C) {
        if (DTYPE == 0 && silu_table_covers(wg[u])) {
          swiglu_block16_tab(wg[u], wu[u], tab, y);
        } else {
          const float gmax = amax16_packed<DTYPE>(wg[u]);
          if (gmax <= 87.0f) swiglu_block16<DTYPE, false, false>(wg[u], wu[u], y);
          else if (gmax != INFINITY) swiglu_block16<DTYPE, true, false>(wg[u], wu[u], y);
          else swiglu_block16<DTYPE, true, true>(wg[u], wu[u], y);
        }
      }
      const int cn = c0n + u * NT;
      if (rn < M && cn < C) {
        ld_block16<V8>(gnext + cn * 16, wg[u]);
        ld_block16<V8>(gnext + H + cn * 16, wu[u]);
      }
      if (c < C) {
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const F2 a = mul2f_rn(F2{y[4 * k], y[4 * k + 1]}, F2{sc, sc});
          const F2 b = mul2f_rn(F2{y[4 * k + 2], y[4 * k + 3]}, F2{sc, sc});
          o[k] = cvt_e4m3x2(a.x, a.y) | (cvt_e4m3x2(b.x, b.y) << 16);
        }
        asm volatile("st.global.cs.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(qrow + c * 16), "r"(o[0]),
                     "r"(o[1]), "r"(o[2]), "r"(o[3])
                     : "memory");
      }
    }
    r = rn;
    ch = chn;
  }
}

// ------------------------------------------------------------------------------ layouts

__global__ void sf_swizzle_kernel(const uint8_t *__restrict__ lin, uint8_t *__restrict__ out,
                                  int64_t R, int64_t C, int layout, int64_t Rp, int64_t Cp) {
  const int64_t total = Rp * Cp;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / Cp, c = i % Cp;
    out[sf_offset(layout, r, c, C, Cp)] = (r < R && c < C) ? lin[r * C + c] : 0;
  }
}

__global__ void sf_unswizzle_kernel(const uint8_t *__restrict__ in, uint8_t *__restrict__ lin,
                                    int64_t R, int64_t C, int layout, int64_t Cp) {
  const int64_t total = R * C;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / C, c = i % C;
    lin[i] = in[sf_offset(layout, r, c, C, Cp)];
  }
}

// ------------------------------------------------------------------------------ launchers

// Threads per CTA for a row of C blocks handled UNROLL at a time: a multiple of 32, at most
// 256, so that the row splits into whole rounds of threads x UNROLL as evenly as possible.
static int row_threads(int64_t C, int unroll) {
  const int64_t per_round = (C + unroll - 1) / unroll;
  const int64_t rounds = (per_round + 255) / 256;
  int64_t t = (per_round + rounds - 1) / rounds;
  t = (t + 31) / 32 * 32;
  if (t < 32) t = 32;
  if (t > 256) t = 256;
  return static_cast<int>(t);
}

static int row_grid(int64_t M, int threads, int num_sms) {
  int64_t per_sm = 2048 / threads;
  if (per_sm > 16) per_sm = 16;
  int64_t g = static_cast<int64_t>(num_sms) * per_sm;
  if (g > M) g = M;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

static int grid_for(int64_t work_items, int threads, int max_ctas) {
  int64_t g = (work_items + threads - 1) / threads;
  if (g < 1) g = 1;
  if (g > max_ctas) g = max_ctas;
  return static_cast<int>(g);
}

// 32-byte loads need every block start 32-byte aligned: the base and the row pitch.
static bool blocks_32b_aligned(const void *x, int64_t ldx) {
  return (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && ((ldx * 2) & 31) == 0;
}

// Instantiates KERNEL<DTYPE, ..., V8> for the four (dtype, alignment) combinations.
#define NVFP4_DISPATCH_DT_V8(dtype, v8, CALL) \
  do {                                         \
    if ((dtype) == kInBf16) {                  \
      if (v8) {                                \
        constexpr int DT = 0;                  \
        constexpr bool VV = true;              \
        CALL;                                  \
      } else {                                 \
        constexpr int DT = 0;                  \
        constexpr bool VV = false;             \
        CALL;                                  \
      }                                        \
    } else {                                   \
      if (v8) {                                \
        constexpr int DT = 1;                  \
        constexpr bool VV = true;              \
        CALL;                                  \
      } else {                                 \
        constexpr int DT = 1;                  \
        constexpr bool VV = false;             \
        CALL;                                  \
      }                                        \
    }                                          \
  } while (0)

cudaError_t launch_global_scale(const void *x, int dtype, int64_t M, int64_t K, int64_t ldx,
                                float *g_out, float *partial, int nparts, cudaStream_t st) {
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  const bool v8 = blocks_32b_aligned(x, ldx);
  NVFP4_DISPATCH_DT_V8(dtype, v8,
                       (amax_partial_kernel<DT, VV><<<nparts, 256, 0, st>>>(xp, M, K, ldx, partial)));
  amax_finalize_kernel<<<1, 1024, 0, st>>>(partial, nparts, g_out);
  return cudaGetLastError();
}

int global_scale_parts(int64_t M, int64_t K, int num_sms) {
  return grid_for(M * (K / 16), 256, num_sms * 8);
}

cudaError_t launch_quantize(const void *x, int dtype, int64_t M, int64_t K, int64_t ldx, float *g,
                            int per_token, uint8_t *q, uint8_t *sf, int layout, int64_t Rp,
                            int64_t Cp, int num_sms, int max_smem_optin, cudaStream_t st) {
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  const bool v8 = blocks_32b_aligned(x, ldx);
  if (!per_token) {
    const int threads = row_threads(K / 16, 2);
    const int grid = row_grid(M, threads, num_sms);
    NVFP4_DISPATCH_DT_V8(dtype, v8,
                         (quant_stream_kernel<DT, 2, VV><<<grid, threads, 0, st>>>(
                             xp, M, K, ldx, g, 0, q, sf, layout, Rp, Cp)));
    return cudaGetLastError();
  }
  const int C = static_cast<int>(K / 16);
  // A row lives in the registers of one CTA: 128 threads with 1, 2, 4 or 8 blocks each up to
  // 1024 blocks per row (K = 16384), 256 threads with 4 or 8 blocks each up to 2048
  // (K = 32768). The grid is the number of CTAs the launch bounds guarantee resident.
#define NVFP4_LAUNCH_REGS(B, NT, MINB)                                                          \
  do {                                                                                          \
    int64_t cg = static_cast<int64_t>(num_sms) * (MINB);                                        \
    if (cg > M) cg = M;                                                                         \
    if (cg < 1) cg = 1;                                                                         \
    if (dtype == kInBf16)                                                                       \
      quant_pertoken_regs_kernel<0, B, NT, MINB><<<static_cast<int>(cg), NT, 0, st>>>(          \
          xp, M, K, ldx, g, q, sf, layout, Rp, Cp, v8);                                         \
    else                                                                                        \
      quant_pertoken_regs_kernel<1, B, NT, MINB><<<static_cast<int>(cg), NT, 0, st>>>(          \
          xp, M, K, ldx, g, q, sf, layout, Rp, Cp, v8);                                         \
    return cudaGetLastError();                                                                  \
  } while (0)
  if (C <= 128) NVFP4_LAUNCH_REGS(1, 128, 8);
  if (C <= 256) NVFP4_LAUNCH_REGS(2, 128, 8);
  if (C <= 512) NVFP4_LAUNCH_REGS(4, 128, 8);
  if (C <= 1024) NVFP4_LAUNCH_REGS(8, 128, 4);
  if (C <= 2048) NVFP4_LAUNCH_REGS(8, 256, 2);
#undef NVFP4_LAUNCH_REGS
  // Rows too long to stage: row amax pass, then the streaming pass with per-row g.
  const int rgrid = static_cast<int>(M < num_sms * 8 ? M : num_sms * 8);
  const int threads = row_threads(K / 16, 2);
  const int grid = row_grid(M, threads, num_sms);
  NVFP4_DISPATCH_DT_V8(dtype, v8, (row_scale_kernel<DT, VV><<<rgrid, 256, 0, st>>>(xp, M, K, ldx, g)));
  NVFP4_DISPATCH_DT_V8(dtype, v8,
                       (quant_stream_kernel<DT, 2, VV><<<grid, threads, 0, st>>>(
                           xp, M, K, ldx, g, 1, q, sf, layout, Rp, Cp)));
  return cudaGetLastError();
}

cudaError_t launch_swiglu_quantize(const void *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                                   const float *g, uint8_t *q, uint8_t *sf, int layout, int64_t Rp,
                                   int64_t Cp, int num_sms, cudaStream_t st) {
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  // 224 threads x 2 blocks: a 14336-wide output row (896 blocks) is two chunks. Four CTAs per
  // SM are resident (launch bounds), and the grid is exactly that many.
  constexpr int kNT = 224, kUnroll = 2, kMinB = 4;
  const int64_t C = H / 16;
  const int cpr = static_cast<int>((C + kNT * kUnroll - 1) / (kNT * kUnroll));
  int64_t grid = static_cast<int64_t>(num_sms) * kMinB;
  if (grid > M * cpr) grid = M * cpr;
  if (grid < 1) grid = 1;
  const bool v8 = blocks_32b_aligned(x, ldx);
  const int smem = dtype == kInBf16 ? kSiluTabBytes : 0;
  NVFP4_DISPATCH_DT_V8(dtype, v8,
                       (swiglu_quant_kernel<DT, kUnroll, VV, kNT, kMinB>
                        <<<static_cast<int>(grid), kNT, smem, st>>>(xp, M, H, ldx, g, q, sf, layout,
                                                                    Rp, Cp, cpr)));
  return cudaGetLastError();
}

cudaError_t launch_swiglu_fp8(const void *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                              const float *scale, uint8_t *q, int num_sms, cudaStream_t st) {
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  constexpr int kNT = 224, kUnroll = 2, kMinB = 4;
  const int64_t C = H / 16;
  const int cpr = static_cast<int>((C + kNT * kUnroll - 1) / (kNT * kUnroll));
  int64_t grid = static_cast<int64_t>(num_sms) * kMinB;
  if (grid > M * cpr) grid = M * cpr;
  if (grid < 1) grid = 1;
  const bool v8 = blocks_32b_aligned(x, ldx);
  const int smem = dtype == kInBf16 ? kSiluTabBytes : 0;
  NVFP4_DISPATCH_DT_V8(dtype, v8,
                       (swiglu_fp8_kernel<DT, kUnroll, VV, kNT, kMinB>
                        <<<static_cast<int>(grid), kNT, smem, st>>>(xp, M, H, ldx, scale, q, cpr)));
  return cudaGetLastError();
}

cudaError_t launch_sf_swizzle(const uint8_t *lin, uint8_t *out, int64_t R, int64_t C, int layout,
                              int64_t Rp, int64_t Cp, int num_sms, cudaStream_t st) {
  const int grid = grid_for(Rp * Cp, 256, num_sms * 8);
  sf_swizzle_kernel<<<grid, 256, 0, st>>>(lin, out, R, C, layout, Rp, Cp);
  return cudaGetLastError();
}

cudaError_t launch_sf_unswizzle(const uint8_t *in, uint8_t *lin, int64_t R, int64_t C, int layout,
                                int64_t Cp, int num_sms, cudaStream_t st) {
  const int grid = grid_for(R * C, 256, num_sms * 8);
  sf_unswizzle_kernel<<<grid, 256, 0, st>>>(in, lin, R, C, layout, Cp);
  return cudaGetLastError();
}

}  // namespace nvfp4
