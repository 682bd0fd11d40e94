// quantize.cu -- NVFP4 quantization kernels for sm_100a (memory-bound, CUDA cores).
//
//  * global amax -> per-tensor encode scale g (two launches, partial maxima in workspace)
//  * streaming quantize: one thread owns one 16-element block (one 32-byte load), given g
//    per tensor or per row
//  * per-token quantize: whole rows staged in shared memory by bulk TMA copies (several rows
//    in flight per CTA), row amax -> g_row, then the blocks of the row are quantized from
//    shared memory, so X is read from HBM once
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

// Quantizes 16 fp32 values with encode scale g. Returns the 8 packed bytes (element 2j in
// the low nibble of byte j) and the E4M3 scale code.
__device__ __forceinline__ uint64_t quant_block16(const float (&y)[16], float g, uint32_t &s_enc) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(y[i]));
  const float s = __fmul_rn(__fdiv_rn(amax, 6.0f), g);
  s_enc = cvt_e4m3(s);
  const float s_dec = e4m3_to_f32(s_enc);
  const float r = (s_dec == 0.0f) ? 0.0f : fminf(__fdiv_rn(g, s_dec), FLT_MAX);
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    lo |= cvt_e2m1x2(__fmul_rn(y[2 * j], r), __fmul_rn(y[2 * j + 1], r)) << (8 * j);
    hi |= cvt_e2m1x2(__fmul_rn(y[8 + 2 * j], r), __fmul_rn(y[8 + 2 * j + 1], r)) << (8 * j);
  }
  return (static_cast<uint64_t>(hi) << 32) | lo;
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

// One thread per 16-element block, UNROLL blocks in flight per thread.
// g_per_row == 0: g[0] for every row; == 1: g[r].
template <int DTYPE, int UNROLL, bool V8>
__global__ void __launch_bounds__(256) quant_stream_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, const float *__restrict__ g,
    int g_per_row, uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int layout, int64_t Rp,
    int64_t Cp) {
  const int64_t C = K / 16;
  const int64_t nblk = M * C;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const float g0 = g_per_row ? 0.0f : g[0];
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < nblk;
       base += nthreads * UNROLL) {
    uint32_t w[UNROLL][8];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t b = base + u * nthreads;
      if (b < nblk) {
        const int64_t r = b / C, c = b - r * C;
        ld_block16<V8>(x + r * ldx + c * 16, w[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t b = base + u * nthreads;
      if (b < nblk) {
        const int64_t r = b / C, c = b - r * C;
        float y[16];
        unpack16<DTYPE>(w[u], y);
        uint32_t s;
        const uint64_t packed = quant_block16(y, g_per_row ? g[r] : g0, s);
        st_cs_u64(q + r * (K / 2) + c * 8, packed);
        sf[sf_offset(layout, r, c, C, Cp)] = static_cast<uint8_t>(s);
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

// Persistent: CTA b handles rows b, b + gridDim.x, ... Each row (K * 2 bytes) is brought into
// one of `stages` shared-memory slots by a bulk TMA copy issued by thread 0 `stages` rows
// ahead; all threads then reduce the row amax and quantize the row from shared memory.
template <int DTYPE>
__global__ void __launch_bounds__(256) quant_pertoken_rowcache_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float *__restrict__ g,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int layout, int64_t Rp, int64_t Cp,
    int stages) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kRowcacheMaxStages];
  __shared__ float red[32];
  const int64_t C = K / 16;
  const uint32_t row_bytes = static_cast<uint32_t>(K * 2);

  zero_sf_padding(sf, layout, M, C, Rp, Cp);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t first = blockIdx.x;
  const int64_t step = gridDim.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      const int64_t r = first + s * step;
      if (r < M) {
        mbar_arrive_expect_tx(&full[s], row_bytes);
        bulk_g2s(smem + static_cast<size_t>(s) * row_bytes, x + r * ldx, row_bytes, &full[s]);
      }
    }
  }

  int64_t j = 0;
  for (int64_t r = first; r < M; r += step, ++j) {
    const int stage = static_cast<int>(j % stages);
    const uint32_t parity = static_cast<uint32_t>((j / stages) & 1);
    // Bounded wait; every thread takes the same decision so the CTA leaves together.
    const bool ok = mbar_wait_bounded(&full[stage], parity, kWaitTimeoutNs);
    if (__syncthreads_or(!ok)) {
      if (threadIdx.x == 0) atomicOr(&g_device_error, kDevErrTimeout);
      return;
    }
    const uint8_t *row = smem + static_cast<size_t>(stage) * row_bytes;

    // Row amax: plain 16-byte chunks in order (conflict-free).
    float m = 0.0f;
    const uint4 *chunks = reinterpret_cast<const uint4 *>(row);
    for (int64_t i = threadIdx.x; i < static_cast<int64_t>(row_bytes / 16); i += blockDim.x) {
      const uint4 a = chunks[i];
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float lo, hi;
        unpack2<DTYPE>(w[k], lo, hi);
        m = fmaxf(m, fmaxf(fabsf(lo), fabsf(hi)));
      }
    }
    const float gr = global_scale_from_amax(block_max(m, red));
    if (threadIdx.x == 0) g[r] = gr;

    // Each thread quantizes whole 32-byte blocks; lanes 4-7 of each quarter-warp read the
    // upper half first so the 8 lanes of a 128-bit shared-memory phase hit distinct banks.
    const uint32_t h = (threadIdx.x >> 2) & 1u;
    for (int64_t c = threadIdx.x; c < C; c += blockDim.x) {
      const uint4 *p = reinterpret_cast<const uint4 *>(row + c * 32);
      const uint4 first = p[h], second = p[h ^ 1u];
      const uint4 a = h ? second : first, b = h ? first : second;
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      float y[16];
      unpack16<DTYPE>(w, y);
      uint32_t s;
      const uint64_t packed = quant_block16(y, gr, s);
      st_cs_u64(q + r * (K / 2) + c * 8, packed);
      sf[sf_offset(layout, r, c, C, Cp)] = static_cast<uint8_t>(s);
    }
    __syncthreads();  // every thread is done with this slot
    if (threadIdx.x == 0) {
      const int64_t rn = r + static_cast<int64_t>(stages) * step;
      if (rn < M) {
        mbar_arrive_expect_tx(&full[stage], row_bytes);
        bulk_g2s(smem + static_cast<size_t>(stage) * row_bytes, x + rn * ldx, row_bytes,
                 &full[stage]);
      }
    }
  }
}

// ------------------------------------------------------------------------------ SwiGLU

// Library fp32 exponential: clamp to [-87, 88]; k = rint(v * log2 e); Cody-Waite reduction
// f = v - k*ln2_hi - k*ln2_lo; degree-7 Taylor polynomial of e^f (coefficients 1/n!
// rounded to fp32) by fused multiply-add; times 2^k built from exponent bits.
__device__ __forceinline__ float exp_f32(float v) {
  v = fminf(fmaxf(v, -87.0f), 88.0f);
  const float k = rintf(__fmul_rn(v, 0x1.715476p+0f));
  float f = __fmaf_rn(-k, 0x1.62e4p-1f, v);
  f = __fmaf_rn(-k, 0x1.7f7d1cp-20f, f);
  float p = 0x1.a01a02p-13f;             // 1/7!
  p = __fmaf_rn(p, f, 0x1.6c16c2p-10f);  // 1/6!
  p = __fmaf_rn(p, f, 0x1.111112p-7f);   // 1/5!
  p = __fmaf_rn(p, f, 0x1.555556p-5f);   // 1/4!
  p = __fmaf_rn(p, f, 0x1.555556p-3f);   // 1/3!
  p = __fmaf_rn(p, f, 0.5f);             // 1/2!
  p = __fmaf_rn(p, f, 1.0f);             // 1/1!
  p = __fmaf_rn(p, f, 1.0f);             // 1/0!
  const float two_k = __int_as_float((static_cast<int>(k) + 127) << 23);
  return __fmul_rn(p, two_k);
}

__device__ __forceinline__ float swiglu_f32(float gate, float up) {
  const float silu = __fdiv_rn(gate, __fadd_rn(1.0f, exp_f32(-gate)));
  return __fmul_rn(silu, up);
}

template <int DTYPE, int UNROLL, bool V8>
__global__ void __launch_bounds__(256) swiglu_quant_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t H, int64_t ldx, const float *__restrict__ g,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int layout, int64_t Rp, int64_t Cp) {
  const int64_t C = H / 16;
  const int64_t nblk = M * C;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const float g0 = g[0];
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < nblk;
       base += nthreads * UNROLL) {
    uint32_t wg[UNROLL][8], wu[UNROLL][8];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t b = base + u * nthreads;
      if (b < nblk) {
        const int64_t r = b / C, c = b - r * C;
        const uint16_t *row = x + r * ldx;
        ld_block16<V8>(row + c * 16, wg[u]);
        ld_block16<V8>(row + H + c * 16, wu[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t b = base + u * nthreads;
      if (b < nblk) {
        const int64_t r = b / C, c = b - r * C;
        float gate[16], up[16], y[16];
        unpack16<DTYPE>(wg[u], gate);
        unpack16<DTYPE>(wu[u], up);
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = swiglu_f32(gate[i], up[i]);
        uint32_t s;
        const uint64_t packed = quant_block16(y, g0, s);
        st_cs_u64(q + r * (H / 2) + c * 8, packed);
        sf[sf_offset(layout, r, c, C, Cp)] = static_cast<uint8_t>(s);
      }
    }
  }
  zero_sf_padding(sf, layout, M, C, Rp, Cp);
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
  const int64_t nblk = M * (K / 16);
  const bool v8 = blocks_32b_aligned(x, ldx);
  if (!per_token) {
    const int grid = grid_for(nblk, 256, num_sms * 8);
    NVFP4_DISPATCH_DT_V8(dtype, v8,
                         (quant_stream_kernel<DT, 2, VV><<<grid, 256, 0, st>>>(
                             xp, M, K, ldx, g, 0, q, sf, layout, Rp, Cp)));
    return cudaGetLastError();
  }
  const int64_t row_bytes = K * 2;
  // Rows in flight per CTA: up to kRowcacheMaxStages, fewer when three CTAs of that size would
  // not share an SM; at least two or the row is not staged at all.
  int stages = 0;
  for (int s = kRowcacheMaxStages; s >= 2; --s) {
    if (row_bytes * s + 1024 <= max_smem_optin) {
      stages = s;
      break;
    }
  }
  if (stages >= 2) {
    while (stages > 2 && row_bytes * stages * 3 > 220 * 1024) --stages;
    const size_t smem = static_cast<size_t>(row_bytes * stages);
    int per_sm = static_cast<int>((220 * 1024) / (smem + 2048));
    if (per_sm < 1) per_sm = 1;
    if (per_sm > 8) per_sm = 8;
    int64_t grid = static_cast<int64_t>(num_sms) * per_sm;
    if (grid > M) grid = M;
    if (grid < 1) grid = 1;
    cudaError_t e;
    if (dtype == kInBf16) {
      e = cudaFuncSetAttribute(quant_pertoken_rowcache_kernel<0>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      quant_pertoken_rowcache_kernel<0><<<static_cast<int>(grid), 256, smem, st>>>(
          xp, M, K, ldx, g, q, sf, layout, Rp, Cp, stages);
    } else {
      e = cudaFuncSetAttribute(quant_pertoken_rowcache_kernel<1>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      quant_pertoken_rowcache_kernel<1><<<static_cast<int>(grid), 256, smem, st>>>(
          xp, M, K, ldx, g, q, sf, layout, Rp, Cp, stages);
    }
    return cudaGetLastError();
  }
  // Rows too long to stage: row amax pass, then the streaming pass with per-row g.
  const int rgrid = static_cast<int>(M < num_sms * 8 ? M : num_sms * 8);
  const int grid = grid_for(nblk, 256, num_sms * 8);
  NVFP4_DISPATCH_DT_V8(dtype, v8, (row_scale_kernel<DT, VV><<<rgrid, 256, 0, st>>>(xp, M, K, ldx, g)));
  NVFP4_DISPATCH_DT_V8(dtype, v8,
                       (quant_stream_kernel<DT, 2, VV><<<grid, 256, 0, st>>>(
                           xp, M, K, ldx, g, 1, q, sf, layout, Rp, Cp)));
  return cudaGetLastError();
}

cudaError_t launch_swiglu_quantize(const void *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                                   const float *g, uint8_t *q, uint8_t *sf, int layout, int64_t Rp,
                                   int64_t Cp, int num_sms, cudaStream_t st) {
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  const int64_t nblk = M * (H / 16);
  const int grid = grid_for(nblk, 256, num_sms * 8);
  const bool v8 = blocks_32b_aligned(x, ldx);
  NVFP4_DISPATCH_DT_V8(dtype, v8,
                       (swiglu_quant_kernel<DT, 2, VV><<<grid, 256, 0, st>>>(
                           xp, M, H, ldx, g, q, sf, layout, Rp, Cp)));
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
