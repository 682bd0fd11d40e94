// act_planes.cu -- the fp32 activation-scale split that feeds the block-scaled GEMM.
//
// "Fused Nvfp4 GEMM All Reduce Plugin" (TensorRT-Edge-LLM C++ API) takes the activation
// scales as combined FP32 values [B,1,K/16]; the block-scaled MMA reads E4M3 scales only.
// This kernel turns one chunk of up to 32 activation rows into the E4M3 plane words and
// per-row factors that gemm_nvfp4_decode_kernel<STAGES, 3> streams.
#include <cfloat>
#include <cstdint>

#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4 {

// The largest E4M3 value <= t, for 0 <= t <= 448 (as an fp32 value). Every E4M3 value is
// k * 2^E with an integer 0 <= k <= 15, so cutting t to four significant bits (normal range,
// t >= 2^-6) or to a multiple of 2^-9 (subnormal range) lands on one, and t minus it is exact.
__device__ __forceinline__ float e4m3_floor(float t) {
  if (t >= 0x1p-6f) return __uint_as_float(__float_as_uint(t) & 0xFFF00000u);
  return __fmul_rn(floorf(__fmul_rn(t, 512.0f)), 0x1p-9f);
}

// fp32 activation scales ("Fused Nvfp4 GEMM All Reduce Plugin": a combined FP32 scale
// [B,1,K/16] per activation block, which the block-scaled MMA cannot take) become NPL planes of
// E4M3 codes and one fp32 factor per row: with rho = max_c sa[r,c] / 448 and t = sa * (448 /
// max) <= 448, plane 1 holds floor_E4M3(t), plane 2 floor_E4M3 of the exact remainder, plane 3
// the remainder rounded to nearest. Each floor keeps at least four significant bits, so
// rho * (v1 + v2 + v3) is within 2^-12 of sa relative (blocks below 2^-6 / 448 of the row
// maximum within 2^-10 * rho absolute), and all codes are non-negative, as the MMA's unsigned
// scales need. A negative, NaN or infinite scale is an argument error: its block counts as
// zero and kDevErrBadScale is ORed into the status word.
//
// The NPL plane words (four E4M3 codes each, one K64 step of one row) of four fp32 scales.
template <int NPL>
__device__ __forceinline__ void split_scale_word(float4 v, float inv, uint32_t (&w)[NPL], bool &bad) {
  const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int pl = 0; pl < NPL; ++pl) w[pl] = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const bool ok = e[j] >= 0.0f && e[j] <= FLT_MAX;
    bad |= !ok;
    float t = ok ? fminf(__fmul_rn(e[j], inv), 448.0f) : 0.0f;
#pragma unroll
    for (int pl = 0; pl + 1 < NPL; ++pl) {
      const float f = e4m3_floor(t);
      w[pl] |= cvt_e4m3(f) << (8 * j);
      t = __fsub_rn(t, f);
    }
    w[NPL - 1] |= cvt_e4m3(t) << (8 * j);
  }
}


// The split of one chunk of up to 32 activation rows, once per call ahead of the GEMM: CTA r
// (four warps) handles row r. It finds the row maximum over the row's valid scales, writes
// the output factor alpha = rho * w_scale (zero for a row past M or without a positive scale)
// and the NPL plane words of every K64 step to planes[(k64 * NPL + plane) * 32 + r] (zero
// past M). The GEMM kernel is launched after it as a programmatic dependent, so it can start
// at once; it waits for this kernel only where it reads the words and factors.
constexpr int kPlanesThreads = 128;

template <int NPL>
__global__ void __launch_bounds__(kPlanesThreads) act_scale_planes_kernel(
    const float *__restrict__ a_sf32, int M, int64_t k64_per_row, const float *__restrict__ w_scale,
    uint32_t *__restrict__ planes, float *__restrict__ row_alpha, int *dev_status) {
  __shared__ float warp_max[kPlanesThreads / 32];
  griddep_launch_dependents();
  const int r = blockIdx.x;
  const int t = threadIdx.x;
  const bool live = r < M;
  const float4 *src = reinterpret_cast<const float4 *>(a_sf32 + (live ? r : 0) * (k64_per_row * 4));
  float mx = 0.0f;
  if (live) {
#pragma unroll 4
    for (int64_t g = t; g < k64_per_row; g += kPlanesThreads) {
      const float4 v = __ldg(src + g);
      const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (e[j] >= 0.0f && e[j] <= FLT_MAX) mx = fmaxf(mx, e[j]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((t & 31) == 0) warp_max[t >> 5] = mx;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kPlanesThreads / 32; ++w) mx = fmaxf(mx, warp_max[w]);
  const bool use = live && mx > 0.0f;
  const float inv = use ? __fdiv_rn(448.0f, mx) : 0.0f;
  if (t == 0) row_alpha[r] = use ? __fmul_rn(__fdiv_rn(mx, 448.0f), w_scale[0]) : 0.0f;
  bool bad = false;
  for (int64_t g = t; g < k64_per_row; g += kPlanesThreads) {
    const float4 v = live ? __ldg(src + g) : make_float4(0.f, 0.f, 0.f, 0.f);
    uint32_t w[NPL];
    split_scale_word<NPL>(v, inv, w, bad);
#pragma unroll
    for (int pl = 0; pl < NPL; ++pl) planes[(g * NPL + pl) * 32 + r] = w[pl];
  }
  if (bad && dev_status != nullptr) atomicOr(dev_status, kDevErrBadScale);
}

cudaError_t launch_act_scale_planes(const float *a_sf32, int64_t M, int64_t K, const float *w_scale,
                                    uint32_t *planes, float *row_alpha, int *dev_status,
                                    cudaStream_t st) {
  // one CTA per row of the 32-row chunk
  act_scale_planes_kernel<kActPlanes><<<32, kPlanesThreads, 0, st>>>(
      a_sf32, static_cast<int>(M), K / 64, w_scale, planes, row_alpha, dev_status);
  return cudaGetLastError();
}

}  // namespace nvfp4
