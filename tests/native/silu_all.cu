// Test harness: silu of the fused SwiGLU kernel's device arithmetic (swiglu_math.cuh) for a
// list of 16-bit gates, so a test can compare every bf16 and fp16 gate with the oracle.
// Test code only; built by tests/test_swiglu_math_gpu.py with nvcc.
#include <cstdint>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "swiglu_math.cuh"

namespace {

template <bool CLAMP, bool SAFE>
__global__ void silu_kernel(const uint16_t *__restrict__ bits, int dtype, int n, float *__restrict__ out) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const uint32_t b0 = bits[i], b1 = (i + 1 < n) ? bits[i + 1] : 0;
  const uint32_t w = b0 | (b1 << 16);
  const nvfp4::F2 v = dtype == 0 ? nvfp4::unpack2_neg<0>(w) : nvfp4::unpack2_neg<1>(w);
  const nvfp4::F2 s = nvfp4::silu_pair_neg<CLAMP, SAFE>(v);
  out[i] = s.x;
  if (i + 1 < n) out[i + 1] = s.y;
}

}  // namespace

// Returns 0 on success, else the CUDA error code. host_bits: n gates; host_out: n floats.
// form 0: no clamp, no infinite-dividend select; 1: clamp only; 2: clamp and select.
extern "C" int silu_all(const uint16_t *host_bits, int dtype, int n, float *host_out, int form) {
  uint16_t *d_bits = nullptr;
  float *d_out = nullptr;
  cudaError_t e = cudaMalloc(&d_bits, n * sizeof(uint16_t));
  if (e == cudaSuccess) e = cudaMalloc(&d_out, n * sizeof(float));
  if (e == cudaSuccess) e = cudaMemcpy(d_bits, host_bits, n * sizeof(uint16_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) {
    const int pairs = (n + 1) / 2;
    const int grid = (pairs + 255) / 256;
    if (form == 0) silu_kernel<false, false><<<grid, 256>>>(d_bits, dtype, n, d_out);
    else if (form == 1) silu_kernel<true, false><<<grid, 256>>>(d_bits, dtype, n, d_out);
    else silu_kernel<true, true><<<grid, 256>>>(d_bits, dtype, n, d_out);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemcpy(host_out, d_out, n * sizeof(float), cudaMemcpyDeviceToHost);
  cudaFree(d_bits);
  cudaFree(d_out);
  return static_cast<int>(e);
}
