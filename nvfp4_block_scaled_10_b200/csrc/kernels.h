// kernels.h -- internal declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace nvfp4 {

constexpr int kSfLinear = 0;
constexpr int kSf128x4 = 1;
constexpr int kSf8x4 = 2;
constexpr int kInBf16 = 0;
constexpr int kInFp16 = 1;

constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s without progress
constexpr int kDevErrTimeout = 1;
constexpr int kDevErrBadScale = 2;  // an fp32 activation scale was negative, NaN or infinite
constexpr int kDevErrWorkspace = 4;  // a split-K tile counter was not zero when the call began

// testing.cu: the hooks of include/nvfp4_testing.h as the launchers read them.
struct DebugHooks {
  uint64_t wait_ns;      // limit of the small-M GEMM's bounded waits
  int withhold_cta;      // CTA whose producer stops at ring position withhold_it (-1: none)
  int64_t withhold_it;
};
DebugHooks debug_hooks();

// Launches `kernel` as a programmatic dependent of the work before it in the stream
// (cudaLaunchAttributeProgrammaticStreamSerialization): it may start while the kernel before
// it still runs, once that kernel's CTAs have all reached griddepcontrol.launch_dependents
// or exited. Until it has waited for that kernel (griddepcontrol.wait) it may only prefetch
// into L2: no load into shared memory or registers, no write.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// quantize.cu
int *device_error_symbol();
int global_scale_parts(int64_t M, int64_t K, int num_sms);
cudaError_t launch_global_scale(const void *x, int dtype, int64_t M, int64_t K, int64_t ldx,
                                float *g_out, float *partial, int nparts, cudaStream_t st);
cudaError_t launch_quantize(const void *x, int dtype, int64_t M, int64_t K, int64_t ldx, float *g,
                            int per_token, uint8_t *q, uint8_t *sf, int layout, int64_t Rp,
                            int64_t Cp, int num_sms, int max_smem_optin, cudaStream_t st);
cudaError_t launch_swiglu_quantize(const void *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                                   const float *g, uint8_t *q, uint8_t *sf, int layout, int64_t Rp,
                                   int64_t Cp, int num_sms, cudaStream_t st);
cudaError_t launch_swiglu_fp8(const void *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                              const float *scale, uint8_t *q, int num_sms, cudaStream_t st);
cudaError_t launch_sf_swizzle(const uint8_t *lin, uint8_t *out, int64_t R, int64_t C, int layout,
                              int64_t Rp, int64_t Cp, int num_sms, cudaStream_t st);
cudaError_t launch_sf_unswizzle(const uint8_t *in, uint8_t *lin, int64_t R, int64_t C, int layout,
                                int64_t Cp, int num_sms, cudaStream_t st);

// act_planes.cu: the fp32 activation scales of up to 32 rows [M, K/16] become kActPlanes
// planes of E4M3 words planes[(k64 * kActPlanes + plane) * 32 + row] and per-row output
// factors row_alpha[32] (= row maximum / 448 * w_scale; zero past M). Bad scales OR
// kDevErrBadScale into dev_status. Written for the GEMM launched next, which may start early
// (programmatic dependent launch) and waits for this kernel where it reads them.
constexpr int kActPlanes = 3;
cudaError_t launch_act_scale_planes(const float *a_sf32, int64_t M, int64_t K, const float *w_scale,
                                    uint32_t *planes, float *row_alpha, int *dev_status,
                                    cudaStream_t st);

// gemm_sm100.cu
struct GemmArgs {
  const uint8_t *a_q;
  const uint8_t *a_sf;
  int a_layout;
  const float *a_g;
  const uint8_t *w_q;
  const uint8_t *w_sf;
  const float *w_g;
  void *out;
  int64_t M, N, K;
  int32_t *dev_status;
  void *workspace;
  size_t workspace_bytes;
  int a_g_per_row;  // a_g is [M]: one activation encode scale per row
  const float *a_sf32 = nullptr;   // fp32 activation scales [M, K/16] (launch_gemm_act_f32)
  const float *w_scale = nullptr;  // fp32 weight dequantization scale (launch_gemm_act_f32)
};
cudaError_t launch_gemm(const GemmArgs &args, int num_sms, cudaStream_t st);
// Workspace the GEMM needs for (M, N, K) on a device with num_sms SMs (split-K partial sums
// and tile counters of the small-M path; 0 otherwise).
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms);
// The GEMM with fp32 activation scales [M, K/16] and a multiplying fp32 weight scale.
cudaError_t launch_gemm_act_f32(const GemmArgs &args, int num_sms, cudaStream_t st);
size_t gemm_act_f32_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms);
bool gemm_act_f32_supported(int64_t K);

}  // namespace nvfp4
