// api.cu -- the extern "C" entry points declared in include/nvfp4.h.
//
// Each entry point validates its arguments on the host first (no CUDA call on an invalid
// argument), then looks up the per-device facts resolved once (SM count, opt-in shared
// memory) and enqueues its kernels on the caller's stream. Nothing here allocates.
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/nvfp4.h"
#include "kernels.h"

namespace {

using namespace nvfp4;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int num_sms = 0;
  int max_smem_optin = 0;
  int error = 0;  // cudaError_t of the one-time query
};

DeviceInfo g_info[kMaxDevices];
std::once_flag g_once[kMaxDevices];

// Device facts, queried once per device (first call on that device) and cached.
const DeviceInfo *device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_once[dev], [dev]() {
    DeviceInfo &d = g_info[dev];
    cudaError_t e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    d.error = static_cast<int>(e);
  });
  const DeviceInfo *d = &g_info[dev];
  return d->error == 0 ? d : nullptr;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_layout(int layout) {
  return layout == NVFP4_SF_LINEAR || layout == NVFP4_SF_128x4 || layout == NVFP4_SF_8x4;
}

bool valid_dtype(int dtype) { return dtype == NVFP4_IN_BF16 || dtype == NVFP4_IN_FP16; }

int64_t rows_padded(int layout, int64_t R) {
  if (layout == NVFP4_SF_128x4) return (R + 127) / 128 * 128;
  if (layout == NVFP4_SF_8x4) return (R + 7) / 8 * 8;
  return R;
}

int64_t cols_padded(int layout, int64_t C) {
  return layout == NVFP4_SF_LINEAR ? C : (C + 3) / 4 * 4;
}

int finish(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Shared checks of the activation inputs of the quantize entry points.
int check_activation(const void *x, int dtype, int64_t M, int64_t K, int64_t ldx, int64_t min_ld) {
  if (x == nullptr && M > 0) return NVFP4_ERR_INVALID_ARG;
  if (!valid_dtype(dtype) || M < 0 || K <= 0 || K % 16 != 0 || ldx < min_ld)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || ldx % 8 != 0) return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

}  // namespace

extern "C" {

const char *nvfp4_status_str(int status) {
  switch (status) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_MISALIGNED: return "NVFP4_ERR_MISALIGNED";
    case NVFP4_ERR_UNSUPPORTED: return "NVFP4_ERR_UNSUPPORTED";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT";
    case NVFP4_ERR_SCRATCH_LIMIT: return "NVFP4_ERR_SCRATCH_LIMIT";
    default: return "NVFP4_ERR_UNKNOWN";
  }
}

int64_t nvfp4_sf_bytes(int64_t rows, int64_t k, int layout) {
  if (!valid_layout(layout) || rows < 0 || k < 0 || k % 16 != 0) return -1;
  return rows_padded(layout, rows) * cols_padded(layout, k / 16);
}

size_t nvfp4_global_scale_workspace_bytes(int64_t M, int64_t K) {
  if (M < 0 || K <= 0 || K % 16 != 0) return 0;
  // enough for the largest grid any device in this family uses (8 CTAs per SM, 160 SMs)
  int64_t parts = (M * (K / 16) + 255) / 256;
  if (parts < 1) parts = 1;
  if (parts > 8 * 160) parts = 8 * 160;
  return static_cast<size_t>(parts) * sizeof(float);
}

int nvfp4_global_scale(const void *x, int dtype, int64_t M, int64_t K, int64_t ldx, float *g_out,
                       void *workspace, size_t workspace_bytes, void *stream) {
  int s = check_activation(x, dtype, M, K, ldx, K);
  if (s != NVFP4_OK) return s;
  if (g_out == nullptr || workspace == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(workspace) || (reinterpret_cast<uintptr_t>(g_out) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return NVFP4_ERR_CUDA;
  const int parts = global_scale_parts(M, K, d->num_sms);
  if (workspace_bytes < static_cast<size_t>(parts) * sizeof(float)) return NVFP4_ERR_INVALID_ARG;
  return finish(launch_global_scale(x, dtype, M, K, ldx, g_out, static_cast<float *>(workspace),
                                    parts, static_cast<cudaStream_t>(stream)));
}

int nvfp4_quantize(const void *x, int dtype, int64_t M, int64_t K, int64_t ldx, float *g,
                   int per_token, uint8_t *q, uint8_t *sf, int sf_layout, void *stream) {
  int s = check_activation(x, dtype, M, K, ldx, K);
  if (s != NVFP4_OK) return s;
  if (!valid_layout(sf_layout) || (per_token != 0 && per_token != 1)) return NVFP4_ERR_INVALID_ARG;
  if (M == 0) return NVFP4_OK;
  if (g == nullptr || q == nullptr || sf == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(sf) || (reinterpret_cast<uintptr_t>(g) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return NVFP4_ERR_CUDA;
  const int64_t C = K / 16;
  return finish(launch_quantize(x, dtype, M, K, ldx, g, per_token, q, sf, sf_layout,
                                rows_padded(sf_layout, M), cols_padded(sf_layout, C), d->num_sms,
                                d->max_smem_optin, static_cast<cudaStream_t>(stream)));
}

int swiglu_nvfp4_quantize(const void *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                          const float *g, uint8_t *q, uint8_t *sf, int sf_layout, void *stream) {
  int s = check_activation(x, dtype, M, H, ldx, 2 * H);
  if (s != NVFP4_OK) return s;
  if (!valid_layout(sf_layout)) return NVFP4_ERR_INVALID_ARG;
  if (M == 0) return NVFP4_OK;
  if (g == nullptr || q == nullptr || sf == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(sf) || (reinterpret_cast<uintptr_t>(g) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return NVFP4_ERR_CUDA;
  const int64_t C = H / 16;
  return finish(launch_swiglu_quantize(x, dtype, M, H, ldx, g, q, sf, sf_layout,
                                       rows_padded(sf_layout, M), cols_padded(sf_layout, C),
                                       d->num_sms, static_cast<cudaStream_t>(stream)));
}

int swiglu_fp8_quantize(const void *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                        const float *scale, uint8_t *q, void *stream) {
  int s = check_activation(x, dtype, M, H, ldx, 2 * H);
  if (s != NVFP4_OK) return s;
  if (M == 0) return NVFP4_OK;
  if (scale == nullptr || q == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(q) || (reinterpret_cast<uintptr_t>(scale) & 3u) != 0) return NVFP4_ERR_MISALIGNED;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return NVFP4_ERR_CUDA;
  return finish(launch_swiglu_fp8(x, dtype, M, H, ldx, scale, q, d->num_sms,
                                  static_cast<cudaStream_t>(stream)));
}

int nvfp4_sf_swizzle(const uint8_t *lin, uint8_t *out, int64_t R, int64_t C, int layout,
                     void *stream) {
  if (!valid_layout(layout) || R < 0 || C < 0) return NVFP4_ERR_INVALID_ARG;
  if (R == 0 || C == 0) return NVFP4_OK;
  if (lin == nullptr || out == nullptr) return NVFP4_ERR_INVALID_ARG;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return NVFP4_ERR_CUDA;
  return finish(launch_sf_swizzle(lin, out, R, C, layout, rows_padded(layout, R),
                                  cols_padded(layout, C), d->num_sms,
                                  static_cast<cudaStream_t>(stream)));
}

int nvfp4_sf_unswizzle(const uint8_t *in, uint8_t *lin, int64_t R, int64_t C, int layout,
                       void *stream) {
  if (!valid_layout(layout) || R < 0 || C < 0) return NVFP4_ERR_INVALID_ARG;
  if (R == 0 || C == 0) return NVFP4_OK;
  if (lin == nullptr || in == nullptr) return NVFP4_ERR_INVALID_ARG;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return NVFP4_ERR_CUDA;
  return finish(launch_sf_unswizzle(in, lin, R, C, layout, cols_padded(layout, C), d->num_sms,
                                    static_cast<cudaStream_t>(stream)));
}

size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return 0;
  return gemm_workspace_bytes(M, N, K, d->num_sms);
}

static int gemm_impl(const uint8_t *a_q, const uint8_t *a_sf, int a_layout, const float *a_g,
                     int a_g_per_row, const uint8_t *w_q, const uint8_t *w_sf, const float *w_g,
                     void *out, int64_t M, int64_t N, int64_t K, void *workspace,
                     size_t workspace_bytes, int32_t *dev_status, void *stream) {
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || N % 8 != 0) return NVFP4_ERR_INVALID_ARG;
  if (a_layout != NVFP4_SF_128x4 && a_layout != NVFP4_SF_8x4) return NVFP4_ERR_INVALID_ARG;
  if (a_layout == NVFP4_SF_8x4 && M > 32) return NVFP4_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return NVFP4_OK;
  if (a_q == nullptr || a_sf == nullptr || a_g == nullptr || w_q == nullptr || w_sf == nullptr ||
      w_g == nullptr || out == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(a_q) || !aligned16(w_q) || !aligned16(a_sf) || !aligned16(w_sf) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(a_g) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(w_g) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  if (M > (int64_t(1) << 31) - 256 || N > (int64_t(1) << 31) - 256 || K / 2 > (int64_t(1) << 31))
    return NVFP4_ERR_UNSUPPORTED;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return NVFP4_ERR_CUDA;
  const size_t ws_need = gemm_workspace_bytes(M, N, K, d->num_sms);
  if (ws_need > 0 && (workspace == nullptr || workspace_bytes < ws_need)) return NVFP4_ERR_INVALID_ARG;
  if (ws_need > 0 && !aligned16(workspace)) return NVFP4_ERR_MISALIGNED;
  GemmArgs g{a_q,    a_sf,      a_layout,        a_g,        w_q,      w_sf,
             w_g,    out,       M,               N,          K,        dev_status,
             workspace, workspace_bytes, a_g_per_row};
  return finish(launch_gemm(g, d->num_sms, static_cast<cudaStream_t>(stream)));
}

int nvfp4_gemm(const uint8_t *a_q, const uint8_t *a_sf, int a_layout, const float *a_g,
               const uint8_t *w_q, const uint8_t *w_sf, const float *w_g, void *out, int64_t M,
               int64_t N, int64_t K, void *workspace, size_t workspace_bytes, int32_t *dev_status,
               void *stream) {
  return gemm_impl(a_q, a_sf, a_layout, a_g, 0, w_q, w_sf, w_g, out, M, N, K, workspace,
                   workspace_bytes, dev_status, stream);
}

int nvfp4_gemm_per_token(const uint8_t *a_q, const uint8_t *a_sf, int a_layout, const float *a_g,
                         const uint8_t *w_q, const uint8_t *w_sf, const float *w_g, void *out,
                         int64_t M, int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                         int32_t *dev_status, void *stream) {
  return gemm_impl(a_q, a_sf, a_layout, a_g, 1, w_q, w_sf, w_g, out, M, N, K, workspace,
                   workspace_bytes, dev_status, stream);
}

size_t nvfp4_gemm_act_f32_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return 0;
  return gemm_act_f32_workspace_bytes(M, N, K, d->num_sms);
}

int nvfp4_gemm_act_f32(const uint8_t *a_q, const float *a_sf32, const uint8_t *w_q,
                       const uint8_t *w_sf, const float *w_scale, void *out, int64_t M, int64_t N,
                       int64_t K, void *workspace, size_t workspace_bytes, int32_t *dev_status,
                       void *stream) {
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || N % 8 != 0) return NVFP4_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return NVFP4_OK;
  if (a_q == nullptr || a_sf32 == nullptr || w_q == nullptr || w_sf == nullptr ||
      w_scale == nullptr || out == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(a_q) || !aligned16(a_sf32) || !aligned16(w_q) || !aligned16(w_sf) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(w_scale) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  if (M > (int64_t(1) << 31) - 256 || N > (int64_t(1) << 31) - 256 || !gemm_act_f32_supported(K))
    return NVFP4_ERR_UNSUPPORTED;
  const DeviceInfo *d = device_info();
  if (d == nullptr) return NVFP4_ERR_CUDA;
  const size_t ws_need = gemm_act_f32_workspace_bytes(M, N, K, d->num_sms);
  if (ws_need > 0 && (workspace == nullptr || workspace_bytes < ws_need)) return NVFP4_ERR_INVALID_ARG;
  if (ws_need > 0 && !aligned16(workspace)) return NVFP4_ERR_MISALIGNED;
  GemmArgs g{a_q,       nullptr,         NVFP4_SF_8x4, nullptr, w_q, w_sf,
             nullptr,   out,             M,            N,       K,   dev_status,
             workspace, workspace_bytes, 0,            a_sf32,  w_scale};
  return finish(launch_gemm_act_f32(g, d->num_sms, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
