// global_scale_noalloc.cu -- nvfp4_global_scale_noalloc: the per-tensor global scale with
// its reduction scratch held in this library's own device memory instead of a caller
// workspace.
//
// Who needs it: callers that hold only the tensors they were handed and have no way to
// obtain device memory at the call site -- an engine's enqueue() that receives input and
// output pointers but no allocator, or a runtime whose memory plan is fixed before it
// starts serving -- and callers that must not allocate per call because cudaMalloc and
// cudaFree synchronize the device and can fail under memory pressure in mid-request.
//
// The scratch is one file-scope array of kScratchParts fp32 partial maxima (16 KB). Every
// device that loads the library holds its own copy until the process exits. Each call
// uses one CTA per kBlocksPerCta 16-element blocks, so the array bounds the input at
// kScratchParts * kBlocksPerCta * 16 = 2^28 elements; larger inputs are rejected with
// NVFP4_ERR_SCRATCH_LIMIT before anything is enqueued.
//
// All calls on a device share the array and it keeps the last call's contents. Nothing has
// to start at zero: every CTA writes its own partial before the final reduction reads it.
// Two calls whose kernels overlap on the GPU (different streams without ordering) race on
// the array and may return a wrong scale; order such calls on one stream.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/nvfp4.h"
#include "kernels.h"

namespace {

using namespace nvfp4;

constexpr int kScratchParts = 4096;
constexpr int64_t kBlocksPerCta = 4096;  // 16-element blocks reduced by one CTA
constexpr int kMaxDevices = 64;

// The scratch. In host code `g_partial_scratch` is only a stand-in symbol, not a device
// address: its address must come from cudaGetSymbolAddress with the device current.
static __device__ __align__(256) float g_partial_scratch[kScratchParts];

struct ScratchSlot {
  float *ptr = nullptr;
  int num_sms = 0;
  int error = 0;
};

ScratchSlot g_slot[kMaxDevices];
std::once_flag g_slot_once[kMaxDevices];

// Resolves this device's copy of the scratch (first call on a device only).
const ScratchSlot *scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_slot_once[dev], [dev]() {
    ScratchSlot &s = g_slot[dev];
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_partial_scratch);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev);
    s.ptr = static_cast<float *>(p);
    s.error = static_cast<int>(e);
  });
  const ScratchSlot *s = &g_slot[dev];
  return (s->error == 0 && s->ptr != nullptr) ? s : nullptr;
}

}  // namespace

extern "C" int nvfp4_global_scale_noalloc(const void *x, int dtype, int64_t M, int64_t K,
                                          int64_t ldx, float *g_out, void *stream) {
  if (x == nullptr && M > 0) return NVFP4_ERR_INVALID_ARG;
  if ((dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_FP16) || M < 0 || K <= 0 || K % 16 != 0 ||
      ldx < K || g_out == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) != 0 || ldx % 8 != 0 ||
      (reinterpret_cast<uintptr_t>(g_out) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  const int64_t limit = kScratchParts * kBlocksPerCta;  // 16-element blocks the scratch covers
  if (M > 0 && K / 16 > limit / M) return NVFP4_ERR_SCRATCH_LIMIT;
  const int64_t nblk = M * (K / 16);
  const ScratchSlot *s = scratch_for_current_device();
  if (s == nullptr) return NVFP4_ERR_CUDA;
  int parts = static_cast<int>((nblk + kBlocksPerCta - 1) / kBlocksPerCta);
  if (parts < 1) parts = 1;
  const cudaError_t e = launch_global_scale(x, dtype, M, K, ldx, g_out, s->ptr, parts,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
