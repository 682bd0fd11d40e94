// testing.cu -- the test hooks declared in include/nvfp4_testing.h: a wait limit for the
// small-M GEMM's bounded waits and a ring position at which one CTA's producer withholds its
// copies, so that a test can make a device wait run out without a fault.
#include <atomic>
#include <cstdint>

#include "../../include/nvfp4_testing.h"
#include "kernels.h"

namespace nvfp4 {

namespace {
std::atomic<uint64_t> g_wait_ns{kWaitTimeoutNs};
std::atomic<int> g_withhold_cta{-1};
std::atomic<int64_t> g_withhold_it{-1};
}  // namespace

DebugHooks debug_hooks() {
  DebugHooks h;
  h.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  h.withhold_cta = g_withhold_cta.load(std::memory_order_relaxed);
  h.withhold_it = g_withhold_it.load(std::memory_order_relaxed);
  if (h.withhold_cta < 0 || h.withhold_it < 0) {
    h.withhold_cta = -1;
    h.withhold_it = -1;
  }
  return h;
}

}  // namespace nvfp4

extern "C" {

int nvfp4_testing_set_wait_limit(uint64_t ns) {
  constexpr uint64_t kMin = 100000ull, kMax = 10000000000ull;
  if (ns == 0) ns = nvfp4::kWaitTimeoutNs;
  if (ns < kMin) ns = kMin;
  if (ns > kMax) ns = kMax;
  nvfp4::g_wait_ns.store(ns, std::memory_order_relaxed);
  return NVFP4_OK;
}

int nvfp4_testing_withhold_stage(int cta, int64_t ring_position) {
  if (ring_position > (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
  if (cta < 0 || ring_position < 0) {
    cta = -1;
    ring_position = -1;
  }
  nvfp4::g_withhold_cta.store(cta, std::memory_order_relaxed);
  nvfp4::g_withhold_it.store(ring_position, std::memory_order_relaxed);
  return NVFP4_OK;
}

}  // extern "C"
