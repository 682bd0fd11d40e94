/*
 * nvfp4_testing.h -- test hooks of libnvfp4.so. Not part of the computing interface
 * (include/nvfp4.h): nothing here changes a result, and with the hooks at their defaults
 * every call behaves exactly as nvfp4.h documents.
 *
 * Why they exist: every wait on a barrier inside the GEMM kernels is bounded, so a kernel
 * whose data never arrives gives up, reports NVFP4_ERR_TIMEOUT through its dev_status word
 * and leaves the GPU usable instead of hanging it (the failure mode that "Building Custom
 * TensorRT-LLM Plugins for Low-Latency FP8 Inference at Scale", section "Production
 * Pitfalls & Hard Lessons", warns about for custom kernels in a serving engine). These hooks
 * let a test drive that path on purpose, without a fault: a short wait limit, and one CTA
 * whose producer withholds the tile loads of one ring position, so its consumers wait on a
 * barrier that nothing will complete. Nothing is in flight when they give up: the producer
 * issues no copy from that position on.
 *
 * Both settings are process-wide, read on the host when a GEMM is launched, and apply to the
 * small-M GEMM (M <= 32 with E4M3 activation scales: nvfp4_gemm / nvfp4_gemm_per_token).
 * Set them only while no other thread launches GEMMs. Restore the defaults afterwards; a
 * call made while a stage is withheld returns NVFP4_OK but its output is incomplete, its
 * dev_status has bit 1 set, and its workspace must be zero-filled again before reuse.
 */
#ifndef NVFP4_TESTING_H_
#define NVFP4_TESTING_H_

#include <stdint.h>

#include "nvfp4.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Wait limit of the small-M GEMM's bounded waits, in nanoseconds of %globaltimer without
 * progress. 0 restores the default (2 s). Values are clamped to [100 us, 10 s]. Returns
 * NVFP4_OK. Host only.
 */
NVFP4_API int nvfp4_testing_set_wait_limit(uint64_t ns);

/*
 * Makes the producer warp of CTA `cta` of the next small-M GEMM launches stop at ring
 * position `ring_position` (the index of the K-step stage it would fill next, counted from 0
 * over the CTA's whole work list) without issuing that stage's copies or any later ones.
 * cta < 0 or ring_position < 0 turns it off (the default). Returns NVFP4_OK, or
 * NVFP4_ERR_INVALID_ARG for a ring position beyond 2^31. Host only.
 */
NVFP4_API int nvfp4_testing_withhold_stage(int cta, int64_t ring_position);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_TESTING_H_ */
