// gemm_sm100.cu -- block-scaled FP4 GEMM (NVFP4: E2M1 operands, one E4M3 scale per 16 K)
// on the 5th-generation tensor cores of sm_100a.
//
//   out[m,n] = fp16( sum_k a[m,k] sa[m,k/16] w[n,k] sw[n,k/16] / (ga * gw) )
//
// Tensor contract: "Fused Nvfp4 GEMM All Reduce Plugin" (TensorRT-Edge-LLM C++ API), inputs
// activation FP4 [B,K], weight FP4 [N,K], FP8 block scale [N,K/16], scalar FP32 global
// weight scale; output FP16 [B,N]. The AllReduce that plugin appends is not part of this
// kernel.
//
// Structure (one output tile per CTA, 192 threads):
//   warp 0      TMA producer: 2-D tiled copies of the packed operands (128-byte swizzle) and
//               bulk copies of the 512-byte scale atoms into a STAGES-deep shared-memory ring.
//   warp 1      allocates TMEM; one lane issues tcgen05.cp (scales -> TMEM) and
//               tcgen05.mma.kind::mxf4nvf4.block_scale (MMA K = 64) into an fp32 TMEM
//               accumulator, and tcgen05.commit to release ring slots.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one TMEM lane quarter per warp),
//               scale by 1 / (ga * gw), round to fp16, store.
// Small M (decode): the operands swap roles (weights are the MMA's 128-row A operand, the
// tokens its N = BN columns) so the weight stream, not the token count, fills the MMA.
#include <cfloat>
#include <cstdint>

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4 {

constexpr int kBM = 128;        // MMA M: rows of the A operand per tile
constexpr int kBKBytes = 128;   // packed bytes of K per stage (256 FP4 elements)
constexpr int kK64PerStage = 4; // MMA K is 64 elements (32 bytes)
constexpr int kSfAtomBytes = 512;  // 128 rows x 4 scales (the 128x4 atom)
constexpr int kThreads = 192;

template <int BN, int STAGES, bool SWAP>
struct Cfg {
  static constexpr int kABytes = kBM * kBKBytes;
  static constexpr int kBBytes = BN * kBKBytes;
  static constexpr int kSfbBlocks = (BN + 127) / 128;
  static constexpr int kSfaBytes = kK64PerStage * kSfAtomBytes;
  static constexpr int kSfbBytes = kSfbBlocks * kK64PerStage * kSfAtomBytes;
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + STAGES * kABytes;
  static constexpr int kOffSfa = kOffB + STAGES * kBBytes;
  static constexpr int kOffSfb = kOffSfa + STAGES * kSfaBytes;
  static constexpr int kOffBar = kOffSfb + STAGES * kSfbBytes;
  static constexpr int kBarBytes = (2 * STAGES + 1) * 8 + 8;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + alignment slack
  // TMEM columns: accumulator [0, BN) (at least 32), then A scales, then B scales
  static constexpr int kAccCols = BN < 32 ? 32 : BN;
  static constexpr int kSfaCol = kAccCols;
  static constexpr int kSfaCols = 4 * kK64PerStage;
  static constexpr int kSfbCol = kSfaCol + kSfaCols;
  static constexpr int kSfbCols = 4 * kSfbBlocks * kK64PerStage;
  static constexpr int kUsedCols = kSfbCol + kSfbCols;
  static constexpr int kTmemCols = kUsedCols <= 32    ? 32
                                   : kUsedCols <= 64  ? 64
                                   : kUsedCols <= 128 ? 128
                                   : kUsedCols <= 256 ? 256
                                                      : 512;
  static_assert(BN % 8 == 0 && BN >= 8 && BN <= 256, "MMA N");
  static_assert(kSmemBytes <= 232448, "shared memory");
  // Instruction descriptor of tcgen05.mma.kind::mxf4nvf4: A and B are E2M1 (format 1),
  // K-major, dense, UE4M3 scales (bit 23 = 0), N >> 3 at bit 17, M >> 4 at bit 24.
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                     (uint32_t(kBM >> 4) << 24);
};

// Shared-memory matrix descriptor: K-major operand tile with 128-byte swizzle, rows of 128
// bytes, 8-row groups 1024 bytes apart (SBO), descriptor version 1.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Descriptor of one 512-byte scale atom as the tcgen05.cp source: 32 rows of 16 bytes,
// no swizzle, 8-row core matrices 128 bytes apart (SBO); one 16-byte column (LBO unused).
__device__ __forceinline__ uint64_t desc_sf_atom(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(128 >> 4) << 32) |
         (static_cast<uint64_t>(1) << 46);
}

struct KernelParams {
  const uint8_t *sfa;  // scales of the MMA A operand (128x4 layout)
  const uint8_t *sfb;  // scales of the MMA B operand (128x4, or 8x4 when sfb_8x4)
  int sfb_8x4;
  int64_t sfa_rows_padded;  // rows of the A-scale buffer
  int64_t sfb_rows_padded;  // rows of the B-scale buffer
  const float *ga;
  const float *gw;
  __half *out;
  int64_t M, N, K;  // problem shape in the caller's (unswapped) terms
  int32_t *dev_status;
};

__device__ __forceinline__ void report_timeout(int32_t *dev_status) {
  if (dev_status != nullptr) atomicOr(dev_status, kDevErrTimeout);
}

template <int BN, int STAGES, bool SWAP>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_a,
                      const __grid_constant__ CUtensorMap tmap_b, const KernelParams p) {
  using C = Cfg<BN, STAGES, SWAP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *empty = full + STAGES;
  uint64_t *acc_full = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t K = p.K;
  const int num_k64 = static_cast<int>(K / 64);
  const int num_kt = (num_k64 + kK64PerStage - 1) / kK64PerStage;
  const int64_t k64_per_row = K / 64;  // 128x4 atoms per 128-row block

  // tile origin: rows of the MMA A operand (a0) and of the MMA B operand (b0)
  const int64_t a0 = static_cast<int64_t>(blockIdx.x) * kBM;
  const int64_t b0 = static_cast<int64_t>(blockIdx.y) * BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    for (int kt = 0; kt < num_kt; ++kt) {
      const int stage = kt % STAGES;
      const int round = kt / STAGES;
      if (kt >= STAGES) {
        if (!mbar_wait_bounded(&empty[stage], (round - 1) & 1, kWaitTimeoutNs)) {
          if (lane == 0) report_timeout(p.dev_status);
          break;
        }
      }
      const int k64_0 = kt * kK64PerStage;
      const int nk64 = min(kK64PerStage, num_k64 - k64_0);
      // scale bytes this stage brings by bulk copy
      const int64_t sfa_block = a0 / 128;
      uint32_t bytes = C::kABytes + C::kBBytes + nk64 * kSfAtomBytes;
      int sfb_copies = 0;
      if (!p.sfb_8x4) {
        for (int blk = 0; blk < C::kSfbBlocks; ++blk)
          if ((b0 / 128 + blk) * 128 < p.sfb_rows_padded) ++sfb_copies;
        bytes += sfb_copies * nk64 * kSfAtomBytes;
      }
      uint8_t *sA = smem + C::kOffA + stage * C::kABytes;
      uint8_t *sB = smem + C::kOffB + stage * C::kBBytes;
      uint8_t *sSfa = smem + C::kOffSfa + stage * C::kSfaBytes;
      uint8_t *sSfb = smem + C::kOffSfb + stage * C::kSfbBytes;
      if (lane == 0) {
        asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(
                         smem_u32(&full[stage])),
                     "r"(bytes)
                     : "memory");
        tma_load_2d(sA, &tmap_a, kt * kBKBytes, static_cast<int32_t>(a0), &full[stage]);
        tma_load_2d(sB, &tmap_b, kt * kBKBytes, static_cast<int32_t>(b0), &full[stage]);
        bulk_g2s(sSfa, p.sfa + (sfa_block * k64_per_row + k64_0) * kSfAtomBytes,
                 nk64 * kSfAtomBytes, &full[stage]);
        if (!p.sfb_8x4) {
          for (int blk = 0; blk < sfb_copies; ++blk) {
            const int64_t rb = b0 / 128 + blk;
            bulk_g2s(sSfb + blk * kK64PerStage * kSfAtomBytes,
                     p.sfb + (rb * k64_per_row + k64_0) * kSfAtomBytes, nk64 * kSfAtomBytes,
                     &full[stage]);
          }
        }
      }
      if (p.sfb_8x4) {
        // 8x4 activation scales (BN <= 32 tokens): rebuild the 128x4 atom rows the TMEM copy
        // expects. Lane r moves row r's 4 scales of each K64 step into bytes [16 r, 16 r + 4).
        const int64_t r = lane;
        for (int a = 0; a < nk64; ++a) {
          uint32_t v = 0;
          if (r < p.sfb_rows_padded && r < BN) {
            v = *reinterpret_cast<const uint32_t *>(
                p.sfb + ((r / 8) * k64_per_row + (k64_0 + a)) * 32 + (r % 8) * 4);
          }
          *reinterpret_cast<uint32_t *>(sSfb + a * kSfAtomBytes + r * 16) = v;
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[stage]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int kt = 0; kt < num_kt; ++kt) {
        const int stage = kt % STAGES;
        const int round = kt / STAGES;
        if (!mbar_wait_bounded(&full[stage], round & 1, kWaitTimeoutNs)) {
          report_timeout(p.dev_status);
          ok = false;
          break;
        }
        tc_fence_after();
        const int nk64 = min(kK64PerStage, num_k64 - kt * kK64PerStage);
        const uint32_t sA = smem_u32(smem + C::kOffA + stage * C::kABytes);
        const uint32_t sB = smem_u32(smem + C::kOffB + stage * C::kBBytes);
        const uint32_t sSfa = smem_u32(smem + C::kOffSfa + stage * C::kSfaBytes);
        const uint32_t sSfb = smem_u32(smem + C::kOffSfb + stage * C::kSfbBytes);
        for (int a = 0; a < nk64; ++a) {
          tmem_cp_32x128b_x4(tmem_base + C::kSfaCol + 4 * a, desc_sf_atom(sSfa + a * kSfAtomBytes));
          for (int blk = 0; blk < C::kSfbBlocks; ++blk)
            tmem_cp_32x128b_x4(tmem_base + C::kSfbCol + (a * C::kSfbBlocks + blk) * 4,
                               desc_sf_atom(sSfb + (blk * kK64PerStage + a) * kSfAtomBytes));
        }
        for (int a = 0; a < nk64; ++a) {
          mma_nvf4(tmem_base, desc_sw128(sA + a * 32), desc_sw128(sB + a * 32), C::kIdesc,
                   tmem_base + C::kSfaCol + 4 * a,
                   tmem_base + C::kSfbCol + a * C::kSfbBlocks * 4, (kt | a) != 0 ? 1u : 0u);
        }
        tc_commit(&empty[stage]);
      }
      if (ok) tc_commit(acc_full);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    const bool ok = mbar_wait_bounded(acc_full, 0, kWaitTimeoutNs);
    if (!ok) {
      if (lane == 0) report_timeout(p.dev_status);
    } else {
      tc_fence_after();
      const float alpha = __fdiv_rn(1.0f, __fmul_rn(p.ga[0], p.gw[0]));
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      if constexpr (!SWAP) {
        const int64_t m = a0 + row;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + c0, v);
          tmem_wait_ld();
          if (m < p.M) {
            __half *dst = p.out + m * p.N + b0 + c0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int64_t n = b0 + c0 + 8 * j;
              if (n + 8 <= p.N) {
                uint4 pk;
                __half2 h0 = __floats2half2_rn(__fmul_rn(__uint_as_float(v[8 * j + 0]), alpha),
                                               __fmul_rn(__uint_as_float(v[8 * j + 1]), alpha));
                __half2 h1 = __floats2half2_rn(__fmul_rn(__uint_as_float(v[8 * j + 2]), alpha),
                                               __fmul_rn(__uint_as_float(v[8 * j + 3]), alpha));
                __half2 h2 = __floats2half2_rn(__fmul_rn(__uint_as_float(v[8 * j + 4]), alpha),
                                               __fmul_rn(__uint_as_float(v[8 * j + 5]), alpha));
                __half2 h3 = __floats2half2_rn(__fmul_rn(__uint_as_float(v[8 * j + 6]), alpha),
                                               __fmul_rn(__uint_as_float(v[8 * j + 7]), alpha));
                pk.x = *reinterpret_cast<uint32_t *>(&h0);
                pk.y = *reinterpret_cast<uint32_t *>(&h1);
                pk.z = *reinterpret_cast<uint32_t *>(&h2);
                pk.w = *reinterpret_cast<uint32_t *>(&h3);
                *reinterpret_cast<uint4 *>(dst + 8 * j) = pk;
              }
            }
          }
        }
      } else {
        // accumulator lane = weight row n, column = token m
        const int64_t n = a0 + row;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 8) {
          uint32_t v[8];
          tmem_ld_32x32b_x8(t_row + c0, v);
          tmem_wait_ld();
          if (n < p.N) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int64_t m = b0 + c0 + j;
              if (m < p.M)
                p.out[m * p.N + n] = __float2half_rn(__fmul_rn(__uint_as_float(v[j]), alpha));
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// 2-D map over a packed [rows, K/2] byte matrix, box = 128 bytes x box_rows, 128-byte swizzle;
// reads past the last row or column are zero-filled.
static bool make_operand_map(CUtensorMap *map, const void *base, int64_t rows, int64_t k_bytes,
                             int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(k_bytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(k_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBKBytes), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int STAGES, bool SWAP>
static cudaError_t run(const GemmArgs &g, cudaStream_t st) {
  using C = Cfg<BN, STAGES, SWAP>;
  CUtensorMap ma, mb;
  KernelParams p{};
  const int64_t kb = g.K / 2;
  const int64_t rows_sf_w = (g.N + 127) / 128 * 128;
  if (!SWAP) {
    if (!make_operand_map(&ma, g.a_q, g.M, kb, kBM)) return cudaErrorInvalidValue;
    if (!make_operand_map(&mb, g.w_q, g.N, kb, BN)) return cudaErrorInvalidValue;
    p.sfa = g.a_sf;
    p.sfb = g.w_sf;
    p.sfb_8x4 = 0;
    p.sfa_rows_padded = (g.M + 127) / 128 * 128;
    p.sfb_rows_padded = rows_sf_w;
  } else {
    if (!make_operand_map(&ma, g.w_q, g.N, kb, kBM)) return cudaErrorInvalidValue;
    if (!make_operand_map(&mb, g.a_q, g.M, kb, BN)) return cudaErrorInvalidValue;
    p.sfa = g.w_sf;
    p.sfb = g.a_sf;
    p.sfb_8x4 = g.a_layout == kSf8x4 ? 1 : 0;
    p.sfa_rows_padded = rows_sf_w;
    p.sfb_rows_padded = p.sfb_8x4 ? (g.M + 7) / 8 * 8 : (g.M + 127) / 128 * 128;
  }
  p.ga = g.a_g;
  p.gw = g.w_g;
  p.out = static_cast<__half *>(g.out);
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.dev_status = g.dev_status;
  const int64_t rows_a = SWAP ? g.N : g.M;
  const int64_t rows_b = SWAP ? g.M : g.N;
  dim3 grid(static_cast<unsigned>((rows_a + kBM - 1) / kBM),
            static_cast<unsigned>((rows_b + BN - 1) / BN));
  cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_kernel<BN, STAGES, SWAP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  gemm_nvfp4_kernel<BN, STAGES, SWAP><<<grid, kThreads, C::kSmemBytes, st>>>(ma, mb, p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs &g, int num_sms, cudaStream_t st) {
  (void)num_sms;
  if (g.M <= 32) return run<32, 6, true>(g, st);
  return run<256, 4, false>(g, st);
}

}  // namespace nvfp4
