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
// Persistent, warp-specialised kernel (one CTA per SM, tiles handed out round-robin):
//   warp 0        TMA producer: 2-D tiled copies of the packed operands (128-byte swizzle)
//                 and bulk copies of the 512-byte scale atoms into a STAGES-deep ring.
//   warp 1        allocates TMEM; one lane issues tcgen05.mma.kind::mxf4nvf4.block_scale
//                 (MMA K = 64) into an fp32 TMEM accumulator and tcgen05.commit.
//   warps 4..7    scale warps: warp 4+q moves the scale words that TMEM lane quarter q needs
//                 from the shared-memory atoms into TMEM with tcgen05.st, one TMEM scale slot
//                 per ring stage (tcgen05.cp copies of whole atoms cost about as much tensor
//                 pipe time as the MMAs; tcgen05.st from other warps does not slow them).
//   warps 8..     epilogue: tcgen05.ld of the accumulator (lane quarter = warp % 4), scale
//                 by 1 / (ga * gw) and round to fp16 in registers, release the accumulator,
//                 then store.
//
// Scale layout the MMA reads (measured on B200 with probes): TMEM lane quarter q (lanes
// 32 q .. 32 q + 31, accumulator rows 32 q .. 32 q + 31) reads both operands' scales from its
// own lanes. A row m = 32 q + i: the 32-bit word (four E4M3 scales of one K64 step) at lane
// m, column base + q. B row n: lane 32 q + n % 32, column base + n / 32, so B's scales are
// replicated into all four quarters. Bases are column-aligned (4 columns per K64 step, 8 for
// a 256-row B operand); an unaligned base raised a misaligned-address error.
//
// Small M (decode): the operands swap roles (weights are the MMA's 128-row A operand, the
// tokens its N = BN columns) so the weight stream fills the MMA.
#include <cfloat>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4 {

constexpr int kBM = 128;           // MMA M: rows of the A operand per tile
constexpr int kBKBytes = 128;      // packed bytes of K per stage (256 FP4 elements)
constexpr int kK64PerStage = 4;    // MMA K is 64 elements (32 bytes)
constexpr int kSfAtomBytes = 512;  // 128 rows x 4 scales (the 128x4 atom)
constexpr int kSfWarp0 = 4;        // first scale warp
constexpr int kEpiWarp0 = 8;       // first epilogue warp

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
  static constexpr int kAccBufs = BN <= 128 ? 2 : 1;
  // full[S], empty[S], sf_full[S], acc_full[A], acc_empty[A], tmem slot
  static constexpr int kBarBytes = (3 * STAGES + 2 * kAccBufs) * 8 + 16;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + alignment slack
  // TMEM columns: accumulators, then per stage one scale slot (A scales, then B scales)
  static constexpr int kAccCols = BN < 32 ? 32 : BN;
  static constexpr int kSfaColsPerK64 = 4;
  static constexpr int kSfbColsPerK64 = BN > 128 ? 8 : 4;
  static constexpr int kSlotCols = kK64PerStage * (kSfaColsPerK64 + kSfbColsPerK64);
  static constexpr int kSfCol0 = kAccBufs * kAccCols;
  static constexpr int kUsedCols = kSfCol0 + STAGES * kSlotCols;
  static constexpr int kTmemCols = kUsedCols <= 32    ? 32
                                   : kUsedCols <= 64  ? 64
                                   : kUsedCols <= 128 ? 128
                                   : kUsedCols <= 256 ? 256
                                                      : 512;
  // epilogue: 8 warps (two per lane quarter, 128 columns each) for BN = 256, else 4
  static constexpr int kEpiWarps = BN > 128 ? 8 : 4;
  static constexpr int kColsPerEpiWarp = BN * 4 / kEpiWarps;
  static constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
  static_assert(BN % 8 == 0 && BN >= 8 && BN <= 256, "MMA N");
  static_assert(kUsedCols <= 512, "TMEM columns");
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

// 4 consecutive TMEM columns of this warp's 32 lanes, all set to v. The store takes a range
// of four distinct registers, so the value is copied into four temporaries first (naming
// one register four times leaves columns 1-3 with whatever the neighbouring registers hold).
__device__ __forceinline__ void tmem_st_x4_rep(uint32_t taddr, uint32_t v) {
  asm volatile(
      "{\n\t.reg .b32 t0, t1, t2, t3;\n\t"
      "mov.b32 t0, %1;\n\tmov.b32 t1, %1;\n\tmov.b32 t2, %1;\n\tmov.b32 t3, %1;\n\t"
      "tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {t0, t1, t2, t3};\n\t}" ::"r"(taddr),
      "r"(v)
      : "memory");
}

// 4 consecutive TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, uint32_t v0, uint32_t v1, uint32_t v2,
                                           uint32_t v3) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr),
               "r"(v0), "r"(v1), "r"(v2), "r"(v3)
               : "memory");
}

// 8 consecutive TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, uint4 a, uint4 b) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                   taddr),
               "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

struct KernelParams {
  const uint8_t *sfa;  // scales of the MMA A operand (128x4 layout)
  const uint8_t *sfb;  // scales of the MMA B operand (128x4, or 8x4 when sfb_8x4)
  int sfb_8x4;
  int64_t sfb_rows_padded;  // rows of the B-scale buffer
  int64_t sfa_rows_padded;  // rows of the A-scale buffer
  const float *ga;
  const float *gw;
  __half *out;
  int64_t M, N, K;  // problem shape in the caller's (unswapped) terms
  int tiles_a;      // tiles along the MMA A operand (128 rows each)
  int tiles_b;      // tiles along the MMA B operand (BN rows each)
  int32_t *dev_status;
};

__device__ __forceinline__ void report_timeout(int32_t *dev_status) {
  if (dev_status != nullptr) atomicOr(dev_status, kDevErrTimeout);
}

template <int BN, int STAGES, bool SWAP>
__global__ void __launch_bounds__(Cfg<BN, STAGES, SWAP>::kThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_a,
                      const __grid_constant__ CUtensorMap tmap_b, const KernelParams p) {
  using C = Cfg<BN, STAGES, SWAP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *empty = full + STAGES;
  uint64_t *sf_full = empty + STAGES;
  uint64_t *acc_full = sf_full + STAGES;
  uint64_t *acc_empty = acc_full + C::kAccBufs;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + C::kAccBufs);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t K = p.K;
  const int num_k64 = static_cast<int>(K / 64);
  const int num_kt = (num_k64 + kK64PerStage - 1) / kK64PerStage;
  const int64_t k64_per_row = K / 64;  // 128x4 atoms per 128-row block
  const int num_tiles = p.tiles_a * p.tiles_b;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 4);  // one arrival per scale warp
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::kEpiWarps);
    }
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

  // Tile t covers MMA-A rows [a0, a0 + 128) and MMA-B rows [b0, b0 + BN).
  auto tile_origin = [&](int t, int64_t &a0, int64_t &b0) {
    a0 = static_cast<int64_t>(t % p.tiles_a) * kBM;
    b0 = static_cast<int64_t>(t / p.tiles_a) * BN;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    uint32_t it = 0;  // ring position across tiles
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      int64_t a0, b0;
      tile_origin(t, a0, b0);
      int sfb_copies = 0;
      if (!p.sfb_8x4) {
        for (int blk = 0; blk < C::kSfbBlocks; ++blk)
          if ((b0 / 128 + blk) * 128 < p.sfb_rows_padded) ++sfb_copies;
      }
      for (int kt = 0; kt < num_kt; ++kt, ++it) {
        const int stage = static_cast<int>(it % STAGES);
        const uint32_t round = it / STAGES;
        if (it >= STAGES) {
          if (!mbar_wait_warp(&empty[stage], (round - 1) & 1, kWaitTimeoutNs)) {
            if (lane == 0) report_timeout(p.dev_status);
            ok = false;
            break;
          }
        }
        const int k64_0 = kt * kK64PerStage;
        const int nk64 = min(kK64PerStage, num_k64 - k64_0);
        const uint32_t bytes = C::kABytes + C::kBBytes + nk64 * kSfAtomBytes +
                               sfb_copies * nk64 * kSfAtomBytes;
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
          bulk_g2s(sSfa, p.sfa + ((a0 / 128) * k64_per_row + k64_0) * kSfAtomBytes,
                   nk64 * kSfAtomBytes, &full[stage]);
          for (int blk = 0; blk < sfb_copies; ++blk) {
            const int64_t rb = b0 / 128 + blk;
            bulk_g2s(sSfb + blk * kK64PerStage * kSfAtomBytes,
                     p.sfb + (rb * k64_per_row + k64_0) * kSfAtomBytes, nk64 * kSfAtomBytes,
                     &full[stage]);
          }
        }
        if (p.sfb_8x4) {
          // 8x4 activation scales (BN <= 32 tokens): lane r puts row r's 4 scales of each K64
          // step at bytes [16 r, 16 r + 4) of that step's atom, as a 128x4 atom has them.
          const int64_t r = lane;
          for (int a = 0; a < nk64; ++a) {
            uint32_t v = 0;
            if (r < p.sfb_rows_padded && r < BN) {
              v = *reinterpret_cast<const uint32_t *>(
                  p.sfb + ((r / 8) * k64_per_row + (k64_0 + a)) * 32 + (r % 8) * 4);
            }
            *reinterpret_cast<uint32_t *>(sSfb + a * kSfAtomBytes + r * 16) = v;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
      }
    }
    // Tail: wait until the MMAs have released every stage still in use, so no tcgen05.commit
    // arrival is outstanding when the CTA exits.
    if (ok) {
      const uint32_t used = it < STAGES ? it : STAGES;
      for (uint32_t i = 0; i < used; ++i) {
        const uint32_t j = it - used + i;
        if (!mbar_wait_warp(&empty[j % STAGES], (j / STAGES) & 1, kWaitTimeoutNs)) {
          if (lane == 0) report_timeout(p.dev_status);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0;
      uint32_t tile_iter = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++tile_iter) {
        const int buf = static_cast<int>(tile_iter % C::kAccBufs);
        const uint32_t use = tile_iter / C::kAccBufs;
        if (use > 0 && !mbar_wait_bounded(&acc_empty[buf], (use - 1) & 1, kWaitTimeoutNs)) {
          report_timeout(p.dev_status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * C::kAccCols;
        int prev = -1;  // stage whose release (commit) is still to be issued
        for (int kt = 0; kt < num_kt; ++kt, ++it) {
          const int stage = static_cast<int>(it % STAGES);
          const uint32_t round = it / STAGES;
          if (!mbar_wait_bounded(&full[stage], round & 1, kWaitTimeoutNs) ||
              !mbar_wait_bounded(&sf_full[stage], round & 1, kWaitTimeoutNs)) {
            report_timeout(p.dev_status);
            ok = false;
            break;
          }
          tc_fence_after();
          // Release the previous stage only now: a barrier wait issued after a commit holds
          // this thread until that commit's MMAs have completed, so committing stage s before
          // waiting for stage s + 1 would leave the tensor pipe empty in between. Committed
          // here, the wait above overlaps the previous stage's MMAs.
          if (prev >= 0) tc_commit(&empty[prev]);
          const int nk64 = min(kK64PerStage, num_k64 - kt * kK64PerStage);
          const uint32_t sA = smem_u32(smem + C::kOffA + stage * C::kABytes);
          const uint32_t sB = smem_u32(smem + C::kOffB + stage * C::kBBytes);
          const uint32_t slot = tmem_base + C::kSfCol0 + stage * C::kSlotCols;
          for (int a = 0; a < nk64; ++a) {
            mma_nvf4(d_tmem, desc_sw128(sA + a * 32), desc_sw128(sB + a * 32), C::kIdesc,
                     slot + a * C::kSfaColsPerK64,
                     slot + kK64PerStage * C::kSfaColsPerK64 + a * C::kSfbColsPerK64,
                     (kt | a) != 0 ? 1u : 0u);
          }
          prev = stage;
        }
        if (prev >= 0) tc_commit(&empty[prev]);
        if (ok) tc_commit(&acc_full[buf]);
      }
    }
    __syncwarp();
  } else if (warp >= kSfWarp0 && warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------------ scale warps
    const int q = warp & 3;  // TMEM lane quarter this warp writes
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      for (int kt = 0; kt < num_kt; ++kt, ++it) {
        const int stage = static_cast<int>(it % STAGES);
        const uint32_t round = it / STAGES;
        if (!mbar_wait_warp(&full[stage], round & 1, kWaitTimeoutNs)) {
          if (lane == 0) report_timeout(p.dev_status);
          ok = false;
          break;
        }
        tc_fence_after();
        const int nk64 = min(kK64PerStage, num_k64 - kt * kK64PerStage);
        const uint8_t *sSfa = smem + C::kOffSfa + stage * C::kSfaBytes;
        const uint8_t *sSfb = smem + C::kOffSfb + stage * C::kSfbBytes;
        const uint32_t slot = lane_base + C::kSfCol0 + stage * C::kSlotCols;
        const uint32_t slot_b = slot + kK64PerStage * C::kSfaColsPerK64;
        // Each TMEM lane quarter q feeds accumulator rows 32 q .. 32 q + 31 and reads both
        // operands' scales from its own 32 lanes: A row m = 32 q + lane at column
        // (step base + q); B row n at lane 32 q + n % 32, column (step base + n / 32).
        // Writing A's aligned 4-column group with the same word keeps the store aligned;
        // B's scales are replicated into every quarter.
        for (int a = 0; a < nk64; ++a) {
          const uint32_t wa =
              *reinterpret_cast<const uint32_t *>(sSfa + a * kSfAtomBytes + lane * 16 + q * 4);
          tmem_st_x4_rep(slot + a * C::kSfaColsPerK64, wa);
          // atom row `lane` holds B rows lane + 32 t' (t' = 0..3) of its 128-row block
          const uint4 b0 = *reinterpret_cast<const uint4 *>(sSfb + a * kSfAtomBytes + lane * 16);
          if constexpr (C::kSfbBlocks == 1) {
            tmem_st_x4(slot_b + a * C::kSfbColsPerK64, b0.x, b0.y, b0.z, b0.w);
          } else {
            const uint4 b1 = *reinterpret_cast<const uint4 *>(
                sSfb + (kK64PerStage + a) * kSfAtomBytes + lane * 16);
            tmem_st_x8(slot_b + a * C::kSfbColsPerK64, b0, b1);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[stage]);
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------------ epilogue
    const int e = warp - kEpiWarp0;
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int col0 = (e / 4) * C::kColsPerEpiWarp;
    const int row = q * 32 + lane;
    const float alpha = __fdiv_rn(1.0f, __fmul_rn(p.ga[0], p.gw[0]));
    uint32_t tile_iter = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tile_iter) {
      int64_t a0, b0;
      tile_origin(t, a0, b0);
      const int buf = static_cast<int>(tile_iter % C::kAccBufs);
      const uint32_t use = tile_iter / C::kAccBufs;
      if (!mbar_wait_warp(&acc_full[buf], use & 1, kWaitTimeoutNs)) {
        if (lane == 0) report_timeout(p.dev_status);
        break;
      }
      tc_fence_after();
      const uint32_t t_acc =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols + col0;
      if constexpr (!SWAP) {
        // fp16 pairs of this thread's row, columns [col0, col0 + kColsPerEpiWarp)
        uint32_t h2[C::kColsPerEpiWarp / 2];
#pragma unroll
        for (int c = 0; c < C::kColsPerEpiWarp; c += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_acc + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            __half2 h = __floats2half2_rn(__fmul_rn(__uint_as_float(v[2 * j]), alpha),
                                          __fmul_rn(__uint_as_float(v[2 * j + 1]), alpha));
            h2[c / 2 + j] = *reinterpret_cast<uint32_t *>(&h);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        const int64_t m = a0 + row;
        if (m < p.M) {
          __half *dst = p.out + m * p.N + b0 + col0;
#pragma unroll
          for (int j = 0; j < C::kColsPerEpiWarp / 8; ++j) {
            if (b0 + col0 + 8 * j + 8 <= p.N) {
              uint4 pk;
              pk.x = h2[4 * j + 0];
              pk.y = h2[4 * j + 1];
              pk.z = h2[4 * j + 2];
              pk.w = h2[4 * j + 3];
              *reinterpret_cast<uint4 *>(dst + 8 * j) = pk;
            }
          }
        }
      } else {
        // accumulator lane = weight row n, column = token m
        float vals[C::kColsPerEpiWarp];
#pragma unroll
        for (int c = 0; c < C::kColsPerEpiWarp; c += 8) {
          uint32_t v[8];
          tmem_ld_32x32b_x8(t_acc + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) vals[c + j] = __fmul_rn(__uint_as_float(v[j]), alpha);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        const int64_t n = a0 + row;
        if (n < p.N) {
#pragma unroll
          for (int j = 0; j < C::kColsPerEpiWarp; ++j) {
            const int64_t m = b0 + col0 + j;
            if (m < p.M) p.out[m * p.N + n] = __float2half_rn(vals[j]);
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

// ------------------------------------------------------------------------------ CTA pairs

// Large-M form: a cluster of two CTAs computes a 256 x 256 tile with the pair MMA
// (tcgen05.mma.cta_group::2, M = 256, N = 256). CTA r of the pair holds rows
// [128 r, 128 r + 128) of the tile's A and of its B (each CTA stages half of B), and its
// tensor memory holds its 128 accumulator rows for all 256 columns, so every byte staged in a
// CTA feeds twice the MMA work of the single-CTA 128 x 256 tile (a third less L2 -> SM
// traffic per FLOP). Each CTA keeps the scales its half of the MMA reads in its own tensor
// memory: A's for its 128 rows and B's for all 256 (same lane/column layout as the
// single-CTA N = 256 case).
//
// Synchronisation (barriers named by the CTA holding them):
//   full[s]      even CTA; both producers arrive.expect_tx and both CTAs' tile copies
//                complete on it (count 2)
//   sf_ready[s]  each CTA; its own scale atoms landed (count 1, bulk copies)
//   sf_full[s]   even CTA; the four scale warps of both CTAs wrote their tensor memory
//                (count 8)
//   empty[s]     each CTA; pair-MMA commit multicast to both CTAs
//   acc_full     each CTA; pair-MMA commit multicast after a tile's last MMA
//   acc_empty    even CTA; the epilogue warps of both CTAs drained the accumulator (count 16)
// Every wait is bounded; a cluster barrier opens and closes the kernel so no CTA touches its
// peer's shared memory before the peer initialised it or after the peer exited.
template <int STAGES>
struct PairCfg {
  static constexpr int kN = 256;                        // MMA N (tile columns)
  static constexpr int kHalf = 128;                     // rows of A and of B per CTA
  static constexpr int kABytes = kHalf * kBKBytes;      // 16 KB
  static constexpr int kBBytes = kHalf * kBKBytes;      // 16 KB
  static constexpr int kSfaBytes = kK64PerStage * kSfAtomBytes;      // 2 KB
  static constexpr int kSfbBytes = 2 * kK64PerStage * kSfAtomBytes;  // 4 KB (all 256 rows)
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + STAGES * kABytes;
  static constexpr int kOffSfa = kOffB + STAGES * kBBytes;
  static constexpr int kOffSfb = kOffSfa + STAGES * kSfaBytes;
  static constexpr int kOffBar = kOffSfb + STAGES * kSfbBytes;
  // full[S], sf_ready[S], sf_full[S], empty[S], acc_full, acc_empty, tmem slot
  static constexpr int kBarBytes = (4 * STAGES + 2) * 8 + 16;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;
  static constexpr int kAccCols = kN;
  static constexpr int kSfaColsPerK64 = 4;
  static constexpr int kSfbColsPerK64 = 8;
  static constexpr int kSlotCols = kK64PerStage * (kSfaColsPerK64 + kSfbColsPerK64);
  static constexpr int kSfCol0 = kAccCols;
  static constexpr int kTmemCols = 512;
  static constexpr int kEpiWarps = 8;
  static constexpr int kColsPerEpiWarp = kN * 4 / kEpiWarps;  // 128
  static constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
  static_assert(kSfCol0 + STAGES * kSlotCols <= kTmemCols, "TMEM columns");
  static_assert(kSmemBytes <= 232448, "shared memory");
  // kind::mxf4nvf4: E2M1 A and B, K-major, UE4M3 scales; N >> 3 at bit 17, M >> 4 at bit 24
  static constexpr uint32_t kIdesc =
      (1u << 7) | (1u << 10) | (uint32_t(kN >> 3) << 17) | (uint32_t(256 >> 4) << 24);
};

template <int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<STAGES>::kThreads, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                           const __grid_constant__ CUtensorMap tmap_b, const KernelParams p) {
  using C = PairCfg<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *sf_ready = full + STAGES;
  uint64_t *sf_full = sf_ready + STAGES;
  uint64_t *empty = sf_full + STAGES;
  uint64_t *acc_full = empty + STAGES;
  uint64_t *acc_empty = acc_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int64_t K = p.K;
  const int num_k64 = static_cast<int>(K / 64);
  const int num_kt = (num_k64 + kK64PerStage - 1) / kK64PerStage;
  const int64_t k64_per_row = K / 64;
  const int num_tiles = p.tiles_a * p.tiles_b;  // tiles_a along M (256 rows), tiles_b along N
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&sf_ready[s], 1);
      mbar_init(&sf_full[s], 8);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * C::kEpiWarps);
    fence_mbar_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto tile_origin = [&](int t, int64_t &m0, int64_t &n0) {
    m0 = static_cast<int64_t>(t % p.tiles_a) * 256;
    n0 = static_cast<int64_t>(t / p.tiles_a) * C::kN;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (each CTA)
    uint32_t it = 0;
    bool ok = true;
    const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
    for (int t = pair; t < num_tiles && ok; t += npairs) {
      int64_t m0, n0;
      tile_origin(t, m0, n0);
      const int64_t arow = m0 + C::kHalf * rank;  // this CTA's A rows and B rows
      const int64_t brow = n0 + C::kHalf * rank;
      int sfb_copies = 0;
      for (int blk = 0; blk < 2; ++blk)
        if ((n0 / 128 + blk) * 128 < p.sfb_rows_padded) ++sfb_copies;
      const bool sfa_copy = arow < p.sfa_rows_padded;
      for (int kt = 0; kt < num_kt; ++kt, ++it) {
        const int stage = static_cast<int>(it % STAGES);
        const uint32_t round = it / STAGES;
        if (it >= STAGES) {
          if (!mbar_wait_cluster_warp(&empty[stage], (round - 1) & 1, kWaitTimeoutNs)) {
            if (lane == 0) report_timeout(p.dev_status);
            ok = false;
            break;
          }
        }
        const int k64_0 = kt * kK64PerStage;
        const int nk64 = min(kK64PerStage, num_k64 - k64_0);
        uint8_t *sA = smem + C::kOffA + stage * C::kABytes;
        uint8_t *sB = smem + C::kOffB + stage * C::kBBytes;
        uint8_t *sSfa = smem + C::kOffSfa + stage * C::kSfaBytes;
        uint8_t *sSfb = smem + C::kOffSfb + stage * C::kSfbBytes;
        if (lane == 0) {
          const uint32_t sf_bytes = ((sfa_copy ? 1 : 0) + sfb_copies) * nk64 * kSfAtomBytes;
          mbar_arrive_expect_tx(&sf_ready[stage], sf_bytes);
          if (sfa_copy)
            bulk_g2s(sSfa, p.sfa + ((arow / 128) * k64_per_row + k64_0) * kSfAtomBytes,
                     nk64 * kSfAtomBytes, &sf_ready[stage]);
          for (int blk = 0; blk < sfb_copies; ++blk) {
            const int64_t rb = n0 / 128 + blk;
            bulk_g2s(sSfb + blk * kK64PerStage * kSfAtomBytes,
                     p.sfb + (rb * k64_per_row + k64_0) * kSfAtomBytes, nk64 * kSfAtomBytes,
                     &sf_ready[stage]);
          }
          const uint32_t fullc = full0 + stage * 8;
          mbar_arrive_expect_tx_cluster(fullc, C::kABytes + C::kBBytes);
          tma_load_2d_pair(sA, &tmap_a, kt * kBKBytes, static_cast<int32_t>(arow), fullc);
          tma_load_2d_pair(sB, &tmap_b, kt * kBKBytes, static_cast<int32_t>(brow), fullc);
        }
        __syncwarp();
      }
    }
    if (ok) {
      const uint32_t used = it < STAGES ? it : STAGES;
      for (uint32_t i = 0; i < used; ++i) {
        const uint32_t j = it - used + i;
        if (!mbar_wait_cluster_warp(&empty[j % STAGES], (j / STAGES) & 1, kWaitTimeoutNs)) {
          if (lane == 0) report_timeout(p.dev_status);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      uint32_t it = 0;
      uint32_t tile_iter = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += npairs, ++tile_iter) {
        if (tile_iter > 0 && !mbar_wait_cluster(acc_empty, (tile_iter - 1) & 1, kWaitTimeoutNs)) {
          report_timeout(p.dev_status);
          break;
        }
        tc_fence_after();
        int prev = -1;  // stage whose release is still to be issued (see the single-CTA kernel)
        for (int kt = 0; kt < num_kt; ++kt, ++it) {
          const int stage = static_cast<int>(it % STAGES);
          const uint32_t round = it / STAGES;
          if (!mbar_wait_cluster(&full[stage], round & 1, kWaitTimeoutNs) ||
              !mbar_wait_cluster(&sf_full[stage], round & 1, kWaitTimeoutNs)) {
            report_timeout(p.dev_status);
            ok = false;
            break;
          }
          tc_fence_after();
          if (prev >= 0) tc_commit_pair(&empty[prev], 0x3);
          const int nk64 = min(kK64PerStage, num_k64 - kt * kK64PerStage);
          const uint32_t sA = smem_u32(smem + C::kOffA + stage * C::kABytes);
          const uint32_t sB = smem_u32(smem + C::kOffB + stage * C::kBBytes);
          const uint32_t slot = tmem_base + C::kSfCol0 + stage * C::kSlotCols;
          for (int a = 0; a < nk64; ++a) {
            mma_nvf4_pair(tmem_base, desc_sw128(sA + a * 32), desc_sw128(sB + a * 32), C::kIdesc,
                          slot + a * C::kSfaColsPerK64,
                          slot + kK64PerStage * C::kSfaColsPerK64 + a * C::kSfbColsPerK64,
                          (kt | a) != 0 ? 1u : 0u);
          }
          prev = stage;
        }
        if (prev >= 0) tc_commit_pair(&empty[prev], 0x3);
        if (ok) tc_commit_pair(acc_full, 0x3);
      }
    }
    __syncwarp();
  } else if (warp >= kSfWarp0 && warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------------ scale warps (each CTA)
    const int q = warp & 3;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t sf_full0 = mapa_shared(smem_u32(&sf_full[0]), 0);
    uint32_t it = 0;
    bool ok = true;
    for (int t = pair; t < num_tiles && ok; t += npairs) {
      for (int kt = 0; kt < num_kt; ++kt, ++it) {
        const int stage = static_cast<int>(it % STAGES);
        const uint32_t round = it / STAGES;
        if (!mbar_wait_warp(&sf_ready[stage], round & 1, kWaitTimeoutNs)) {
          if (lane == 0) report_timeout(p.dev_status);
          ok = false;
          break;
        }
        const int nk64 = min(kK64PerStage, num_k64 - kt * kK64PerStage);
        const uint8_t *sSfa = smem + C::kOffSfa + stage * C::kSfaBytes;
        const uint8_t *sSfb = smem + C::kOffSfb + stage * C::kSfbBytes;
        const uint32_t slot = lane_base + C::kSfCol0 + stage * C::kSlotCols;
        const uint32_t slot_b = slot + kK64PerStage * C::kSfaColsPerK64;
        // same tensor-memory scale layout as the single-CTA kernel with a 256-row B operand
        for (int a = 0; a < nk64; ++a) {
          const uint32_t wa =
              *reinterpret_cast<const uint32_t *>(sSfa + a * kSfAtomBytes + lane * 16 + q * 4);
          tmem_st_x4_rep(slot + a * C::kSfaColsPerK64, wa);
          const uint4 b0 = *reinterpret_cast<const uint4 *>(sSfb + a * kSfAtomBytes + lane * 16);
          const uint4 b1 = *reinterpret_cast<const uint4 *>(
              sSfb + (kK64PerStage + a) * kSfAtomBytes + lane * 16);
          tmem_st_x8(slot_b + a * C::kSfbColsPerK64, b0, b1);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(sf_full0 + stage * 8);
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------------ epilogue (each CTA)
    const int e = warp - kEpiWarp0;
    const int q = warp & 3;
    const int col0 = (e / 4) * C::kColsPerEpiWarp;
    const int row = q * 32 + lane;
    const float alpha = __fdiv_rn(1.0f, __fmul_rn(p.ga[0], p.gw[0]));
    const uint32_t acc_empty0 = mapa_shared(smem_u32(acc_empty), 0);
    uint32_t tile_iter = 0;
    for (int t = pair; t < num_tiles; t += npairs, ++tile_iter) {
      int64_t m0, n0;
      tile_origin(t, m0, n0);
      if (!mbar_wait_cluster_warp(acc_full, tile_iter & 1, kWaitTimeoutNs)) {
        if (lane == 0) report_timeout(p.dev_status);
        break;
      }
      tc_fence_after();
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + col0;
      uint32_t h2[C::kColsPerEpiWarp / 2];
#pragma unroll
      for (int c = 0; c < C::kColsPerEpiWarp; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_acc + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          __half2 h = __floats2half2_rn(__fmul_rn(__uint_as_float(v[2 * j]), alpha),
                                        __fmul_rn(__uint_as_float(v[2 * j + 1]), alpha));
          h2[c / 2 + j] = *reinterpret_cast<uint32_t *>(&h);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0);
      const int64_t m = m0 + C::kHalf * rank + row;
      if (m < p.M) {
        __half *dst = p.out + m * p.N + n0 + col0;
#pragma unroll
        for (int j = 0; j < C::kColsPerEpiWarp / 8; ++j) {
          if (n0 + col0 + 8 * j + 8 <= p.N) {
            uint4 pk;
            pk.x = h2[4 * j + 0];
            pk.y = h2[4 * j + 1];
            pk.z = h2[4 * j + 2];
            pk.w = h2[4 * j + 3];
            *reinterpret_cast<uint4 *>(dst + 8 * j) = pk;
          }
        }
      }
    }
  }

  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
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
static cudaError_t run(const GemmArgs &g, int num_sms, cudaStream_t st) {
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
    p.sfb_rows_padded = rows_sf_w;
  } else {
    if (!make_operand_map(&ma, g.w_q, g.N, kb, kBM)) return cudaErrorInvalidValue;
    if (!make_operand_map(&mb, g.a_q, g.M, kb, BN)) return cudaErrorInvalidValue;
    p.sfa = g.w_sf;
    p.sfb = g.a_sf;
    p.sfb_8x4 = g.a_layout == kSf8x4 ? 1 : 0;
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
  p.tiles_a = static_cast<int>((rows_a + kBM - 1) / kBM);
  p.tiles_b = static_cast<int>((rows_b + BN - 1) / BN);
  const int64_t tiles = static_cast<int64_t>(p.tiles_a) * p.tiles_b;
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_kernel<BN, STAGES, SWAP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  gemm_nvfp4_kernel<BN, STAGES, SWAP><<<grid, C::kThreads, C::kSmemBytes, st>>>(ma, mb, p);
  return cudaGetLastError();
}

// CTA pairs that can be resident at once (a pair needs two SMs of one GPC, so this can be
// below half the SM count); the persistent grid never exceeds it. Queried once per device.
template <int STAGES>
static int resident_pairs() {
  constexpr int kMaxDevices = 64;
  static std::once_flag once[kMaxDevices];
  static int pairs[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::call_once(once[dev], [dev]() {
    using C = PairCfg<STAGES>;
    pairs[dev] = 0;
    if (cudaFuncSetAttribute(gemm_nvfp4_pair_kernel<STAGES>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess)
      return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_pair_kernel<STAGES>, &cfg) == cudaSuccess)
      pairs[dev] = n;
  });
  return pairs[dev];
}

template <int STAGES>
static cudaError_t run_pair(const GemmArgs &g, int num_sms, cudaStream_t st) {
  (void)num_sms;
  using C = PairCfg<STAGES>;
  CUtensorMap ma, mb;
  KernelParams p{};
  const int64_t kb = g.K / 2;
  if (!make_operand_map(&ma, g.a_q, g.M, kb, C::kHalf)) return cudaErrorInvalidValue;
  if (!make_operand_map(&mb, g.w_q, g.N, kb, C::kHalf)) return cudaErrorInvalidValue;
  p.sfa = g.a_sf;
  p.sfb = g.w_sf;
  p.sfb_8x4 = 0;
  p.sfa_rows_padded = (g.M + 127) / 128 * 128;
  p.sfb_rows_padded = (g.N + 127) / 128 * 128;
  p.ga = g.a_g;
  p.gw = g.w_g;
  p.out = static_cast<__half *>(g.out);
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.dev_status = g.dev_status;
  p.tiles_a = static_cast<int>((g.M + 255) / 256);
  p.tiles_b = static_cast<int>((g.N + C::kN - 1) / C::kN);
  const int64_t tiles = static_cast<int64_t>(p.tiles_a) * p.tiles_b;
  const int resident = resident_pairs<STAGES>();
  if (resident <= 0) return cudaErrorLaunchOutOfResources;
  const int64_t pairs = tiles < resident ? tiles : resident;
  gemm_nvfp4_pair_kernel<STAGES><<<static_cast<int>(2 * pairs), C::kThreads, C::kSmemBytes, st>>>(
      ma, mb, p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs &g, int num_sms, cudaStream_t st) {
  if (g.M <= 32) return run<32, 6, true>(g, num_sms, st);
  if (g.M < 256 || num_sms < 2) return run<256, 4, false>(g, num_sms, st);
  return run_pair<5>(g, num_sms, st);
}

}  // namespace nvfp4
