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

// One TMEM column of this warp's 32 lanes. The A-operand scale word of lane quarter q is
// read from column base + q only (the measured layout), so that column is all a scale warp
// writes for it.
__device__ __forceinline__ void tmem_st_x1(uint32_t taddr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
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

// 32 consecutive TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, "
      "%31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
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
  int ga_per_row;   // ga holds one encode scale per activation row (per-token quantization)
  __half *out;
  int64_t M, N, K;  // problem shape in the caller's (unswapped) terms
  int tiles_a;      // tiles along the MMA A operand (128 rows each)
  int tiles_b;      // tiles along the MMA B operand (BN rows each)
  int32_t *dev_status;
};

// Output scale 1 / (ga * gw) of activation row m: ga[m] when the activation was quantized
// with one encode scale per row, else the scalar ga[0].
__device__ __forceinline__ float out_alpha(const float *ga, int per_row, const float *gw, int64_t m,
                                           int64_t M) {
  const float a = per_row ? (m < M ? ga[m] : 1.0f) : ga[0];
  return __fdiv_rn(1.0f, __fmul_rn(a, gw[0]));
}

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
          tmem_st_x1(slot + a * C::kSfaColsPerK64 + q, wa);  // quarter q reads column base + q
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
    uint32_t tile_iter = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tile_iter) {
      int64_t a0, b0;
      tile_origin(t, a0, b0);
      // this thread's output row (unswapped), or per column below (swapped)
      const float alpha = out_alpha(p.ga, p.ga_per_row, p.gw, a0 + row, p.M);
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
          for (int j = 0; j < 8; ++j)
            vals[c + j] = __fmul_rn(__uint_as_float(v[j]),
                                    out_alpha(p.ga, p.ga_per_row, p.gw, b0 + col0 + c + j, p.M));
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

// ------------------------------------------------------------------------------ small M

// Small-M (decode) form, M <= 32: the operands swap roles (128 weight rows are the MMA's A
// operand, the <= 32 tokens its N = 32 columns) and the work is split evenly over a resident
// grid of G CTAs ("stream-K"). CTA c owns the whole weight tiles c, c + G, ...; the K-steps
// of the tiles left over are cut into one contiguous slice per CTA, which it runs first, so
// every CTA streams the same amount of weight bytes whatever the tile count and ends on a
// whole tile. A CTA whose slice covers only part of a tile's K writes its fp32 partial
// accumulator to the workspace; the last CTA to finish such a tile (a per-tile arrival
// counter) adds the pieces in piece order (deterministic), writes the fp16 result and zeroes
// the counter again, so a workspace zero-filled once stays ready for the next call with no
// memset node per call. Activation scales: with the 8x4 layout the <= 32 rows of all K (K/16
// bytes each, four contiguous 8-row blocks) are copied into shared memory once per CTA; with
// the 128x4 layout the activation atoms of each ring stage are copied with the weight atoms.
constexpr int kDecBN = 32;
constexpr int kDecMaxSfbBytes = 48 * 1024;  // preloaded activation scales: K <= 24576

// NPL = 1: E4M3 activation scales. NPL = 3: fp32 activation scales split per row into three
// planes of E4M3 codes (act_planes.cu), copied with each ring stage. The MMA's N operand then holds the 32 token
// rows three times (rows 32 p + j = token j under plane p's scales), one N = 96 MMA per K step
// makes three partial sums per token, and the epilogue adds them.
template <int STAGES, int NPL = 1>
struct DecCfg {
  static constexpr int kMmaN = kDecBN * NPL;
  static constexpr int kABytes = kBM * kBKBytes;                 // 16 KB of weights
  static constexpr int kBBytes = kMmaN * kBKBytes;               // 4 KB of activations a copy
  static constexpr int kSfaBytes = kK64PerStage * kSfAtomBytes;  // 2 KB of weight scales
  // per stage: token scales, 128x4 atoms (E4M3 scales) or the plane words [K64][plane][32]
  static constexpr int kSfbBytes = NPL > 1 ? kK64PerStage * NPL * 128 : kK64PerStage * kSfAtomBytes;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + STAGES * kABytes;
  static constexpr int kOffSfa = kOffB + STAGES * kBBytes;
  static constexpr int kOffSfbStage = kOffSfa + STAGES * kSfaBytes;
  static constexpr int kOffBar = kOffSfbStage + STAGES * kSfbBytes;
  static constexpr int kAccBufs = 2;
  // full[S], empty[S], sf_full[S], sf_loaded[S], acc_full[2], acc_empty[2], sfb_ready, tmem
  // slot + flag
  static constexpr int kBarBytes = (4 * STAGES + 2 * kAccBufs + 1) * 8 + 16;
  static constexpr int kOffSfb = (kOffBar + kBarBytes + 127) / 128 * 128;  // 8x4 rows 0..31
  static constexpr int kAccCols = kMmaN;
  // per K step: A scales 4 columns, B scales 4 (column p for the rows of plane p)
  static constexpr int kSlotCols = kK64PerStage * (4 + 4);
  static_assert(kSlotCols == 32, "a full stage's scale words go out in one 32-column store");
  static constexpr int kSfCol0 = kAccBufs * kAccCols;
  static constexpr int kTmemCols = 512;
  static constexpr int kEpiWarps = 4;
  static constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
  static_assert(kSfCol0 + STAGES * kSlotCols <= kTmemCols, "TMEM columns");
  // E4M3 scales in 8x4: the copy of 4 blocks of K/64 x 32 bytes
  static constexpr int smem_bytes(int k64_total, bool sfb_8x4) {
    return kOffSfb + (NPL == 1 && sfb_8x4 ? k64_total * 128 : 0) + 1024;
  }
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(kMmaN >> 3) << 17) |
                                     (uint32_t(kBM >> 4) << 24);
};

struct DecParams {
  const uint8_t *w_sf;  // weight scales (128x4), MMA A operand
  const uint8_t *a_sf;  // activation scales (128x4 or 8x4), MMA B operand
  int a_sf_8x4;
  int64_t a_sf_rows;    // rows of the activation-scale buffer (padded)
  const float *ga;
  const float *gw;
  int ga_per_row;       // ga holds one encode scale per token
  __half *out;
  int64_t M, N, K;
  int tiles;            // 128-row weight tiles
  int max_pieces;       // CTAs a split tile's K range can be cut over
  float *partials;      // [split tiles][max_pieces][128][32] fp32
  int *counters;        // [tiles], zero on entry and zeroed again by each tile's last arriver
  int32_t *dev_status;
  const uint32_t *planes;  // NPL = 3: plane words [K/64][NPL][32] (launch_act_scale_planes)
  const float *row_alpha;  // NPL = 3: per-token output factors [32] from the same kernel
  int full_per_cta;     // whole tiles per CTA: CTA c owns tiles c, c + G, ... below tile_base
  int tile_base;        // = grid x full_per_cta; tiles from here on are split stream-K
  int64_t rem_units;    // (tiles - tile_base) x K-steps, cut evenly over CTAs 0 .. rem_ctas - 1
  int rem_ctas;         // min(grid, rem_units): every one of them gets at least one unit
  uint64_t wait_ns;     // limit of every bounded wait (2 s unless a test hook shortens it)
  int withhold_cta;     // test hook: CTA whose producer stops at ring position withhold_it
  int withhold_it;      // (-1: none; E4M3 activation scales only)
};

// Contiguous unit range [u0, u1) of CTA c among G over U units (units = tile x K-step).
__device__ __forceinline__ void dec_range(int64_t U, int c, int G, int64_t &u0, int64_t &u1) {
  u0 = static_cast<int64_t>(c) * U / G;
  u1 = static_cast<int64_t>(c + 1) * U / G;
}

// Index of the CTA whose range holds unit u.
__device__ __forceinline__ int dec_owner(int64_t u, int G, int64_t U) {
  return static_cast<int>(((u + 1) * G - 1) / U);
}

// A CTA's work in order: first its contiguous slice [r, r1) of the split region's units
// (tiles from tile_base on, each a run of num_kt K-steps), then its whole tiles c, c + G, ...
// The split pieces come first so that their partial writes and the last arrivers' sums run
// while the grid still streams, and every CTA ends on a whole tile (plain epilogue). Every
// role builds the same iterator and walks the same segments.
struct DecIter {
  int64_t r, r1;
  int next_full, full_left, G, num_kt, tile_base;
  __device__ __forceinline__ bool next(int &tile, int &kb, int &ke) {
    if (r < r1) {
      const int64_t t = r / num_kt;
      tile = tile_base + static_cast<int>(t);
      kb = static_cast<int>(r - t * num_kt);
      ke = static_cast<int>(kb + (r1 - r) < num_kt ? kb + (r1 - r) : num_kt);
      r += ke - kb;
      return true;
    }
    if (full_left > 0) {
      tile = next_full;
      kb = 0;
      ke = num_kt;
      next_full += G;
      --full_left;
      return true;
    }
    return false;
  }
};

// AND of `v` over the `nthreads` threads of named barrier `id` (a group of warps that must
// leave a loop together).
__device__ __forceinline__ bool group_all(bool v, int id, int nthreads) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Named barrier 1: the epilogue warps.
__device__ __forceinline__ bool epi_all(bool v, int nthreads) { return group_all(v, 1, nthreads); }


template <int STAGES, int NPL>
__global__ void __launch_bounds__(DecCfg<STAGES, NPL>::kThreads, 1)
    gemm_nvfp4_decode_kernel(const __grid_constant__ CUtensorMap tmap_w,
                             const __grid_constant__ CUtensorMap tmap_a, const DecParams p) {
  using C = DecCfg<STAGES, NPL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *empty = full + STAGES;
  uint64_t *sf_full = empty + STAGES;
  uint64_t *sf_loaded = sf_full + STAGES;
  uint64_t *acc_full = sf_loaded + STAGES;
  uint64_t *acc_empty = acc_full + C::kAccBufs;
  uint64_t *sfb_ready = acc_empty + C::kAccBufs;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sfb_ready + 1);
  volatile int *last_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint8_t *sfb_8x4 = smem + C::kOffSfb;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_k64 = static_cast<int>(p.K / 64);
  const int num_kt = (num_k64 + kK64PerStage - 1) / kK64PerStage;
  const int64_t k64_per_row = p.K / 64;
  const int G = gridDim.x;
  const int c = blockIdx.x;
  DecIter start;
  start.r = start.r1 = 0;
  if (c < p.rem_ctas) dec_range(p.rem_units, c, p.rem_ctas, start.r, start.r1);
  start.next_full = c;
  start.full_left = p.full_per_cta;
  start.G = G;
  start.num_kt = num_kt;
  start.tile_base = p.tile_base;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 4);
      mbar_init(&sf_loaded[s], 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::kEpiWarps);
    }
    mbar_init(sfb_ready, 1);  // the 8x4 copy (E4M3 activation scales)
    fence_mbar_init();
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_a);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The next kernel in the stream, if it was launched as a programmatic dependent, may start
  // as this kernel's CTAs leave their SMs; the GEMM kernels here only prefetch into L2 until
  // this kernel has finished.
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    uint32_t it = 0;
    bool ok = true;
    // Each stage has two barriers: sf_loaded[s] for the scale words (the scale warps start on
    // them as soon as they land) and full[s] for the weight and token tiles (the MMA thread).
    // This kernel is launched as a programmatic dependent of the kernel before it: while that
    // kernel finishes, the weights and weight scales of the first ring pass are prefetched
    // into L2 (no shared-memory write, nothing read before it is complete), and every copy
    // into shared memory waits for it (griddepcontrol.wait), so the kernel before may write
    // any of this call's inputs.
    if (lane == 0) {
      DecIter pit = start;
      int tile, kb, ke;
      int n = 0;
      while (n < STAGES && pit.next(tile, kb, ke)) {
        for (int kt = kb; kt < ke && n < STAGES; ++kt, ++n) {
          const int k64_0 = kt * kK64PerStage;
          const int nk64 = min(kK64PerStage, num_k64 - k64_0);
          tma_prefetch_l2_2d(&tmap_w, kt * kBKBytes, tile * kBM);
          bulk_prefetch_l2(p.w_sf + (static_cast<int64_t>(tile) * k64_per_row + k64_0) * kSfAtomBytes,
                           nk64 * kSfAtomBytes);
        }
      }
      griddep_wait();
      if (NPL == 1 && p.a_sf_8x4) {
        // rows 0..31 of the 8x4 activation scales: four blocks of K/64 x 32 contiguous bytes
        const uint32_t blk = static_cast<uint32_t>(k64_per_row * 32);
        const int nblk = static_cast<int>(p.a_sf_rows / 8);
        mbar_arrive_expect_tx(sfb_ready, blk * nblk);
        for (int b = 0; b < nblk; ++b)
          bulk_g2s(smem + C::kOffSfb + b * blk, p.a_sf + static_cast<int64_t>(b) * blk, blk, sfb_ready);
      }
    }
    __syncwarp();
    DecIter itr = start;
    int tile, kb, ke;
    while (ok && itr.next(tile, kb, ke)) {
      const int64_t w0 = static_cast<int64_t>(tile) * kBM;
      for (int kt = kb; kt < ke; ++kt, ++it) {
        const int stage = static_cast<int>(it % STAGES);
        const uint32_t round = it / STAGES;
        // test hook: this CTA issues nothing from this ring position on, so its consumers'
        // bounded waits run out with no copy in flight
        if (NPL == 1 && c == p.withhold_cta && static_cast<int>(it) == p.withhold_it) {
          ok = false;
          break;
        }
        if (it >= STAGES && !mbar_wait_warp(&empty[stage], (round - 1) & 1, p.wait_ns)) {
          if (lane == 0) report_timeout(p.dev_status);
          ok = false;
          break;
        }
        const int k64_0 = kt * kK64PerStage;
        const int nk64 = min(kK64PerStage, num_k64 - k64_0);
        if (lane == 0) {
          const uint32_t sf_bytes =
              nk64 * kSfAtomBytes + (NPL > 1 ? nk64 * NPL * 128 : p.a_sf_8x4 ? 0 : nk64 * kSfAtomBytes);
          mbar_arrive_expect_tx(&sf_loaded[stage], sf_bytes);
          bulk_g2s(smem + C::kOffSfa + stage * C::kSfaBytes,
                   p.w_sf + ((w0 / 128) * k64_per_row + k64_0) * kSfAtomBytes, nk64 * kSfAtomBytes,
                   &sf_loaded[stage]);
          if (NPL > 1)
            bulk_g2s(smem + C::kOffSfbStage + stage * C::kSfbBytes,
                     p.planes + static_cast<int64_t>(k64_0) * NPL * 32, nk64 * NPL * 128, &sf_loaded[stage]);
          else if (!p.a_sf_8x4)  // tokens 0..31: the first 128-row block of the 128x4 scales
            bulk_g2s(smem + C::kOffSfbStage + stage * C::kSfbBytes,
                     p.a_sf + static_cast<int64_t>(k64_0) * kSfAtomBytes, nk64 * kSfAtomBytes,
                     &sf_loaded[stage]);
          mbar_arrive_expect_tx(&full[stage], C::kABytes + C::kBBytes);
          tma_load_2d(smem + C::kOffA + stage * C::kABytes, &tmap_w, kt * kBKBytes,
                      static_cast<int32_t>(w0), &full[stage]);
#pragma unroll
          for (int pl = 0; pl < NPL; ++pl)  // the token tile once per scale plane
            tma_load_2d(smem + C::kOffB + stage * C::kBBytes + pl * (kDecBN * kBKBytes), &tmap_a,
                        kt * kBKBytes, 0, &full[stage]);
        }
        __syncwarp();
      }
    }
    if (ok) {
      const uint32_t used = it < STAGES ? it : STAGES;
      for (uint32_t i = 0; i < used; ++i) {
        const uint32_t j = it - used + i;
        if (!mbar_wait_warp(&empty[j % STAGES], (j / STAGES) & 1, p.wait_ns)) {
          if (lane == 0) report_timeout(p.dev_status);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, seg = 0;
      bool ok = true;
      DecIter itr = start;
      int tile, kb, ke;
      for (; ok && itr.next(tile, kb, ke); ++seg) {
        const int buf = static_cast<int>(seg % C::kAccBufs);
        const uint32_t use = seg / C::kAccBufs;
        if (use > 0 && !mbar_wait_bounded(&acc_empty[buf], (use - 1) & 1, p.wait_ns)) {
          report_timeout(p.dev_status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * C::kAccCols;
        int prev = -1;
        uint32_t prev_round = 0;
        for (int kt = kb; kt < ke; ++kt, ++it) {
          const int stage = static_cast<int>(it % STAGES);
          const uint32_t round = it / STAGES;
          if (!mbar_wait_bounded(&full[stage], round & 1, p.wait_ns) ||
              !mbar_wait_bounded(&sf_full[stage], round & 1, p.wait_ns)) {
            report_timeout(p.dev_status);
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk64 = min(kK64PerStage, num_k64 - kt * kK64PerStage);
          const uint32_t sA = smem_u32(smem + C::kOffA + stage * C::kABytes);
          const uint32_t sB = smem_u32(smem + C::kOffB + stage * C::kBBytes);
          const uint32_t slot = tmem_base + C::kSfCol0 + stage * C::kSlotCols;
          for (int a = 0; a < nk64; ++a) {
            mma_nvf4(d_tmem, desc_sw128(sA + a * 32), desc_sw128(sB + a * 32), C::kIdesc, slot + a * 4,
                     slot + kK64PerStage * 4 + a * 4, (kt != kb || a != 0) ? 1u : 0u);
          }
          // the stage goes back to the producer as soon as its MMAs complete (28.2 against
          // 28.6 us per call at M = 32, N = 28672, K = 8192 on B200, where releasing it
          // only after the next stage's barriers were passed kept it one stage longer)
          tc_commit(&empty[stage]);
          prev = stage;
          prev_round = round;
        }
        if (ok) tc_commit(&acc_full[buf]);
        // after a timeout the producer skips its final waits on the stages' releases, so the
        // MMAs issued so far are waited for here: none is in flight when the CTA frees its
        // tensor memory
        if (!ok && prev >= 0) (void)mbar_wait_bounded(&empty[prev], prev_round & 1, p.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp >= kSfWarp0 && warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------------ scale warps
    const int q = warp & 3;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t it = 0;
    bool ok = true;
    if (p.a_sf_8x4 && !mbar_wait_warp(sfb_ready, 0, p.wait_ns)) {
      if (lane == 0) report_timeout(p.dev_status);
      ok = false;
    }
    // token `lane`'s 8x4 words: block lane / 8, byte (lane % 8) * 4 of each 32-byte step
    const uint8_t *my8x4 = sfb_8x4 + (lane / 8) * (k64_per_row * 32) + (lane % 8) * 4;
    DecIter itr = start;
    int tile, kb, ke;
    while (ok && itr.next(tile, kb, ke)) {
      for (int kt = kb; kt < ke; ++kt, ++it) {
        const int stage = static_cast<int>(it % STAGES);
        const uint32_t round = it / STAGES;
        const int k64_0 = kt * kK64PerStage;
        const int nk64 = min(kK64PerStage, num_k64 - k64_0);
        if (!mbar_wait_warp(&sf_loaded[stage], round & 1, p.wait_ns)) {
          if (lane == 0) report_timeout(p.dev_status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t *sSfa = smem + C::kOffSfa + stage * C::kSfaBytes;
        const uint32_t slot = lane_base + C::kSfCol0 + stage * C::kSlotCols;
        // A (weights): row 32 q + lane's word at column (step base + q); B (tokens, N = 32):
        // token lane's word at lane 32 q + lane, column (step base + 0), in every quarter
        // (plane p's words at column base + p).
        if (nk64 == kK64PerStage) {
          // a full stage: the whole 32-column slot in one store. A's word fills its step's four
          // columns and the B words their columns; the columns the MMA does not read for this
          // lane quarter hold copies. (One store instead of eight measured 2 % faster.)
          uint32_t v[C::kSlotCols];
#pragma unroll
          for (int a = 0; a < kK64PerStage; ++a) {
            const uint32_t wa =
                *reinterpret_cast<const uint32_t *>(sSfa + a * kSfAtomBytes + lane * 16 + q * 4);
            uint32_t wb[4];
            if constexpr (NPL > 1) {
              const uint8_t *sB = smem + C::kOffSfbStage + stage * C::kSfbBytes + a * (NPL * 128) + lane * 4;
#pragma unroll
              for (int j = 0; j < 4; ++j)
                wb[j] = *reinterpret_cast<const uint32_t *>(sB + (j < NPL ? j : NPL - 1) * 128);
            } else {
              const uint32_t w =
                  p.a_sf_8x4 ? *reinterpret_cast<const uint32_t *>(my8x4 + (k64_0 + a) * 32)
                             : *reinterpret_cast<const uint32_t *>(smem + C::kOffSfbStage + stage * C::kSfbBytes +
                                                                   a * kSfAtomBytes + lane * 16);
#pragma unroll
              for (int j = 0; j < 4; ++j) wb[j] = w;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              v[4 * a + j] = wa;
              v[kK64PerStage * 4 + 4 * a + j] = wb[j];
            }
          }
          tmem_st_x32(slot, v);
        } else {
          for (int a = 0; a < nk64; ++a) {
            const uint32_t wa =
                *reinterpret_cast<const uint32_t *>(sSfa + a * kSfAtomBytes + lane * 16 + q * 4);
            tmem_st_x1(slot + a * 4 + q, wa);  // quarter q reads column base + q
            if constexpr (NPL > 1) {  // plane p's words to column p of the step
              const uint8_t *sB = smem + C::kOffSfbStage + stage * C::kSfbBytes + a * (NPL * 128) + lane * 4;
#pragma unroll
              for (int pl = 0; pl < NPL; ++pl)
                tmem_st_x1(slot + kK64PerStage * 4 + a * 4 + pl, *reinterpret_cast<const uint32_t *>(sB + pl * 128));
            } else if (p.a_sf_8x4) {
              tmem_st_x1(slot + kK64PerStage * 4 + a * 4,
                         *reinterpret_cast<const uint32_t *>(my8x4 + (k64_0 + a) * 32));
            } else {
              tmem_st_x1(slot + kK64PerStage * 4 + a * 4,
                         *reinterpret_cast<const uint32_t *>(smem + C::kOffSfbStage + stage * C::kSfbBytes +
                                                             a * kSfAtomBytes + lane * 16));
            }
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
    const int q = warp & 3;
    const int row = q * 32 + lane;  // weight row within the tile (accumulator lane)
    float alpha[kDecBN];  // per token (accumulator column)
    // the row factors and global scales may come from the kernel before this one, and the
    // output and workspace may still be in use by it
    griddep_wait();
    if constexpr (NPL > 1) {
#pragma unroll
      for (int j = 0; j < kDecBN; ++j) alpha[j] = __ldcg(p.row_alpha + j);
    } else {
#pragma unroll
      for (int j = 0; j < kDecBN; ++j) alpha[j] = out_alpha(p.ga, p.ga_per_row, p.gw, j, p.M);
    }
    uint32_t seg = 0;
    DecIter itr = start;
    int tile, kb, ke;
    for (; itr.next(tile, kb, ke); ++seg) {
      const int buf = static_cast<int>(seg % C::kAccBufs);
      const uint32_t use = seg / C::kAccBufs;
      // the four epilogue warps leave together (they meet at named barriers below)
      const bool got = mbar_wait_warp(&acc_full[buf], use & 1, p.wait_ns);
      if (!epi_all(got, C::kEpiWarps * 32)) {
        if (lane == 0) report_timeout(p.dev_status);
        break;
      }
      tc_fence_after();
      float vals[kDecBN];
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols;
      static_assert(kDecBN == 32, "one 32-column load per plane");
      {
        uint32_t v[kDecBN];
        tmem_ld_32x32b_x32(t_acc, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kDecBN; ++j) vals[j] = __uint_as_float(v[j]);
      }
      // the planes' partial sums of token j sit in columns j, 32 + j, 64 + j
#pragma unroll
      for (int pl = 1; pl < NPL; ++pl) {
        uint32_t v[kDecBN];
        tmem_ld_32x32b_x32(t_acc + pl * kDecBN, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kDecBN; ++j) vals[j] = __fadd_rn(vals[j], __uint_as_float(v[j]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      const int64_t n = static_cast<int64_t>(tile) * kBM + row;
      if (kb == 0 && ke == num_kt) {
        if (n < p.N) {
#pragma unroll
          for (int j = 0; j < kDecBN; ++j)
            if (j < p.M) p.out[j * p.N + n] = __float2half_rn(__fmul_rn(vals[j], alpha[j]));
        }
        continue;
      }
      // partial tile: publish this piece, the last arriver sums the pieces in order
      const int st = tile - p.tile_base;  // index among the split tiles
      const int64_t tu0 = static_cast<int64_t>(st) * num_kt;
      const int first = dec_owner(tu0, p.rem_ctas, p.rem_units);
      const int pieces = dec_owner(tu0 + num_kt - 1, p.rem_ctas, p.rem_units) - first + 1;
      const int piece = c - first;
      float *part_base = p.partials + static_cast<int64_t>(st) * p.max_pieces * kBM * kDecBN;
      float4 *mine = reinterpret_cast<float4 *>(part_base + (static_cast<int64_t>(piece) * kBM + row) * kDecBN);
#pragma unroll
      for (int j = 0; j < kDecBN / 4; ++j)
        mine[j] = make_float4(vals[4 * j], vals[4 * j + 1], vals[4 * j + 2], vals[4 * j + 3]);
      asm volatile("bar.sync 1, %0;" ::"n"(C::kEpiWarps * 32) : "memory");
      if (warp == kEpiWarp0 && lane == 0) {
        __threadfence();
        const int old = atomicAdd(p.counters + st, 1);
        *last_flag = (old == pieces - 1) ? 1 : 0;
        // the last arriver hands the counter back zeroed for the next call on this
        // workspace; a count past the pieces means the workspace was not zero on entry (a
        // count left part-way by a call that gave up cannot be told from a live one, so the
        // caller zero-fills the workspace again after any dev_status error)
        if (old == pieces - 1) atomicExch(p.counters + st, 0);
        if ((old < 0 || old >= pieces) && p.dev_status != nullptr) atomicOr(p.dev_status, kDevErrWorkspace);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(C::kEpiWarps * 32) : "memory");
      const bool last = *last_flag != 0;
      asm volatile("bar.sync 1, %0;" ::"n"(C::kEpiWarps * 32) : "memory");  // flag read before reuse
      if (!last) continue;
      __threadfence();
      float acc[kDecBN];
#pragma unroll
      for (int j = 0; j < kDecBN; ++j) acc[j] = 0.0f;
      for (int pc = 0; pc < pieces; ++pc) {
        if (pc == piece) {
#pragma unroll
          for (int j = 0; j < kDecBN; ++j) acc[j] = __fadd_rn(acc[j], vals[j]);
        } else {
          const float4 *src = reinterpret_cast<const float4 *>(
              part_base + (static_cast<int64_t>(pc) * kBM + row) * kDecBN);
#pragma unroll
          for (int j = 0; j < kDecBN / 4; ++j) {
            const float4 v4 = __ldcg(src + j);
            acc[4 * j] = __fadd_rn(acc[4 * j], v4.x);
            acc[4 * j + 1] = __fadd_rn(acc[4 * j + 1], v4.y);
            acc[4 * j + 2] = __fadd_rn(acc[4 * j + 2], v4.z);
            acc[4 * j + 3] = __fadd_rn(acc[4 * j + 3], v4.w);
          }
        }
      }
      if (n < p.N) {
#pragma unroll
        for (int j = 0; j < kDecBN; ++j)
          if (j < p.M) p.out[j * p.N + n] = __float2half_rn(__fmul_rn(acc[j], alpha[j]));
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
//                complete on it, and the four scale warps of both CTAs arrive once they
//                wrote their tensor memory (count 2 + 8): the MMA thread waits on one
//                barrier per stage
//   sf_ready[s]  each CTA; its own scale atoms landed (count 1, bulk copies)
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
  // the epilogue's staging of this CTA's 128 x 256 fp16 output tile: four 128-row x 64-column
  // boxes (16 KB each) in the 128-byte swizzled layout the TMA store reads
  static constexpr int kOutBoxBytes = kHalf * 128;
  static constexpr int kOffOut = kOffSfb + STAGES * kSfbBytes;
  static constexpr int kOffBar = kOffOut + 4 * kOutBoxBytes;
  // full[S], sf_ready[S], empty[S], acc_full, acc_empty, tmem slot
  static constexpr int kBarBytes = (3 * STAGES + 2) * 8 + 16;
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
                           const __grid_constant__ CUtensorMap tmap_b,
                           const __grid_constant__ CUtensorMap tmap_out, const KernelParams p) {
  using C = PairCfg<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *sf_ready = full + STAGES;
  uint64_t *empty = sf_ready + STAGES;
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
      mbar_init(&full[s], 2 + 8);  // two producers (with their bytes), eight scale warps
      mbar_init(&sf_ready[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * C::kEpiWarps);
    fence_mbar_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_out);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The next kernel in the stream, if it was launched as a programmatic dependent, may start
  // as this kernel's CTAs leave their SMs; the GEMM kernels here only prefetch into L2 until
  // this kernel has finished.
  griddep_launch_dependents();

  auto tile_origin = [&](int t, int64_t &m0, int64_t &n0) {
    m0 = static_cast<int64_t>(t % p.tiles_a) * 256;
    n0 = static_cast<int64_t>(t / p.tiles_a) * C::kN;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (each CTA)
    uint32_t it = 0;
    bool ok = true;
    const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
    // This kernel is launched as a programmatic dependent of the kernel before it: while that
    // kernel finishes, this CTA's B rows (the weights) and B's scale atoms for the first ring
    // pass are prefetched into L2 (no shared-memory write, nothing read before it is
    // complete), and every copy into shared memory waits for it (griddepcontrol.wait), so the
    // kernel before may write any of this call's inputs.
    if (lane == 0) {
      int n = 0;
      for (int t = pair; t < num_tiles && n < STAGES; t += npairs) {
        int64_t m0, n0;
        tile_origin(t, m0, n0);
        const int64_t brow = n0 + C::kHalf * rank;
        for (int kt = 0; kt < num_kt && n < STAGES; ++kt, ++n) {
          const int k64_0 = kt * kK64PerStage;
          const int nk64 = min(kK64PerStage, num_k64 - k64_0);
          tma_prefetch_l2_2d(&tmap_b, kt * kBKBytes, static_cast<int32_t>(brow));
          for (int blk = 0; blk < 2; ++blk) {
            const int64_t rb = n0 / 128 + blk;
            if (rb * 128 < p.sfb_rows_padded)
              bulk_prefetch_l2(p.sfb + (rb * k64_per_row + k64_0) * kSfAtomBytes, nk64 * kSfAtomBytes);
          }
        }
      }
      griddep_wait();
    }
    __syncwarp();
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
        // One barrier per stage (operands and scales), and the stage is released right after
        // its MMAs. (Measured on B200 against the single-CTA kernel's order, where a stage is
        // released only after the next stage's barriers: 2.5 % faster here together with the
        // one-store scale path below.)
        for (int kt = 0; kt < num_kt; ++kt, ++it) {
          const int stage = static_cast<int>(it % STAGES);
          const uint32_t round = it / STAGES;
          if (!mbar_wait_cluster(&full[stage], round & 1, kWaitTimeoutNs)) {
            report_timeout(p.dev_status);
            ok = false;
            break;
          }
          tc_fence_after();
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
          tc_commit_pair(&empty[stage], 0x3);
        }
        if (ok) tc_commit_pair(acc_full, 0x3);
      }
    }
    __syncwarp();
  } else if (warp >= kSfWarp0 && warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------------ scale warps (each CTA)
    const int q = warp & 3;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
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
        // same tensor-memory scale layout as the single-CTA kernel with a 256-row B operand;
        // a full stage's B words (four K64 steps x 8 columns) are contiguous columns and go
        // out in one 32-column store
        if (nk64 == kK64PerStage) {
          uint32_t bw[4 * C::kSfbColsPerK64];
#pragma unroll
          for (int a = 0; a < kK64PerStage; ++a) {
            const uint32_t wa =
                *reinterpret_cast<const uint32_t *>(sSfa + a * kSfAtomBytes + lane * 16 + q * 4);
            tmem_st_x1(slot + a * C::kSfaColsPerK64 + q, wa);  // quarter q reads column base + q
            const uint4 b0 = *reinterpret_cast<const uint4 *>(sSfb + a * kSfAtomBytes + lane * 16);
            const uint4 b1 = *reinterpret_cast<const uint4 *>(
                sSfb + (kK64PerStage + a) * kSfAtomBytes + lane * 16);
            bw[8 * a + 0] = b0.x; bw[8 * a + 1] = b0.y; bw[8 * a + 2] = b0.z; bw[8 * a + 3] = b0.w;
            bw[8 * a + 4] = b1.x; bw[8 * a + 5] = b1.y; bw[8 * a + 6] = b1.z; bw[8 * a + 7] = b1.w;
          }
          tmem_st_x32(slot_b, bw);
        } else {
          for (int a = 0; a < nk64; ++a) {
            const uint32_t wa =
                *reinterpret_cast<const uint32_t *>(sSfa + a * kSfAtomBytes + lane * 16 + q * 4);
            tmem_st_x1(slot + a * C::kSfaColsPerK64 + q, wa);
            const uint4 b0 = *reinterpret_cast<const uint4 *>(sSfb + a * kSfAtomBytes + lane * 16);
            const uint4 b1 = *reinterpret_cast<const uint4 *>(
                sSfb + (kK64PerStage + a) * kSfAtomBytes + lane * 16);
            tmem_st_x8(slot_b + a * C::kSfbColsPerK64, b0, b1);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(full0 + stage * 8);
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------------ epilogue (each CTA)
    // The fp16 tile goes out through shared memory: the warps drain the accumulator, release
    // it, write their rows into the 128-byte swizzled staging boxes, and one thread stores the
    // four boxes with TMA (full 128-byte lines; rows and columns past the output are not
    // written). Per-thread 16-byte global stores of 32 different rows had slowed the next
    // tile's MMAs by about 13 % on B200.
    const int e = warp - kEpiWarp0;
    const int q = warp & 3;
    const int col0 = (e / 4) * C::kColsPerEpiWarp;
    const int row = q * 32 + lane;
    const uint32_t acc_empty0 = mapa_shared(smem_u32(acc_empty), 0);
    uint8_t *const out_stage = smem + C::kOffOut;
    const bool issuer = e == 0 && lane == 0;
    // the global scales may come from the kernel before this one, and the output may still be
    // in use by it
    griddep_wait();
    uint32_t tile_iter = 0;
    for (int t = pair; t < num_tiles; t += npairs, ++tile_iter) {
      int64_t m0, n0;
      tile_origin(t, m0, n0);
      const float alpha = out_alpha(p.ga, p.ga_per_row, p.gw, m0 + C::kHalf * rank + row, p.M);
      // the eight warps leave together: they meet at named barriers below
      const bool got = mbar_wait_cluster_warp(acc_full, tile_iter & 1, kWaitTimeoutNs);
      if (!group_all(got, 1, C::kEpiWarps * 32)) {
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
      // the staging boxes are free once the previous tile's stores have read them
      if (issuer) bulk_wait_group_read0();
      named_bar_sync(1, C::kEpiWarps * 32);
      // this thread's 128 columns are 16 pieces of 8 fp16: piece k of box j goes to 16-byte
      // chunk k ^ (row % 8) of row `row` (the TMA 128-byte swizzle)
#pragma unroll
      for (int h = 0; h < C::kColsPerEpiWarp / 64; ++h) {
        uint8_t *box_row = out_stage + (col0 / 64 + h) * C::kOutBoxBytes + row * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int b = 32 * h + 4 * k;
          *reinterpret_cast<uint4 *>(box_row + ((k ^ (row & 7)) << 4)) =
              make_uint4(h2[b], h2[b + 1], h2[b + 2], h2[b + 3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1, C::kEpiWarps * 32);
      if (issuer) {
        const int64_t y = m0 + C::kHalf * rank;
        if (y < p.M) {
          for (int j = 0; j < 4; ++j) {
            const int64_t x = n0 + 64 * j;  // output column of the box
            if (x < p.N)
              tma_store_2d(&tmap_out, out_stage + j * C::kOutBoxBytes, static_cast<int32_t>(2 * x),
                           static_cast<int32_t>(y));
          }
        }
        bulk_commit_group();
      }
    }
    if (issuer) bulk_wait_group0();
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
// reads past the last row or column are zero-filled. L2 promotion of 128 bytes (one box row):
// on B200 the small-M GEMM ran 0.7 % faster than with 256-byte promotion, the prefill GEMM the same.
static bool encode_operand_map(CUtensorMap *map, const void *base, int64_t rows, int64_t k_bytes,
                               int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(k_bytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(k_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBKBytes), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Encoding a tensor map is host work of about a microsecond; decode-sized GEMMs run in tens
// of microseconds and are launched with the same operands over and over, so maps are kept
// in a small table keyed by (address, rows, row bytes, box rows). The map holds no device
// state: a hit for a freed-and-reused address describes the same layout and stays valid.
struct MapKey {
  const void *base;
  int64_t rows, k_bytes;
  int box_rows;
};

static bool make_operand_map(CUtensorMap *map, const void *base, int64_t rows, int64_t k_bytes,
                             int box_rows) {
  constexpr int kSlots = 64;
  static std::mutex mu;
  static MapKey keys[kSlots];
  static CUtensorMap maps[kSlots];
  static int used = 0, next = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
      const MapKey &k = keys[i];
      if (k.base == base && k.rows == rows && k.k_bytes == k_bytes && k.box_rows == box_rows) {
        *map = maps[i];
        return true;
      }
    }
  }
  if (!encode_operand_map(map, base, rows, k_bytes, box_rows)) return false;
  std::lock_guard<std::mutex> lock(mu);
  const int slot = used < kSlots ? used++ : next;
  next = (slot + 1) % kSlots;
  keys[slot] = MapKey{base, rows, k_bytes, box_rows};
  maps[slot] = *map;
  return true;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel, device and size: the
// call costs host time on every launch otherwise.
template <typename Kernel>
static cudaError_t ensure_smem_attr(Kernel kernel, int bytes) {
  struct Entry {
    const void *fn;
    int dev;
    int bytes;
  };
  static std::mutex mu;
  static Entry done[64];
  static int n = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const void *fn = reinterpret_cast<const void *>(kernel);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n; ++i)
    if (done[i].fn == fn && done[i].dev == dev && done[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  for (int i = 0; i < n; ++i)
    if (done[i].fn == fn && done[i].dev == dev) {
      done[i].bytes = bytes;
      return cudaSuccess;
    }
  if (n < 64) done[n++] = Entry{fn, dev, bytes};
  return cudaSuccess;
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
  p.ga_per_row = g.a_g_per_row;
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
  cudaError_t e = ensure_smem_attr(gemm_nvfp4_kernel<BN, STAGES, SWAP>, C::kSmemBytes);
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
    if (ensure_smem_attr(gemm_nvfp4_pair_kernel<STAGES>, C::kSmemBytes) != cudaSuccess) return;
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
  // the fp16 output [M, N] as bytes [M, 2N]: 128-byte (64-column) x 128-row boxes
  CUtensorMap mo;
  if (!make_operand_map(&mo, g.out, g.M, 2 * g.N, C::kHalf)) return cudaErrorInvalidValue;
  p.sfa = g.a_sf;
  p.sfb = g.w_sf;
  p.sfb_8x4 = 0;
  p.sfa_rows_padded = (g.M + 127) / 128 * 128;
  p.sfb_rows_padded = (g.N + 127) / 128 * 128;
  p.ga = g.a_g;
  p.gw = g.w_g;
  p.ga_per_row = g.a_g_per_row;
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
  // clusters of two (compiled in); a programmatic dependent of the kernel before it
  return launch_dependent(gemm_nvfp4_pair_kernel<STAGES>, dim3(static_cast<unsigned>(2 * pairs)),
                          dim3(C::kThreads), C::kSmemBytes, st, ma, mb, mo, p);
}

// Small-M stream-K layout for a device with num_sms SMs: grid, pieces per tile, workspace.
struct DecPlan {
  int grid = 0;
  int tiles = 0;
  int full_per_cta = 0;  // whole tiles per CTA, taken round robin from tile 0
  int64_t rem_units = 0; // K-steps of the tiles after those, cut evenly over rem_ctas CTAs
  int rem_ctas = 0;
  int max_pieces = 0;
  size_t partial_bytes = 0;
  bool usable = false;
};

// Workspace layout: the tile counters first, in a region sized by the workspace length alone,
// then the fp32 partial tiles. Every partial tile takes 16 KB, so a workspace of W bytes
// serves at most W / 16384 tiles and 16 * (W / 65536 + 1) bytes hold all their counters:
// whatever shape uses the workspace, its counters fall in this region and no call's partial
// tiles ever overwrite another shape's counters. The last arriver of every split tile
// zeroes its counter, so a workspace zero-filled once stays valid call after call.
static size_t counter_region(size_t W) { return 16 * (W / 65536 + 1); }

// Smallest workspace whose space after the counter region holds P bytes of partials; any
// larger one does too (counter_region(W) <= W / 4096 + 16).
static size_t workspace_for(size_t P) {
  return P == 0 ? 0 : (P + 16) + (P + 16 + 4094) / 4095 + 16;
}

static DecPlan dec_plan(int64_t M, int64_t N, int64_t K, int num_sms, bool sfb_fits = true) {
  DecPlan d;
  if (M > kDecBN || !sfb_fits) return d;
  const int64_t num_kt = (K / 64 + kK64PerStage - 1) / kK64PerStage;
  d.tiles = static_cast<int>((N + kBM - 1) / kBM);
  const int64_t U = d.tiles * num_kt;
  d.grid = static_cast<int>(U < num_sms ? U : num_sms);
  if (d.grid < 1) return d;
  d.full_per_cta = d.tiles / d.grid;
  const int64_t split_tiles = d.tiles - static_cast<int64_t>(d.full_per_cta) * d.grid;
  d.rem_units = split_tiles * num_kt;
  // with fewer split units than CTAs only the first rem_units CTAs take one each, so that no
  // CTA range inside a tile's K range is empty (the piece count assumes none is)
  d.rem_ctas = static_cast<int>(d.rem_units < d.grid ? d.rem_units : d.grid);
  if (split_tiles == 0) {
    d.max_pieces = 1;
    d.partial_bytes = 0;
  } else {
    // the most CTAs any split tile's K range meets (fewer split tiles than CTAs: a short loop)
    auto owner = [&](int64_t u) { return ((u + 1) * d.rem_ctas - 1) / d.rem_units; };
    int64_t mp = 1;
    for (int64_t t = 0; t < split_tiles; ++t) {
      const int64_t pieces = owner((t + 1) * num_kt - 1) - owner(t * num_kt) + 1;
      if (pieces > mp) mp = pieces;
    }
    d.max_pieces = static_cast<int>(mp);
    d.partial_bytes = static_cast<size_t>(split_tiles) * d.max_pieces * kBM * kDecBN * sizeof(float);
  }
  d.usable = true;
  return d;
}

static bool sfb_8x4_fits(int64_t K) { return K / 64 * 128 <= kDecMaxSfbBytes; }

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  const DecPlan d = dec_plan(M, N, K, num_sms, sfb_8x4_fits(K));
  return d.usable ? workspace_for(d.partial_bytes) : 0;
}

// fp32 activation scales: after the partial tiles, the plane words of one 32-row chunk
// ([K/64][3][32] words) and its 32 row factors.
static size_t act_planes_bytes(int64_t K) {
  return static_cast<size_t>(K / 64) * kActPlanes * 128 + kDecBN * sizeof(float);
}

size_t gemm_act_f32_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  const DecPlan d = dec_plan(M < kDecBN ? M : kDecBN, N, K, num_sms);
  return d.usable ? workspace_for(d.partial_bytes + act_planes_bytes(K)) : 0;
}

template <int STAGES, int NPL = 1>
static cudaError_t run_decode(const GemmArgs &g, const DecPlan &d, cudaStream_t st) {
  using C = DecCfg<STAGES, NPL>;
  CUtensorMap mw, ma;
  const int64_t kb = g.K / 2;
  if (!make_operand_map(&mw, g.w_q, g.N, kb, kBM)) return cudaErrorInvalidValue;
  if (!make_operand_map(&ma, g.a_q, g.M, kb, kDecBN)) return cudaErrorInvalidValue;
  DecParams p{};
  p.w_sf = g.w_sf;
  p.a_sf = g.a_sf;
  p.a_sf_8x4 = (NPL == 1 && g.a_layout == kSf8x4) ? 1 : 0;
  p.a_sf_rows = p.a_sf_8x4 ? (g.M + 7) / 8 * 8 : (g.M + 127) / 128 * 128;
  p.ga = g.a_g;
  p.gw = g.w_g;
  p.ga_per_row = g.a_g_per_row;
  p.out = static_cast<__half *>(g.out);
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.tiles = d.tiles;
  p.full_per_cta = d.full_per_cta;
  p.tile_base = d.full_per_cta * d.grid;
  p.rem_units = d.rem_units;
  p.rem_ctas = d.rem_ctas;
  p.max_pieces = d.max_pieces;
  p.counters = static_cast<int *>(g.workspace);
  p.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(g.workspace) +
                                         counter_region(g.workspace_bytes));
  p.dev_status = g.dev_status;
  const DebugHooks hooks = debug_hooks();
  p.wait_ns = hooks.wait_ns;
  p.withhold_cta = hooks.withhold_cta;
  p.withhold_it = static_cast<int>(hooks.withhold_it);
  cudaError_t e = cudaSuccess;
  const int smem = C::smem_bytes(static_cast<int>(g.K / 64), p.a_sf_8x4 != 0);
  e = ensure_smem_attr(gemm_nvfp4_decode_kernel<STAGES, NPL>, smem);
  if (e != cudaSuccess) return e;
  if constexpr (NPL > 1) {
    // the split kernel first (one CTA per row); the GEMM may start while it runs and waits
    // for it only where it reads the words and factors (griddepcontrol)
    static_assert(NPL == kActPlanes, "the split kernel writes kActPlanes planes");
    uint8_t *region = static_cast<uint8_t *>(g.workspace) + counter_region(g.workspace_bytes) + d.partial_bytes;
    uint32_t *planes = reinterpret_cast<uint32_t *>(region);
    float *row_alpha = reinterpret_cast<float *>(region + static_cast<size_t>(g.K / 64) * NPL * 128);
    p.planes = planes;
    p.row_alpha = row_alpha;
    e = launch_act_scale_planes(g.a_sf32, g.M, g.K, g.w_scale, planes, row_alpha, g.dev_status, st);
    if (e != cudaSuccess) return e;
  }
  // a programmatic dependent of the kernel before it: the weights of the first ring pass are
  // prefetched into L2 while that kernel's last CTAs finish
  return launch_dependent(gemm_nvfp4_decode_kernel<STAGES, NPL>, dim3(d.grid), dim3(C::kThreads), smem, st,
                          mw, ma, p);
}

bool gemm_act_f32_supported(int64_t K) { return K / 2 <= (int64_t(1) << 31); }

// The GEMM with fp32 activation scales: per 32 activation rows, the split kernel and the
// small-M stream-K kernel with three scale planes (the rows of a chunk are independent; the
// chunks run in stream order and share the workspace).
cudaError_t launch_gemm_act_f32(const GemmArgs &g, int num_sms, cudaStream_t st) {
  for (int64_t m0 = 0; m0 < g.M; m0 += kDecBN) {
    GemmArgs c = g;
    c.M = g.M - m0 < kDecBN ? g.M - m0 : kDecBN;
    c.a_q = g.a_q + m0 * (g.K / 2);
    c.a_sf32 = g.a_sf32 + m0 * (g.K / 16);
    c.out = static_cast<__half *>(g.out) + m0 * g.N;
    const DecPlan d = dec_plan(c.M, g.N, g.K, num_sms);
    if (!d.usable) return cudaErrorNotSupported;
    // 5 stages of 31.5 KB: 34.9 us per call (split kernel included) at M = 32, N = 28672,
    // K = 8192 on B200, against 35.1 (6 stages) and 36.3 (7)
    const cudaError_t e = run_decode<5, kActPlanes>(c, d, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm(const GemmArgs &g, int num_sms, cudaStream_t st) {
  if (g.M <= 32) {
    const DecPlan d = dec_plan(g.M, g.N, g.K, num_sms, sfb_8x4_fits(g.K));
    // 5 stages of 24 KB: 29.2 us per call at M = 32, N = 28672, K = 8192 on B200, against
    // 29.4 (6 stages), 30.1 (7), 30.3 (8), 30.8 (9) and 30.6 (4)
    if (d.usable) return run_decode<5>(g, d, st);
    return run<32, 6, true>(g, num_sms, st);
  }
  if (g.M < 256 || num_sms < 2) return run<256, 4, false>(g, num_sms, st);
  return run_pair<4>(g, num_sms, st);
}

}  // namespace nvfp4
