// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, bulk/tensor TMA copies,
// tcgen05 (TMEM allocation, block-scaled MMA, shared->TMEM copies, TMEM loads) and the
// FP4/FP8 conversions. Device-only; no host code.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace nvfp4 {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// Makes barrier initialisation visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Programmatic dependent launch: let the next kernel in the stream (launched with the
// programmatic-serialization attribute) start now; and, in that kernel, wait until the
// kernels it depends on have finished and their memory writes are visible.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete. Gives up after `timeout_ns` of
// wall time without completion and returns false; the caller reports the timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 255u) == 0u && globaltimer_ns() - t0 > timeout_ns) return false;
  }
}


// Whole-warp form of mbar_wait_bounded: every lane waits, then the warp reconverges and
// agrees on the outcome, so warp-collective (.sync.aligned) instructions that follow run
// with all 32 lanes together.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, uint64_t timeout_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------------------------------------ TMA

// Untiled bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                        uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Tiled 2-D tensor copy global -> shared (x = innermost coordinate in elements).
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const void *tmap, int32_t x, int32_t y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Tiled 2-D tensor copy shared -> global (x = innermost coordinate in elements), tracked in
// this thread's bulk async-group. Parts of the box outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const void *tmap, const void *smem_src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap),
               "r"(x), "r"(y), "r"(smem_u32(smem_src))
               : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until this thread's committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Waits until this thread's committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_group0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Makes this thread's ordinary shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Prefetch into L2 only (no shared-memory write, no completion to wait for): a 2-D tile of a
// tensor map, or `bytes` (a multiple of 16, 16-byte aligned) of global memory.
__device__ __forceinline__ void tma_prefetch_l2_2d(const void *tmap, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(tmap), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_prefetch_l2(const void *gmem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gmem_src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void *tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ------------------------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t *smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D(tmem) (+)= A(smem desc) x B(smem desc)^T with per-16 E4M3 scales from TMEM.
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Arrives on `bar` once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------------------------ CTA pairs
// Helpers for the two-CTA (cluster of 2) form of the tensor-core instructions: one MMA issued
// by the even CTA of the pair computes a 256-row tile whose halves live in the two CTAs'
// shared memory and tensor memory.

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// All threads of both CTAs (like __syncthreads across the cluster).
__device__ __forceinline__ void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (default semantics: release at
// CTA scope). Used after tcgen05.wait::st / wait::ld, which already hold the thread until its
// tensor-memory stores or loads are complete. (Release at cluster scope also waits for the
// thread's other outstanding memory operations: about a microsecond per call measured on
// B200, on the critical path of every stage.)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}

// Registers the bytes a tensor copy will deliver to a (possibly remote) mbarrier and arrives.
__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t caddr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cluster.b64 _, [%0], %1;" ::"r"(caddr), "r"(bytes)
               : "memory");
}

// try_wait for barriers that the peer CTA (or a multicast tensor-core commit) arrives on.
// Default semantics (acquire at CTA scope): what the waiter consumes is tensor-copy data and
// tensor-memory contents, whose completion the barrier's phase itself reports; an acquire at
// cluster scope made every wait cost a memory round trip.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
  return mbar_try_wait(bar, parity);
}

__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((++spins & 255u) == 0u && globaltimer_ns() - t0 > timeout_ns) return false;
  }
}

__device__ __forceinline__ bool mbar_wait_cluster_warp(uint64_t *bar, uint32_t parity,
                                                       uint64_t timeout_ns) {
  const bool ok = mbar_wait_cluster(bar, parity, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

// 2-D tiled copy into this CTA's shared memory whose completion is counted on the mbarrier
// at shared::cluster address `mbar` (the even CTA's barrier for a CTA pair). No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const void *tmap, int32_t x, int32_t y,
                                                 uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t *smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Pair MMA (issued by one thread of the even CTA): each CTA's tensor memory accumulates its
// 128 rows of the 256-row tile; A and B descriptors address the same offsets in both CTAs.
__device__ __forceinline__ void mma_nvf4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Arrive on the mbarrier at this shared offset in every CTA of `cta_mask` once all prior
// pair MMAs of this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 bits, repeated over 8 consecutive columns.
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
}

// 32 lanes x 32 bits, repeated over 32 consecutive columns.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// ------------------------------------------------------------------------------ FP4 / FP8


// fp32 -> E4M3 code (round to nearest even, saturate to +-448).
__device__ __forceinline__ uint32_t cvt_e4m3(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return static_cast<uint32_t>(out) & 0xFFu;
}

// Two fp32 -> two signed E4M3 codes, lo in the low byte (round to nearest even, saturate to
// +-448, NaN -> NaN).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(hi), "f"(lo));
  return static_cast<uint32_t>(out);
}

// E4M3 code -> fp32 (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(code & 0xFFu)));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// ------------------------------------------------------------------------------ loads

// 32 bytes (16 x 16-bit elements) through the read-only path, not kept in L1.
__device__ __forceinline__ void ld_nc_v8(const void *p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

// 16 bytes through the read-only path, not kept in L1.
__device__ __forceinline__ void ld_nc_v4(const void *p, uint32_t *r) {
  asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "l"(p));
}

// One 16-element block: a single 32-byte load when the address is 32-byte aligned (V8),
// else two 16-byte loads.
template <bool V8>
__device__ __forceinline__ void ld_block16(const uint16_t *p, uint32_t (&r)[8]) {
  if constexpr (V8) {
    ld_nc_v8(p, r);
  } else {
    ld_nc_v4(p, r);
    ld_nc_v4(p + 8, r + 4);
  }
}

__device__ __forceinline__ void st_cs_u64(void *p, uint64_t v) {
  asm volatile("st.global.cs.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Two packed 16-bit inputs -> two fp32 (exact for bf16 and fp16).
template <int DTYPE>
__device__ __forceinline__ void unpack2(uint32_t w, float &lo, float &hi) {
  if constexpr (DTYPE == 0) {  // bfloat16: the upper half of an fp32
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
  } else {
    __half2 h = *reinterpret_cast<__half2 *>(&w);
    float2 f = __half22float2(h);
    lo = f.x;
    hi = f.y;
  }
}

}  // namespace nvfp4

namespace nvfp4 {

// (a0, a1) * (b, b) with one packed fp32x2 multiply (two IEEE round-to-nearest products).
__device__ __forceinline__ void mul2_rn(float a0, float a1, float b, float &d0, float &d1) {
  uint64_t d;
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%1, %2};\n\t"
      "mov.b64 rb, {%3, %3};\n\t"
      "mul.rn.f32x2 %0, ra, rb;\n\t}"
      : "=l"(d)
      : "f"(a0), "f"(a1), "f"(b));
  d0 = __uint_as_float(static_cast<uint32_t>(d));
  d1 = __uint_as_float(static_cast<uint32_t>(d >> 32));
}

// Four E2M1 byte pairs -> one 32-bit word (byte j from pair j).
__device__ __forceinline__ uint32_t e2m1x8_from_pairs(float y0, float y1, float y2, float y3,
                                                     float y4, float y5, float y6, float y7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(y0), "f"(y1), "f"(y2), "f"(y3), "f"(y4), "f"(y5), "f"(y6), "f"(y7));
  return out;
}

// max |x| over the 16 elements of 8 packed 16-bit words, in the input's own type (exact),
// returned as fp32. max.xorsign.abs takes |a|, |b| for free; the sign it leaves (the xor of
// the signs) is cleared at the end.
template <int DTYPE>
__device__ __forceinline__ float amax16_packed(const uint32_t (&w)[8]) {
  uint32_t m0 = w[0], m1 = w[1];
#pragma unroll
  for (int i = 2; i < 8; i += 2) {
    if constexpr (DTYPE == 0) {
      asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m0) : "r"(w[i]));
      asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m1) : "r"(w[i + 1]));
    } else {
      asm("max.xorsign.abs.f16x2 %0, %0, %1;" : "+r"(m0) : "r"(w[i]));
      asm("max.xorsign.abs.f16x2 %0, %0, %1;" : "+r"(m1) : "r"(w[i + 1]));
    }
  }
  if constexpr (DTYPE == 0) {
    asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m0) : "r"(m1));
  } else {
    asm("max.xorsign.abs.f16x2 %0, %0, %1;" : "+r"(m0) : "r"(m1));
  }
  const uint32_t m = m0 & 0x7FFF7FFFu;
  float lo, hi;
  if constexpr (DTYPE == 0) {
    lo = __uint_as_float(m << 16);
    hi = __uint_as_float(m & 0xFFFF0000u);
  } else {
    __half2 h = *reinterpret_cast<const __half2 *>(&m);
    lo = __low2float(h);
    hi = __high2float(h);
  }
  return fmaxf(lo, hi);
}

}  // namespace nvfp4

namespace nvfp4 {

// Packed fp32x2 arithmetic (sm_100a): two independent IEEE round-to-nearest results per
// instruction, bit-identical to the scalar operations.
struct F2 {
  float x, y;
};

__device__ __forceinline__ F2 f2_from_u64(uint64_t v) {
  return F2{__uint_as_float(static_cast<uint32_t>(v)), __uint_as_float(static_cast<uint32_t>(v >> 32))};
}

__device__ __forceinline__ F2 fma2_rn(F2 a, F2 b, F2 c) {
  uint64_t d;
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%1, %2};\n\t"
      "mov.b64 rb, {%3, %4};\n\t"
      "mov.b64 rc, {%5, %6};\n\t"
      "fma.rn.f32x2 %0, ra, rb, rc;\n\t}"
      : "=l"(d)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return f2_from_u64(d);
}

__device__ __forceinline__ F2 mul2f_rn(F2 a, F2 b) {
  uint64_t d;
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%1, %2};\n\t"
      "mov.b64 rb, {%3, %4};\n\t"
      "mul.rn.f32x2 %0, ra, rb;\n\t}"
      : "=l"(d)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return f2_from_u64(d);
}

__device__ __forceinline__ F2 add2f_rn(F2 a, F2 b) {
  uint64_t d;
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%1, %2};\n\t"
      "mov.b64 rb, {%3, %4};\n\t"
      "add.rn.f32x2 %0, ra, rb;\n\t}"
      : "=l"(d)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return f2_from_u64(d);
}

}  // namespace nvfp4
