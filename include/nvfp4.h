/*
 * nvfp4.h -- C ABI of libnvfp4.so: NVFP4 block-scaled quantization and the block-scaled
 * FP4 GEMM it feeds, for NVIDIA B200 (sm_100a).
 *
 * Conventions (all entry points):
 *  - Every pointer argument named as "device" is caller-owned device memory; the library
 *    never allocates, frees or retains it (scratch comes from caller workspaces, or from
 *    the fixed library array of nvfp4_global_scale_noalloc). Sizes are element counts
 *    unless stated.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Calls
 *    are asynchronous on that stream and return once the work is enqueued. The GEMM kernels
 *    are launched as programmatic dependents of the kernel before them on the stream: they
 *    may start while it finishes, but until it has completed they only prefetch weights
 *    into L2, so every call keeps plain stream order (any earlier work may write any input).
 *  - Return value: an nvfp4_status. Argument errors are detected on the host before any
 *    launch and nothing is enqueued. NVFP4_ERR_CUDA reports a launch error
 *    (cudaGetLastError after the launch). Errors raised later by a kernel surface on the
 *    stream as CUDA errors; a bounded wait that gave up inside the GEMM is reported through
 *    its `dev_status` word.
 *  - Functions are thread-safe and keep no per-call state: the same call may run on
 *    different streams concurrently (calls sharing a workspace must not overlap). The first
 *    call on a device resolves the tensor-map encoder, the SM count and the GEMM's
 *    resident cluster count once; encoded tensor maps are cached on the host; later calls
 *    issue no device queries.
 *  - Empty input is valid: M == 0 (or N == 0) returns NVFP4_OK and enqueues nothing. K and
 *    H must be positive.
 *
 * Number formats: E2M1 (OCP MX FP4: magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}, sign bit 3),
 * packed two per byte, element 2j in the low nibble of byte j. Block scales are E4M3
 * (OCP OFP8, largest 448), one per 16 consecutive elements along K. Global scales are fp32
 * "encode" scales g: a value x is stored as E2M1(x * g / s) with block scale s, and
 * dequantizes to q * s / g.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1, /* a size, layout, dtype or NULL pointer is not allowed */
  NVFP4_ERR_MISALIGNED = 2,  /* a pointer or leading dimension breaks the 16-byte rule */
  NVFP4_ERR_UNSUPPORTED = 3, /* valid but outside what this build implements */
  NVFP4_ERR_CUDA = 4,        /* a CUDA runtime/driver call or a launch failed */
  NVFP4_ERR_TIMEOUT = 5,     /* a bounded device wait gave up (see nvfp4_gemm dev_status) */
  NVFP4_ERR_SCRATCH_LIMIT = 6 /* input larger than a fixed library scratch array covers */
} nvfp4_status;

/* Block-scale buffer layouts. For R rows and C = K/16 scale columns:
 *  NVFP4_SF_LINEAR: [R, C] row-major, R*C bytes.
 *  NVFP4_SF_128x4 : rows padded to R' = ceil(R/128)*128, columns to C' = ceil(C/4)*4;
 *                   512-byte atoms of 128 rows x 4 columns, atom (r/128, c/4) at
 *                   ((r/128)*(C'/4) + c/4)*512; inside an atom row r%32 strides 16 bytes,
 *                   row group (r/32)%4 strides 4 bytes, column c%4 strides 1 byte.
 *                   (The block-scaling-factor layout named get_sf_out_offset_128x4 in
 *                   FlashInfer PR #3237 and "128x4" in FlashInfer PR #1355; the byte order
 *                   is the public cuBLAS one.)
 *  NVFP4_SF_8x4   : rows padded to R' = ceil(R/8)*8, columns to C' = ceil(C/4)*4; 32-byte
 *                   atoms of 8 rows x 4 columns at ((r/8)*(C'/4) + c/4)*32; row r%8
 *                   strides 4 bytes, column c%4 strides 1 byte. (The "8x4" layout of the
 *                   same two PRs; the pages name it without giving bytes.)
 * Padding bytes are written as zero by every producer in this library. */
typedef enum { NVFP4_SF_LINEAR = 0, NVFP4_SF_128x4 = 1, NVFP4_SF_8x4 = 2 } nvfp4_sf_layout;

/* Input element type of the activations: raw IEEE bfloat16 or binary16. */
typedef enum { NVFP4_IN_BF16 = 0, NVFP4_IN_FP16 = 1 } nvfp4_in_dtype;

/* Human-readable name of a status code (static storage, never NULL). */
NVFP4_API const char *nvfp4_status_str(int status);

/*
 * Bytes of a block-scale buffer for `rows` rows of `k` elements (k/16 scale columns) in
 * `layout`, padding included. Returns -1 for an unknown layout, k % 16 != 0 or a negative
 * size. Host only; no CUDA call.
 */
NVFP4_API int64_t nvfp4_sf_bytes(int64_t rows, int64_t k, int layout);

/*
 * Workspace bytes nvfp4_global_scale needs for an [M, K] input (a few KB at most; one fp32
 * partial maximum per CTA of the reduction). Host only.
 */
NVFP4_API size_t nvfp4_global_scale_workspace_bytes(int64_t M, int64_t K);

/*
 * Dynamic per-tensor global scale (the "dynamic scaling, max value per tensor" remedy of
 * "Building Custom TensorRT-LLM Plugins for Low-Latency FP8 Inference at Scale", section
 * "FP8 Saturation and Underflow", with workspace handed in as in its section "Thread-Safety
 * in Triton and Concurrent Streams"):
 *   amax = max |x[m,k]| over the tensor;  g = 448*6 / amax  (g = 1 if amax == 0; an
 *   overflowing quotient is clamped to FLT_MAX).
 * x        device, [M, K] elements of `dtype`, row stride `ldx` elements (ldx >= K).
 * g_out    device, one fp32, written.
 * workspace device, >= nvfp4_global_scale_workspace_bytes(M, K) bytes, 16-byte aligned;
 *          contents on entry do not matter (two launches: partial maxima, then the final
 *          reduction).
 * Requires: x 16-byte aligned, K % 16 == 0, ldx % 8 == 0. Inputs must be finite.
 */
NVFP4_API int nvfp4_global_scale(const void *x, int dtype, int64_t M, int64_t K, int64_t ldx, float *g_out,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * nvfp4_global_scale without a workspace argument, for callers that cannot allocate device
 * memory where they call it: an engine's enqueue() that is handed tensor pointers but no
 * allocator, or a runtime with a fixed memory plan that must not cudaMalloc/cudaFree per
 * call (both synchronize the device and can fail under memory pressure mid-request). The
 * pages have no counterpart to this entry point; it computes the same g as
 * nvfp4_global_scale (bit-identical result) from the same arguments minus the workspace.
 * The reduction scratch is a 16 KB array inside the library, one per device, kept until the
 * process exits. The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress) and the SM count; make that first call before any stream capture.
 * Limit: M * K <= 2^28 elements (268,435,456); larger inputs return
 * NVFP4_ERR_SCRATCH_LIMIT and enqueue nothing. All calls on a device share the array:
 * calls whose kernels may overlap on the GPU (unordered streams) race and can return a
 * wrong g -- order them on one stream. Allocates nothing.
 * Requires: x 16-byte aligned, K % 16 == 0, ldx % 8 == 0, ldx >= K, g_out 4-byte aligned.
 */
NVFP4_API int nvfp4_global_scale_noalloc(const void *x, int dtype, int64_t M, int64_t K,
                                         int64_t ldx, float *g_out, void *stream);

/*
 * NVFP4 quantize ("perf: optimize per-token nvfp4 quantization kernel", FlashInfer PR
 * #3237: cvt_warp_fp16_to_fp4 with the exact, non-fast-math path, the per-token global
 * scale with the row cached on chip, and get_sf_out_offset_128x4/8x4).
 * For every 16-element block of a row, with the row's global scale g:
 *   amax_b = max |x|;  s = (amax_b / 6) * g  (fp32, two roundings);  s_enc = E4M3(s)
 *   (round to nearest even, saturating at 448);  r = g / value(s_enc) (IEEE division;
 *   0 when the scale is 0; clamped to FLT_MAX);  q = E2M1(x * r) (round to nearest even,
 *   saturating at 6, sign kept).
 * x         device, [M, K] `dtype`, row stride ldx elements.
 * g         device fp32. per_token == 0: g[0] is read (the per-tensor encode scale).
 *           per_token == 1: g[m] = 448*6 / max_k |x[m,k]| is written for every row
 *           (1 for an all-zero row), then used for that row.
 * q         device, [M, K/2] packed E2M1 bytes, row stride K/2 bytes, written.
 * sf        device, nvfp4_sf_bytes(M, K, sf_layout) bytes, written (padding zeroed).
 * Requires: K % 16 == 0, ldx % 8 == 0, ldx >= K, x/q/sf 16-byte aligned, g 4-byte aligned.
 * Bit-exact: q and sf match the definition above for every finite input.
 */
NVFP4_API int nvfp4_quantize(const void *x, int dtype, int64_t M, int64_t K, int64_t ldx, float *g,
                   int per_token, uint8_t *q, uint8_t *sf, int sf_layout, void *stream);

/*
 * Fused SwiGLU + NVFP4 quantize ("Building Custom TensorRT-LLM Plugins for Low-Latency FP8
 * Inference at Scale", sections "The Cost of Non-Fused Quantization" and "Fusing the
 * Kernel in CUDA": the activation is computed in fp32 registers and only the quantized
 * result is written; here the output is NVFP4 instead of FP8).
 *   y[m,h] = silu(x[m,h]) * x[m,H+h],  silu(v) = v / (1 + e(-v)),
 * where e() is the library's fp32 exponential (clamp to [-87, 88]; k = the integer nearest
 * the exact product v * fl(log2 e), ties to even; Cody-Waite reduction with ln2 =
 * 0x3F317200 + 0x35BFBE8E; degree-7 Taylor polynomial by fused multiply-add; times 2^k). y stays fp32 and is quantized exactly as in
 * nvfp4_quantize with the per-tensor scale g[0]. Y is never written to memory.
 * x   device, [M, 2H] `dtype` (gate = columns [0,H), up = columns [H,2H)), row stride ldx.
 * g   device, one fp32, read.
 * q   device, [M, H/2] packed, written.   sf  device, nvfp4_sf_bytes(M, H, layout), written.
 * Requires: H % 16 == 0, ldx % 8 == 0, ldx >= 2H, x/q/sf 16-byte aligned.
 */
NVFP4_API int swiglu_nvfp4_quantize(const void *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                          const float *g, uint8_t *q, uint8_t *sf, int sf_layout, void *stream);

/*
 * Fused SwiGLU + FP8 E4M3 quantize, the kernel of "Building Custom TensorRT-LLM Plugins for
 * Low-Latency FP8 Inference at Scale" ("Fusing the Kernel in CUDA"; plugin I/O: BF16/FP16
 * [N, 2H] activations, an fp32 scale, FP8 E4M3 [N, H] output in linear layout):
 *   q[r, h] = E4M3( fp32(silu(gate) * up) * scale ), round to nearest even, saturating to
 *   +-448, NaN -> 0x7F; silu and its exponential exactly as in swiglu_nvfp4_quantize.
 * x      device, [M, 2H] bf16/fp16 row-major (gate = columns [0, H), up = [H, 2H)), row
 *        stride ldx >= 2H elements, 16-byte aligned rows.
 * scale  device fp32 [1]: multiplies y (a static calibration scale, or 448 / amax(y)).
 * q      device, [M, H] bytes, row-major, 16-byte aligned.
 * Requires H % 16 == 0. Y is never written to memory: 4NH bytes read + NH written.
 */
NVFP4_API int swiglu_fp8_quantize(const void *x, int dtype, int64_t M, int64_t H, int64_t ldx,
                                  const float *scale, uint8_t *q, void *stream);

/*
 * Scale-layout conversion (the 128x4 / 8x4 layouts of "feature: add fp4 mm using trtllm
 * backend", FlashInfer PR #1355, description item 1; weight/scale preparation).
 * nvfp4_sf_swizzle:   lin [R, C] bytes (row-major)  ->  out in `layout` (padding zeroed).
 * nvfp4_sf_unswizzle: in (layout)  ->  lin [R, C].
 * Both buffers device memory; C is the number of scale columns (K/16). NVFP4_SF_LINEAR is a
 * plain copy. Any alignment.
 */
NVFP4_API int nvfp4_sf_swizzle(const uint8_t *lin, uint8_t *out, int64_t R, int64_t C, int layout,
                     void *stream);
NVFP4_API int nvfp4_sf_unswizzle(const uint8_t *in, uint8_t *lin, int64_t R, int64_t C, int layout,
                       void *stream);

/*
 * Workspace bytes nvfp4_gemm needs for this shape on the current device. Non-zero only for
 * M <= 32 (K <= 24576): that path splits the K range of the weight tiles evenly over the
 * SMs ("stream-K") and keeps one int arrival counter per 128-row weight tile (at the front,
 * in 16 * (workspace_bytes / 65536 + 1) bytes whatever the shape) and fp32 partial tiles
 * [split tiles][pieces][128][32] after them (about 3.7 MB for N = 28672, K = 8192 on 148
 * SMs: each SM owns whole weight tiles and only the tiles left over are split).
 * Pass the same workspace_bytes with a given buffer. The workspace must be zero-filled
 * before its first use (cudaMemset once); every
 * call that completes leaves the counters zero again, so it needs no per-call reset. After
 * a call reports an error in dev_status, zero it again. Calls that share a workspace must
 * not overlap on the GPU. Returns 0 when no device is current. Host only.
 */
NVFP4_API size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * Block-scaled FP4 GEMM with FP16 output (tensor contract of "Fused Nvfp4 GEMM All Reduce
 * Plugin", TensorRT-Edge-LLM C++ API: activation FP4 [B,K], weight FP4 [N,K], FP8 weight
 * block scale [N,K/16], scalar FP32 global weight scale, result FP16 [B,N]; the AllReduce
 * is not part of this call):
 *   out[m,n] = fp16( sum_k E2M1(a[m,k]) * E4M3(sa[m,k/16]) * E2M1(w[n,k]) * E4M3(sw[n,k/16])
 *                    / (a_g * w_g) )
 * accumulated in fp32 on the tensor cores (tcgen05 block-scaled MMA, TMEM accumulator).
 * a_q      device, [M, K/2] packed E2M1 (row stride K/2 bytes).
 * a_sf     device, activation block scales in a_layout (NVFP4_SF_128x4 or NVFP4_SF_8x4),
 *          padding rows/columns zero (as written by nvfp4_quantize).
 * a_g      device, one fp32 (the activation's encode scale).
 * w_q      device, [N, K/2] packed E2M1.   w_sf device, 128x4 layout.   w_g device fp32.
 * out      device, [M, N] fp16, row-major, row stride N.
 * workspace/workspace_bytes: device, 16-byte aligned, >= nvfp4_gemm_workspace_bytes(M, N,
 *          K) (NVFP4_ERR_INVALID_ARG when smaller); may be NULL when that is 0. Zero-filled
 *          before its first use; each completed call leaves it zero-filled (see
 *          nvfp4_gemm_workspace_bytes).
 * dev_status: device int32 or NULL. Each bounded wait inside the kernel that gives up
 *          (about 2 s without progress) ORs 1 into it and the kernel returns without
 *          finishing. A split-K tile counter found at or above its tile's piece count (a
 *          workspace that was not zero-filled) ORs 4. A counter left part-way by a call
 *          that gave up is NOT detected by the next call, which would then add stale
 *          partial sums: after any call that set a dev_status bit, zero-fill the workspace
 *          again before reusing it. The caller reads dev_status after synchronizing.
 * Requires: K % 64 == 0, N % 8 == 0, a_q/w_q/a_sf/w_sf/out 16-byte aligned, a_layout in
 *          {128x4, 8x4} (8x4 only when M <= 32).
 */
NVFP4_API int nvfp4_gemm(const uint8_t *a_q, const uint8_t *a_sf, int a_layout, const float *a_g,
               const uint8_t *w_q, const uint8_t *w_sf, const float *w_g, void *out, int64_t M,
               int64_t N, int64_t K, void *workspace, size_t workspace_bytes, int32_t *dev_status,
               void *stream);

/*
 * The GEMM for an activation quantized per token (nvfp4_quantize with per_token = 1): same
 * arguments and contract as nvfp4_gemm except that a_g is a device fp32 [M] array, one
 * encode scale per activation row, so
 *   out[m,n] = fp16( sum_k E2M1(a[m,k]) * E4M3(sa[m,k/16]) * E2M1(w[n,k]) * E4M3(sw[n,k/16])
 *                    / (a_g[m] * w_g) ).
 * It closes the loop the per-token quantize PR ("perf: optimize per-token nvfp4 quantization
 * kernel", FlashInfer PR #3237, which tests per-token scales in the MoE path) implies: the
 * row scale is applied in the epilogue, fp32(1 / (a_g[m] * w_g)) times the fp32 accumulator.
 */
NVFP4_API int nvfp4_gemm_per_token(const uint8_t *a_q, const uint8_t *a_sf, int a_layout,
                                   const float *a_g, const uint8_t *w_q, const uint8_t *w_sf,
                                   const float *w_g, void *out, int64_t M, int64_t N, int64_t K,
                                   void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                   void *stream);

/*
 * The GEMM under the activation contract of "Fused Nvfp4 GEMM All Reduce Plugin"
 * (TensorRT-Edge-LLM C++ API, inputs [1] and [4]): the activation scales are combined FP32
 * values [B,1,K/16] (the E4M3 block scale already multiplied by the activation's FP32
 * dequantization scale) and the scalar FP32 weight scale multiplies (DequantizeLinear form):
 *   out[m,n] = fp16( sum_k E2M1(a[m,k]) * sa32[m,k/16] * E2M1(w[n,k]) * E4M3(sw[n,k/16])
 *                    * w_scale ).
 * The block-scaled MMA takes E4M3 scales only, so the kernel splits each activation row's
 * scales into three planes of E4M3 codes and one fp32 factor (rho = row maximum / 448):
 * rho * (v1 + v2 + v3) is within 2^-12 of each scale relative. One MMA per K step takes the
 * token rows once per plane (N = 96) and the epilogue adds the three fp32 partial sums. Per
 * 32 activation rows, in stream order, a small kernel splits the scales into the workspace
 * and the GEMM kernel, launched as its programmatic dependent, streams them from there.
 * a_q      device, [M, K/2] packed E2M1, 16-byte aligned.
 * a_sf32   device, fp32 [M, K/16] row-major (the [B,1,K/16] tensor), 16-byte aligned; every
 *          scale finite and >= 0. A negative, NaN or infinite scale is an argument error the
 *          kernel detects: its block counts as zero and 2 is ORed into *dev_status.
 * w_q      device, [N, K/2] packed E2M1.   w_sf device, 128x4 layout (E4M3).
 * w_scale  device, one fp32 (multiplies; 1 / the weight's encode scale).
 * out      device, [M, N] fp16, row-major.
 * workspace/workspace_bytes: device, 16-byte aligned, >= nvfp4_gemm_act_f32_workspace_bytes
 *          (M, N, K); used as in nvfp4_gemm, plus the plane words (K/64 x 384 bytes) and 32
 *          row factors of one 32-row chunk after the partial tiles, rewritten by every call.
 * dev_status: device int32 or NULL; bit 1 a bounded wait gave up (NVFP4_ERR_TIMEOUT), bit 2
 *          a bad activation scale, bit 4 a workspace that was not zero-filled (detected as
 *          in nvfp4_gemm: zero-fill the workspace again after any call that set a bit). The
 *          caller reads it after synchronizing.
 * Requires: K % 64 == 0, N % 8 == 0.
 */
NVFP4_API size_t nvfp4_gemm_act_f32_workspace_bytes(int64_t M, int64_t N, int64_t K);
NVFP4_API int nvfp4_gemm_act_f32(const uint8_t *a_q, const float *a_sf32, const uint8_t *w_q,
                                 const uint8_t *w_sf, const float *w_scale, void *out, int64_t M,
                                 int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                                 int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
