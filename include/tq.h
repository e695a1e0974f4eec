/*
 * tq.h -- C ABI of libtq.so: a weight-only low-bit linear layer for NVIDIA B200 (sm_100a).
 *
 *   y[M,N] = x[M,K] . What[N,K]^T (+ bias[N])      x, y, bias: fp16;   accumulation: fp32
 *
 * The weights stay packed in device memory and are decoded inside the GEMM kernels; they are
 * never written back as fp16.  Two packed formats:
 *
 *   ternary  What[n,k] = scale[n] * (code[n,k] - 1),  code in {0,1,2} (2 bits, 4 per byte)
 *   W4A16    What[n,k] = scales[n, k/128] * (u[n,k] - 8),  u in [0,15] (4 bits, 8 per int32)
 *
 * Sources (cited by short tag everywhere in this library):
 *   [TQ]  "Squeezing ternary-quantised models into vLLM: reverse engineering, reconciliation
 *          and kernel optimisation" (wzjinhao.cn/news/47283).  Section numbers are the article's.
 *   [VQ]  "Model quantisation - the vLLM runtime quantisation architecture"
 *          (notes.devxops.cn, LLM high-performance computing series).  Section numbers are the
 *          article's (chapter four = "weight parameters and post-load processing").
 *   [QS]  "10.6 Quantisation selection and vLLM in practice: decision tree + verification"
 *          (jennyma11.github.io/infra/ch10-06.html).
 *
 * Conventions shared by every entry point
 *   - Every tensor is row-major and contiguous.  fp16 data is passed as its IEEE binary16 bit
 *     pattern (uint16_t).  All pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory and keeps no per-call host state.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued
 *     asynchronously on it, on the device that is current in the calling thread ([TQ] §5.1:
 *     the library never selects device 0 behind the caller's back).  No entry point
 *     synchronises the stream, so calls can be captured in a CUDA graph ([TQ] §5.4).
 *   - Argument errors are detected on the host before anything is launched and returned as a
 *     negative tq_status; nothing is enqueued in that case.  A launch failure returns
 *     TQ_ERR_CUDA.  Kernels never trap: a bounded device-side wait that runs out records
 *     TQ_ERR_TIMEOUT in a device status word read by tq_device_status().
 *   - M == 0 or N == 0 is a valid empty problem (TQ_OK, nothing launched).  K must be > 0.
 *   - Inputs must be finite; results for Inf/NaN weights or activations are unspecified.
 *   - The tensor-core GEMM kernels are launched with programmatic dependent launch: they start
 *     while the preceding kernel on the stream is still running and wait for it before reading x
 *     or writing y, but they read the packed weights, scales, zero-points and bias (model
 *     constants) before that wait.  The library's own writers of packed data (the pack and
 *     repack calls) therefore end with an empty kernel in plain stream order, so a GEMM enqueued
 *     right after them sees their results.  A caller that writes weights, scales or bias with
 *     its OWN kernel must not enqueue a GEMM immediately after that kernel on the same stream:
 *     put any other operation, an event wait or a synchronisation in between.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TQ_OK = 0,
    TQ_ERR_NULL = -1,         /* a required pointer is NULL                                   */
    TQ_ERR_SHAPE = -2,        /* a size is negative, zero where it must not be, or too large  */
    TQ_ERR_ALIGN = -3,        /* a forced fast path was asked for with misaligned pointers    */
    TQ_ERR_DTYPE = -4,        /* unknown tq_dtype                                             */
    TQ_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed                         */
    TQ_ERR_TIMEOUT = -6,      /* a bounded device-side wait ran out (see tq_device_status)    */
    TQ_ERR_INVALID_CODE = -7, /* packed ternary data holds the unused code 0b11               */
    TQ_ERR_PATH = -8          /* unknown tq_path, or the forced path cannot take this shape   */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_F16 = 1 } tq_dtype;

/* GEMM execution paths.  AUTO applies tq_select_path(); the others force one path (tests).
 * The decode path runs at most 16 tokens per CTA; 17 <= M <= 64 runs ceil(M/16) token chunks
 * in the same launch.  tq_select_path picks decode up to the crossover measured on Llama-3-8B /
 * Qwen2-7B shaped linears (M <= 16 for both formats) and the tensor-core path above. */
typedef enum {
    TQ_PATH_AUTO = 0,
    TQ_PATH_DECODE = 1,  /* memory-bound skinny path, M <= 64: mma.sync on in-register decode  */
    TQ_PATH_PREFILL = 2, /* tensor-core path: TMA + smem decode + tcgen05.mma into TMEM         */
    TQ_PATH_GENERIC = 3  /* any shape / alignment: CUDA-core kernel (correct, not fast)         */
} tq_path;

typedef enum { TQ_FMT_TERNARY = 0, TQ_FMT_W4G128 = 1 } tq_format;

/* --------------------------------------------------------------------------------------------
 * tq_quantize_pack -- ternarise and pack one weight matrix ([TQ] §1, §3.1).
 *
 *   w       [N,K] fp32 (w_dtype = TQ_F32) or fp16 (TQ_F16), device.
 *   packed  [N, ceil(K/4)] uint8, device, written.  Element k of row n is code (packed[n][k/4]
 *           >> 2*(k%4)) & 3 ([TQ] §3.1 dequant_ternary, §4 unpack rule); the row stride is
 *           ceil(K/4) bytes and the codes past K in the last byte are 0b01 (= 0), the
 *           ceil-not-floor rule of [TQ] §3.2-3.3.
 *   scale   [N] fp16, device, written ([TQ] §2.1, §3.1: one fp16 scale per output row).
 *
 * Per row n, with S the exact sum of |w[n,k]| rounded once to fp64:
 *   t = 0.7 * (S / K)                                         (fp64; [TQ] §3.1: 0.7*mean|w|)
 *   code = 0b00 (-1) if w < -t,  0b10 (+1) if w > t,  0b01 (0) if |w| <= t     ([TQ] §1)
 *   scale = fp16_rne( A / nz )  where nz = #nonzero codes and A = exact sum of |w| over them,
 *           rounded once to fp64; scale = 0 when nz == 0.
 * The result is bit-exact: it does not depend on summation order.
 * Requires K <= 2^28, N*ceil(K/4) < 2^62.  Returns TQ_OK or an error listed above.
 * ------------------------------------------------------------------------------------------ */
TQ_API int tq_quantize_pack(const void* w, int w_dtype, uint8_t* packed, uint16_t* scale,
                     int64_t N, int64_t K, void* stream);

/* --------------------------------------------------------------------------------------------
 * tq_gemm -- y = x . What^T (+ bias) with ternary weights ([TQ] §2.3 apply_weights(input,
 * weight, bias, scale); §4 kernel; §4.2 decode to fp16 fragments, fp32 accumulation, scale
 * applied after the MMA).
 *
 *   x       [M,K] fp16, device.              packed  [N, ceil(K/4)] uint8 (tq_quantize_pack).
 *   scale   [N] fp16, device.                bias    [N] fp16 or NULL.
 *   y       [M,N] fp16, device, written.  x and y must not overlap.
 * Codes 0b11 are invalid; the output for a row holding one is unspecified (tq_validate_packed
 * finds them).  tq_gemm_ex forces a path: DECODE needs M <= 64, K % 64 == 0 and 16-byte aligned
 * x / packed; PREFILL needs K % 64 == 0 and 16-byte aligned x / packed / y; otherwise
 * TQ_ERR_PATH (shape) or TQ_ERR_ALIGN (pointers).  GENERIC takes any shape.
 * ------------------------------------------------------------------------------------------ */
TQ_API int tq_gemm(const uint16_t* x, const uint8_t* packed, const uint16_t* scale, const uint16_t* bias,
            uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream);
TQ_API int tq_gemm_ex(const uint16_t* x, const uint8_t* packed, const uint16_t* scale,
               const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, int path,
               void* stream);

/* --------------------------------------------------------------------------------------------
 * w4g_quantize_pack -- symmetric INT4, group size 128 along K, no act-order ([VQ] §5 GPTQ
 * config {"bits": 4, "group_size": 128, "desc_act": false, "sym": true}; [VQ] §4.2 packing of
 * 8 INT4 values per int32, weight [d_out, d_in/8], weight_scale [d_out, d_in/128]).
 *
 *   w        [N,K] fp32 or fp16, device; K % 128 == 0.
 *   qweight  [N, K/8] int32, device, written: nibble i (bits 4i..4i+3) of word j holds
 *            u = q + 8 for k = 8j + i.
 *   scales   [N, K/128] fp16, device, written.
 * Per (row n, group g): s = fp16_rne(max|w| / 7) (fp64 division); q = 0 if s == 0, else
 * clamp(rint(w / s), -8, 7) with the fp64 quotient by the STORED fp16 s, ties to even.
 * Bit-exact.  Calibration-based GPTQ (Hessian error feedback) is not performed.
 * ------------------------------------------------------------------------------------------ */
TQ_API int w4g_quantize_pack(const void* w, int w_dtype, int32_t* qweight, uint16_t* scales,
                      int64_t N, int64_t K, void* stream);

/* w4g_gemm -- y = x . What^T (+ bias), What = scales[n,k/128] * (u - 8) ([VQ] §5 forward:
 * INT4 weight x fp16 activation -> fp16 output).  Shapes as tq_gemm with K % 128 == 0.
 * DECODE needs M <= 64 and 16-byte aligned x / qweight; PREFILL needs 16-byte aligned pointers. */
TQ_API int w4g_gemm(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
             const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream);
TQ_API int w4g_gemm_ex(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, int path,
                void* stream);

/* --------------------------------------------------------------------------------------------
 * INT4 variants ([VQ] §5: GPTQ's sym / desc_act options, the weight_zp zero-point parameter and
 * the optional g_idx of activation ordering; [TQ] §2.1: AWQ checkpoints carry qweight, scales
 * and zeros).
 *
 * w4g_quantize_pack_ex -- the general INT4 packer, group size 128 along K.
 *   w        [N,K] fp32 or fp16, device; K % 128 == 0.
 *   perm     NULL, or device int32 [K]: a permutation of 0..K-1, the order in which the columns
 *            are quantised (activation order: column perm[j] belongs to group j / 128).  NULL:
 *            group g is columns 128 g .. 128 g + 127.
 *   qweight  [N, K/8] int32, written, in the ORIGINAL column order: nibble i of word j holds the
 *            code of column 8j + i.
 *   scales   [N, K/128] fp16, written, by group.
 *   zeros    NULL: symmetric, exactly as w4g_quantize_pack (u = q + 8, s = fp16(max|w|/7)).
 *            Else [N, K/128] uint8, written: asymmetric, per group lo = min(0, min w),
 *            hi = max(0, max w), s = fp16((hi - lo) / 15), z = clamp(rint(-lo / s), 0, 15),
 *            u = clamp(rint(w / s) + z, 0, 15) (fp64 quotients by the stored fp16 s, ties to
 *            even; an all-zero group gives s = 0, z = 0, u = 0).  What = s * (u - z).
 *   g_idx    NULL, or device int32 [K], written: the group of each column (k / 128 without perm).
 * Bit-exact.  With perm, qweight is cleared first (the kernel ORs nibbles into it).
 * Returns TQ_OK, TQ_ERR_DTYPE, TQ_ERR_SHAPE (K % 128), TQ_ERR_NULL or TQ_ERR_CUDA.
 *
 * w4g_gemm_zp / w4g_gemm_zp_ex -- y = x . What^T (+ bias) with What[n,k] = s[n, k/128] *
 *   (u[n,k] - zeros[n, k/128]) (asymmetric, consecutive groups); shapes, paths and errors as
 *   w4g_gemm / w4g_gemm_ex; zeros must not be NULL.
 *
 * Activation order at run time, the way the Marlin path of [VQ] §4.3 takes it: the product is
 * summed over k in the quantisation order, x . What^T = (x P) . (What P)^T, where P is the
 * column permutation perm.  Once, after packing:
 *   w4g_repack_act_order(qweight, perm, out, N, K): out[n, column j] = qweight[n, column
 *     perm[j]] (nibbles moved; out must not overlap qweight); the groups of `out` are then
 *     consecutive, so it is an ordinary W4A16 / zero-point matrix for the scales and zeros.
 * Per call:
 *   tq_permute_columns(x, perm, x_out, M, K): x_out[m, j] = x[m, perm[j]] (fp16 [M, K]; no
 *     overlap), then w4g_gemm / w4g_gemm_zp (or the batch calls) on (x_out, out, scales[, zeros]).
 * Both return TQ_OK, TQ_ERR_SHAPE, TQ_ERR_NULL or TQ_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
TQ_API int w4g_quantize_pack_ex(const void* w, int w_dtype, const int32_t* perm, int32_t* qweight,
                                uint16_t* scales, uint8_t* zeros, int32_t* g_idx, int64_t N, int64_t K,
                                void* stream);
TQ_API int w4g_gemm_zp(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                       const uint8_t* zeros, const uint16_t* bias, uint16_t* y, int64_t M, int64_t N,
                       int64_t K, void* stream);
TQ_API int w4g_gemm_zp_ex(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                          const uint8_t* zeros, const uint16_t* bias, uint16_t* y, int64_t M, int64_t N,
                          int64_t K, int path, void* stream);
TQ_API int w4g_repack_act_order(const int32_t* qweight, const int32_t* perm, int32_t* out, int64_t N,
                                int64_t K, void* stream);
TQ_API int tq_permute_columns(const uint16_t* x, const int32_t* perm, uint16_t* x_out, int64_t M,
                              int64_t K, void* stream);

/* --------------------------------------------------------------------------------------------
 * tq_gemm_grouped / w4g_gemm_grouped -- several linears that read the same input, as a serving
 * engine's fused q/k/v or gate/up projections do: for g < count,
 *     y_g[M, N_g] = x[M, K] . What_g[N_g, K]^T (+ bias_g)
 * Same results contract as `count` separate tq_gemm / w4g_gemm calls (each element within the
 * stated bound; the split of K over CTAs may differ, so the bits may differ).  When
 * tq_select_path picks the decode path (M up to the crossover) for every matrix, all matrices
 * run in ONE decode launch; when it picks the tensor-core prefill path for every matrix and their
 * tiles together fill at most four waves of the GPU, in ONE prefill launch whose grid covers the
 * row tiles of all of them (one kernel boundary instead of `count`, and small matrices fill the
 * GPU together; when those tiles would end in a nearly empty wave, the last few row tiles run in
 * a second launch with K split over a cluster); otherwise the call issues `count` single-matrix
 * GEMMs (each of which may split off its last row tiles the same way).
 *   count              1 .. 4
 *   packed / qweight   HOST array of `count` device pointers (layouts as in tq_gemm / w4g_gemm)
 *   scale / scales     HOST array of `count` device pointers
 *   bias               NULL (no bias) or a HOST array of `count` device pointers, each nullable
 *   y                  HOST array of `count` device pointers to [M, N_g] fp16 outputs
 *   N                  HOST array of `count` row counts
 * The host arrays are read during the call only.  Errors as in tq_gemm (TQ_ERR_SHAPE for count
 * outside 1..4 or a negative N_g).
 * ------------------------------------------------------------------------------------------ */
TQ_API int tq_gemm_grouped(const uint16_t* x, int count, const uint8_t* const* packed,
                           const uint16_t* const* scale, const uint16_t* const* bias,
                           uint16_t* const* y, const int64_t* N, int64_t M, int64_t K, void* stream);
TQ_API int w4g_gemm_grouped(const uint16_t* x, int count, const int32_t* const* qweight,
                            const uint16_t* const* scales, const uint16_t* const* bias,
                            uint16_t* const* y, const int64_t* N, int64_t M, int64_t K,
                            void* stream);

/* --------------------------------------------------------------------------------------------
 * tq_gemm_batch / w4g_gemm_batch -- a work list of independent linears that share M, all in ONE
 * persistent kernel launch ([TQ] §1: decode time goes to fetching packed weights; a serving
 * engine's decode step runs many small linears, and every launch boundary costs microseconds of
 * idle SMs).  For i < count:
 *     y_i[M, N_i] = x_i[M, K_i] . What_i[N_i, K_i]^T (+ bias_i)
 * The items must be independent: no item's y may overlap any item's x, weights, scales or bias,
 * nor another item's y.  Items may share x (fused q/k/v, gate/up).
 *
 *   items      HOST array of `count` tq_linear descriptors (read during the call only):
 *                x      [M, K] fp16, device, 16-byte aligned
 *                w      ternary: packed uint8 [N, K/4] (tq_quantize_pack), K % 64 == 0;
 *                       W4A16:   qweight int32 [N, K/8] (w4g_quantize_pack), K % 128 == 0;
 *                       device, 16-byte aligned
 *                scale  ternary: fp16 [N]; W4A16: fp16 [N, K/128]
 *                zeros  W4A16 only: NULL (symmetric) or uint8 [N, K/128] zero-points
 *                       (w4g_quantize_pack_ex); ignored by tq_gemm_batch
 *                bias   fp16 [N] or NULL
 *                y      [M, N] fp16, written
 *                N, K   N >= 0 (an item with N == 0 is skipped), 0 < K <= 2^28
 *   count      1 .. 8
 *   M          0 .. 32 tokens (0: nothing is launched)
 *   workspace  device buffer of at least tq_batch_workspace_size() bytes, 16-byte aligned,
 *              ZERO-FILLED before its first use (e.g. cudaMemset).  It holds the partial sums of
 *              row blocks that the kernel splits between CTAs and one arrival counter per split;
 *              every call leaves the counters at zero again, so a workspace is zeroed once and
 *              then reused by any number of calls.  Calls that may run concurrently (different
 *              streams) need different workspaces.  After a call that ended in TQ_ERR_TIMEOUT
 *              (tq_device_status) or a CUDA error, zero it again.
 * Results: the same bound as tq_gemm / w4g_gemm; deterministic (partial sums are added in K
 * order whichever CTA finishes last).  Errors: TQ_ERR_SHAPE (count, M, N, K out of range or
 * workspace too small), TQ_ERR_NULL, TQ_ERR_ALIGN, TQ_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
typedef struct tq_linear {
    const uint16_t* x;
    const void* w;
    const uint16_t* scale;
    const uint16_t* bias;
    uint16_t* y;
    int64_t N;
    int64_t K;
    const uint8_t* zeros;
} tq_linear;

TQ_API int tq_gemm_batch(const tq_linear* items, int count, int64_t M, void* workspace,
                         size_t workspace_bytes, void* stream);
TQ_API int w4g_gemm_batch(const tq_linear* items, int count, int64_t M, void* workspace,
                          size_t workspace_bytes, void* stream);

/* The batch calls run one of two kernels over the same work split (tests and benchmarks force
 * one with the _ex forms; AUTO picks by M):
 *   TQ_BATCH_MMA_SYNC     M <= 16: two CTAs per SM, mma.sync on the in-register decode;
 *   TQ_BATCH_TENSOR_CORE  M <= 32: one CTA per SM, decoded weights stored to tensor memory as
 *                         the A operand of tcgen05.mma (N = 16 or 32 tokens), accumulators in
 *                         tensor memory.
 * TQ_BATCH_INTERLEAVED may be OR-ed into the variant of tq_gemm_batch_ex: every item's ternary
 * weights are then in the pair-interleaved layout of tq_interleave_packed (same scales, same
 * results up to the fp32 summation order); the mma.sync kernel only (M <= 16).
 * Errors as above, plus TQ_ERR_PATH for an unknown variant, M > 16 with TQ_BATCH_MMA_SYNC, or
 * TQ_BATCH_INTERLEAVED with W4A16 items or the tensor-core kernel. */
typedef enum { TQ_BATCH_AUTO = 0, TQ_BATCH_MMA_SYNC = 1, TQ_BATCH_TENSOR_CORE = 2,
               TQ_BATCH_INTERLEAVED = 16 } tq_batch_variant;
TQ_API int tq_gemm_batch_ex(const tq_linear* items, int count, int64_t M, void* workspace,
                            size_t workspace_bytes, int variant, void* stream);
TQ_API int w4g_gemm_batch_ex(const tq_linear* items, int count, int64_t M, void* workspace,
                             size_t workspace_bytes, int variant, void* stream);

/* tq_gemm_batch_next / w4g_gemm_batch_next -- tq_gemm_batch_ex / w4g_gemm_batch_ex that also
 * names the batch call which will follow it on the same stream (a serving engine knows its next
 * layer): `next` is a HOST array of `next_count` (0 .. 8) items of which only w, N and K are read
 * (w 16-byte aligned, the same format and shape rules as `items`), and next_M its token count
 * (0 .. 32).  While this call computes, each CTA requests into L2 the packed-weight tiles that
 * the next call's CTA of the same index loads first (the mma.sync variant's ring fill, for
 * next_M <= 16; larger next_M prefetch nothing), so that launch starts on L2 hits.  Results are
 * exactly those of tq_gemm_batch_ex: the prefetch is a hint that moves no output.  Naming a
 * call that does not follow only costs the prefetched bytes.
 * ------------------------------------------------------------------------------------------ */
TQ_API int tq_gemm_batch_next(const tq_linear* items, int count, int64_t M, void* workspace,
                              size_t workspace_bytes, int variant, const tq_linear* next, int next_count,
                              int64_t next_M, void* stream);
TQ_API int w4g_gemm_batch_next(const tq_linear* items, int count, int64_t M, void* workspace,
                               size_t workspace_bytes, int variant, const tq_linear* next, int next_count,
                               int64_t next_M, void* stream);

/* --------------------------------------------------------------------------------------------
 * tq_interleave_packed -- relayout of packed ternary rows for the decode kernels ([VQ] §4.3: the
 * post-load repack a checkpoint's weights go through once before inference; the layout itself
 * is this library's, the pages have no counterpart).
 *
 *   packed  device, [N][K/4] bytes in the canonical layout of tq_quantize_pack.
 *   out     device, [N][K/4] bytes; may be `packed` itself (in place).
 *   K       multiple of 16 (rows of whole 32-bit words of 16 codes).
 * Per little-endian 32-bit word of a row (codes k = 16q .. 16q + 15, code s at bits 2s..2s+1 in
 * the canonical layout) the interleaved word holds k = 16q + 2j at bits 2j..2j+1 and
 * k = 16q + 2j + 1 at bits 16 + 2j.. (j = 0..7): the two fp16 halves a decode reads at one bit
 * position then hold two consecutive k, matching the activations' natural fp16 pairs.  The
 * scales are unchanged.  Pass the result to tq_gemm_batch_ex with TQ_BATCH_INTERLEAVED.
 * Like the pack calls it ends with an empty kernel in plain stream order (safe before a GEMM
 * that reads the weights before waiting for the previous kernel).
 * Errors: TQ_ERR_SHAPE (K not a multiple of 16, N < 0), TQ_ERR_NULL, TQ_ERR_ALIGN (pointers not
 * 4-byte aligned), TQ_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
TQ_API int tq_interleave_packed(const uint8_t* packed, uint8_t* out, int64_t N, int64_t K, void* stream);

/* --------------------------------------------------------------------------------------------
 * tq_gemm_batch_noalloc -- tq_gemm_batch without a workspace argument and without allocating.
 * (An addition of this library for its callers; the pages have no counterpart.)
 *
 * For callers that get no workspace buffer from their host framework and must not allocate
 * one: a custom operator behind an interface that passes only inputs and outputs, or a process
 * whose device memory is all reserved by its framework's caching allocator, where a raw
 * cudaMalloc fails or synchronises the device mid-step.  The batch kernel's scratch (arrival
 * counters and partial sums) lives instead in one static device array of 5.0 MiB inside the
 * library, which every GPU that loads the library holds until the process exits; it covers
 * GPUs with up to 160 SMs.
 *
 *   items, count, M, stream  as tq_gemm_batch (ternary linears, AUTO variant).
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current and caches it: make that first call before any stream capture.  Every
 * call clears the array's counters on `stream` before its kernel, and all calls share the
 * array: calls that may overlap on the GPU (different streams, or different host threads on
 * one device) race and give wrong results; serialise them.  No cudaMalloc, cudaFree or other
 * allocating call is made.
 * Errors: as tq_gemm_batch; TQ_ERR_SHAPE also when the current device has more SMs than the
 * array covers; TQ_ERR_CUDA when the address lookup or the clear fails.
 * ------------------------------------------------------------------------------------------ */
TQ_API int tq_gemm_batch_noalloc(const tq_linear* items, int count, int64_t M, void* stream);

/* tq_batch_workspace_size -- bytes of workspace tq_gemm_batch / w4g_gemm_batch need on the
 * device that is current in the calling thread (it depends on the number of SMs). */
TQ_API size_t tq_batch_workspace_size(void);

/* --------------------------------------------------------------------------------------------
 * tq_shard_plan -- what one rank of a tensor-parallel group holds of a packed matrix [N, K]
 * ([TQ] §5.2: under tensor parallelism each GPU keeps a part of the weight but the FULL per-row
 * scale, shared by broadcast, never gathered; [VQ] §4.2 _adjust_shard_indexes_for_packing: a
 * shard's offset and size along the packed dimension are divided by the packed factor).
 *   fmt    tq_format; mode: TQ_SHARD_ROWS or TQ_SHARD_K; world >= 1; 0 <= rank < world.
 *   TQ_SHARD_ROWS  output rows [row0, row0 + rows) with row0 = floor(N rank / world) (sizes
 *                  differ by at most one); every column; the scales of the rank's rows.  The
 *                  ranks' y are concatenated along N.
 *   TQ_SHARD_K     every row; input columns [k0, k0 + K/world); K / world must be a multiple of
 *                  4 (ternary: whole bytes) or 128 (W4A16: whole groups), else TQ_ERR_SHAPE.
 *                  Ternary scales are the full-row scales of all N rows (scale_full = 1); W4A16
 *                  scales / zero-points are the rank's groups.  The ranks' y are summed.
 *   out    packed0 / packed: the same columns in packed units (bytes for ternary, int32 words
 *          for W4A16), i.e. k0 / packed factor and (K / world) / packed factor; group0 / groups:
 *          W4A16 scale and zero-point columns.
 * Host arithmetic only (no device access).  Returns TQ_OK, TQ_ERR_SHAPE, TQ_ERR_PATH (fmt or
 * mode unknown) or TQ_ERR_NULL.
 * ------------------------------------------------------------------------------------------ */
typedef enum { TQ_SHARD_ROWS = 0, TQ_SHARD_K = 1 } tq_shard_mode;
typedef struct tq_shard {
    int64_t row0, rows;
    int64_t k0, cols;
    int64_t packed0, packed;
    int64_t group0, groups;
    int scale_full;
} tq_shard;
TQ_API int tq_shard_plan(int fmt, int mode, int64_t N, int64_t K, int world, int rank, tq_shard* out);

/* tq_validate_packed -- count the bytes of a packed ternary matrix [N, ceil(K/4)] that hold
 * the unused code 0b11 in one of their first K codes of the row ([TQ] §3.1: the table maps
 * 00/01/10 only).  *bad_count (device int) is OVERWRITTEN with the count (set to 0 first, on
 * `stream`).  Returns TQ_OK or an argument error; the count is ready when the stream is. */
TQ_API int tq_validate_packed(const uint8_t* packed, int64_t N, int64_t K, int* bad_count, void* stream);

/* tq_select_path -- the host-side dispatch rule used by TQ_PATH_AUTO, exposed so that it can be
 * tested without a GPU.  fmt is a tq_format; aligned16 says whether every pointer is 16-byte
 * aligned.  Returns a tq_path (never AUTO) or a negative tq_status for an invalid shape. */
TQ_API int tq_select_path(int fmt, int64_t M, int64_t N, int64_t K, int aligned16);

/* tq_device_status -- synchronise the current device, then read and clear the device-side
 * status word written by kernels whose bounded waits ran out.  Returns TQ_OK,
 * TQ_ERR_TIMEOUT, or TQ_ERR_CUDA if the synchronisation itself failed. */
TQ_API int tq_device_status(void);

/* --------------------------------------------------------------------------------------------
 * Failure-path test hooks ([TQ] §5.4-5.5: kernels that fail by status, never by hanging).
 * They exist so that tests can make a bounded device-side wait run out on purpose without
 * faulting or hanging the GPU; a serving process never calls them.  Both apply to the current
 * device, synchronise it, and stay in effect until changed.
 *
 * tq_debug_set_wait_limit -- every bounded wait (mbarrier polls of the GEMM kernels) gives up
 *   after `cycles` SM clock cycles instead of the default 4e9 (~2 s); cycles <= 0 restores the
 *   default.  A wait that gives up records TQ_ERR_TIMEOUT for tq_device_status(); the kernel
 *   then skips the rest of its work (its outputs are unspecified), frees what it holds and exits.
 * tq_debug_skip_activation_loads -- on != 0: the GEMM kernels' producers issue no activation
 *   (x) loads, so the stage barriers that count those bytes never complete and the consumers'
 *   waits run out; 0 restores normal operation.  Batch calls made while it is set leave their
 *   workspace counters untouched.
 * Returns TQ_OK or TQ_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
TQ_API int tq_debug_set_wait_limit(long long cycles);
TQ_API int tq_debug_skip_activation_loads(int on);

/* tq_status_string -- static, human-readable text for a tq_status value. */
TQ_API const char* tq_status_string(int status);

/* tq_version -- library ABI version, (major << 16) | minor. */
TQ_API int tq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
