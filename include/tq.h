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
 *     or writing y, but they read the packed weights, scales and bias (model constants) before
 *     that wait.  Those must therefore not be written by the kernel enqueued immediately before
 *     a GEMM call on the same stream (e.g. tq_quantize_pack followed directly by tq_gemm): put
 *     any other operation, an event wait or a synchronisation in between.
 */
#ifndef TQ_H
#define TQ_H

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
 * Qwen2-7B shaped linears (ternary M <= 48, W4A16 M <= 16) and the tensor-core path above. */
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
 * tq_gemm_grouped / w4g_gemm_grouped -- several linears that read the same input, as a serving
 * engine's fused q/k/v or gate/up projections do: for g < count,
 *     y_g[M, N_g] = x[M, K] . What_g[N_g, K]^T (+ bias_g)
 * Same results contract as `count` separate tq_gemm / w4g_gemm calls (each element within the
 * stated bound; the split of K over CTAs may differ, so the bits may differ).  When
 * tq_select_path picks the decode path (M up to the crossover) on shapes it takes, all
 * matrices run in ONE kernel launch (one kernel boundary
 * instead of `count`); otherwise the call issues `count` single-matrix GEMMs.
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

/* tq_status_string -- static, human-readable text for a tq_status value. */
TQ_API const char* tq_status_string(int status);

/* tq_version -- library ABI version, (major << 16) | minor. */
TQ_API int tq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
