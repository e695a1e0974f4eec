// tq_common.cuh -- shared device helpers: binary16 rounding from fp64, exact sums, reductions,
// and the internal launch interface between the kernel files and the C ABI (tq_api.cu).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_ptx.cuh"

namespace tq {

// fp64 -> IEEE 754 binary16 bit pattern, round to nearest, ties to even (written from the
// format definition).  d = M * 2^(e-52) with a 53-bit M; the binary16 quantum in the binade of
// d is 2^(max(e,-14) - 10); round M to a multiple of it and rebuild the pattern.  A rounding
// carry from 2047 quanta moves into the exponent field, and from exponent 15 it lands exactly
// on the infinity pattern 0x7C00, as IEEE 754 overflow under round-to-nearest requires.
__device__ __forceinline__ uint16_t f64_to_f16_rne(double d) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(d));
  const uint32_t sign = static_cast<uint32_t>((b >> 48) & 0x8000u);
  const int ef = static_cast<int>((b >> 52) & 0x7FF);
  const unsigned long long frac = b & ((1ull << 52) - 1);
  if (ef == 0x7FF) return static_cast<uint16_t>(sign | (frac ? 0x7E00u : 0x7C00u));
  if (ef == 0) return static_cast<uint16_t>(sign);  // zero, or far below the binary16 range
  const int e = ef - 1023;
  if (e > 15) return static_cast<uint16_t>(sign | 0x7C00u);
  const unsigned long long M = (1ull << 52) | frac;
  const int eh = e < -14 ? -14 : e;
  int shift = (eh - 10) - (e - 52);  // >= 42
  if (shift > 63) shift = 63;        // M < 2^53 < 2^62: rounds to zero either way
  unsigned long long r = M >> shift;
  const unsigned long long rem = M & ((1ull << shift) - 1);
  const unsigned long long half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (r & 1ull))) ++r;
  return static_cast<uint16_t>(sign | static_cast<uint32_t>(((eh + 14) << 10) + static_cast<int>(r)));
}

__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
  return static_cast<double>(__half2float(__ushort_as_half(h)));
}

// Exact sum of n nonnegative doubles that are integer multiples of 2^-149 and below 2^230,
// rounded once to fp64 (ties to even).  Fixed point with 32-bit limbs, LSB = 2^-149.
// Runs in one thread; used once per row, so it is not performance critical.
__device__ __noinline__ double exact_sum_fixed149(const double* v, int n) {
  constexpr int kLimbs = 12;  // 384 bits
  uint32_t L[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) L[i] = 0;
  for (int i = 0; i < n; ++i) {
    const double d = v[i];
    if (!(d > 0.0)) continue;
    const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(d));
    const int ef = static_cast<int>((b >> 52) & 0x7FF);
    unsigned long long M = (b & ((1ull << 52) - 1)) | (ef ? (1ull << 52) : 0ull);
    int pos = (ef ? ef : 1) - 1075 + 149;  // position of M's unit bit, in units of 2^-149
    while (pos < 0) {                      // only zero bits are dropped (d is a multiple)
      M >>= 1;
      ++pos;
    }
    const int limb = pos >> 5, sh = pos & 31;
    const unsigned long long lo = M << sh;
    const unsigned long long hi = sh ? (M >> (64 - sh)) : 0ull;
    uint32_t add[3] = {static_cast<uint32_t>(lo), static_cast<uint32_t>(lo >> 32),
                       static_cast<uint32_t>(hi)};
    unsigned long long carry = 0;
    for (int k = limb; k < kLimbs; ++k) {
      const unsigned long long a = (k - limb < 3) ? add[k - limb] : 0u;
      const unsigned long long s = static_cast<unsigned long long>(L[k]) + a + carry;
      L[k] = static_cast<uint32_t>(s);
      carry = s >> 32;
      if (k - limb >= 2 && carry == 0) break;
    }
  }
  int top = -1;
  for (int k = kLimbs - 1; k >= 0; --k)
    if (L[k]) {
      top = k;
      break;
    }
  if (top < 0) return 0.0;
  const int H = 32 * top + (31 - __clz(L[top]));  // highest set bit position
  // the 64-bit window of bits [H-63, H]
  auto bits64_at = [&](int lo) -> unsigned long long {
    unsigned long long r = 0;
    for (int j = 0; j < 64; j += 32) {
      const int p = lo + j;  // bits p .. p+31
      unsigned long long part = 0;
      if (p + 32 > 0 && p < 32 * kLimbs) {
        const int k = p >> 5;  // arithmetic shift: floor division
        const int s = p - 32 * k;
        const unsigned long long a = (k >= 0 && k < kLimbs) ? L[k] : 0u;
        const unsigned long long c = (k + 1 >= 0 && k + 1 < kLimbs) ? L[k + 1] : 0u;
        part = ((a | (c << 32)) >> s) & 0xFFFFFFFFull;
      }
      r |= part << j;
    }
    return r;
  };
  if (H < 53) {  // the whole value fits in 53 bits: exact
    const unsigned long long I = bits64_at(0);
    return static_cast<double>(I) * 0x1p-149;
  }
  const unsigned long long win = bits64_at(H - 63);
  unsigned long long M53 = win >> 11;
  const unsigned long long rbit = (win >> 10) & 1ull;
  bool sticky = (win & 0x3FFull) != 0;
  const int below = H - 63;  // bits at positions < below are not in the window
  for (int k = 0; k < kLimbs && !sticky; ++k) {
    const int p0 = 32 * k;
    if (p0 >= below) break;
    const int nb = below - p0 >= 32 ? 32 : below - p0;
    const uint32_t mask = nb == 32 ? 0xFFFFFFFFu : ((1u << nb) - 1u);
    if (L[k] & mask) sticky = true;
  }
  int Hr = H;
  if (rbit && (sticky || (M53 & 1ull))) {
    ++M53;
    if (M53 == (1ull << 53)) {
      M53 >>= 1;
      ++Hr;
    }
  }
  const long long bexp = static_cast<long long>(Hr - 149 + 1023);
  const unsigned long long bits = (static_cast<unsigned long long>(bexp) << 52) | (M53 & ((1ull << 52) - 1));
  return __longlong_as_double(static_cast<long long>(bits));
}

// --------------------------------------------------------------------------------------------
// Block reductions (fixed trees: deterministic)
// --------------------------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ int warp_max_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Sum over the block; every thread gets the result.  `scratch` holds >= 32 elements.
template <typename T>
__device__ __forceinline__ T block_sum(T v, T* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  T r = (lane < nw) ? scratch[lane] : T(0);
  r = warp_sum(r);
  return r;
}
__device__ __forceinline__ int block_max_int(int v, int* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max_int(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  int r = (lane < nw) ? scratch[lane] : 0;
  return warp_max_int(r);
}

}  // namespace tq

// ---------------------------------------------------------------------------------------------
// Internal launch interface (host side), implemented by the kernel files.
// Each returns cudaSuccess or the launch error; arguments are validated by the caller.
// ---------------------------------------------------------------------------------------------
namespace tq {

struct DeviceInfo {
  int device;
  int num_sms;
};
DeviceInfo current_device_info();

cudaError_t launch_tq_pack(const void* w, bool w_f16, uint8_t* packed, uint16_t* scale, int64_t N,
                           int64_t K, cudaStream_t s);
cudaError_t launch_w4g_pack(const void* w, bool w_f16, int32_t* qweight, uint16_t* scales,
                            int64_t N, int64_t K, cudaStream_t s);
// General W4 pack: zeros != null -> asymmetric (zero-point per group); perm != null -> the groups
// are the columns perm[128 g ..] (activation order); g_idx (nullable) receives each column's group.
cudaError_t launch_w4g_pack_ex(const void* w, bool w_f16, const int32_t* perm, int32_t* qweight, uint16_t* scales,
                               uint8_t* zeros, int32_t* g_idx, int64_t N, int64_t K, cudaStream_t s);
cudaError_t launch_permute_cols(const uint16_t* x, const int32_t* perm, uint16_t* out, int64_t M, int64_t K,
                                cudaStream_t s);
cudaError_t launch_repack_act_order(const int32_t* qweight, const int32_t* perm, int32_t* out, int64_t N,
                                    int64_t K, cudaStream_t s);
cudaError_t launch_iota_groups(int32_t* g_idx, int64_t K, cudaStream_t s);
cudaError_t launch_tq_gemm_generic(const __half* x, const uint8_t* packed, const __half* scale,
                                   const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                   cudaStream_t s);
// W4A16 GEMMs: zeros == null is the symmetric format (What = s (u - 8)); otherwise
// What = s (u - zeros[n, k / 128]).
cudaError_t launch_w4g_gemm_generic(const __half* x, const int32_t* qweight, const __half* scales,
                                    const uint8_t* zeros, const __half* bias, __half* y, int64_t M, int64_t N,
                                    int64_t K, cudaStream_t s);
cudaError_t launch_tq_validate(const uint8_t* packed, int64_t N, int64_t K, int* bad,
                               cudaStream_t s);
// Decode (skinny) path: at most 16 tokens per CTA; larger M runs token chunks of 16 over grid z.
constexpr int64_t kDecodeMaxM = 64;
// Largest M the automatic dispatch sends to the decode path, per format (the measured crossover
// with the tensor-core path on Llama-3-8B and Qwen2-7B shaped linears).
constexpr int64_t kDecodeAutoMaxM_Ternary = 16;
constexpr int64_t kDecodeAutoMaxM_W4g = 16;
cudaError_t launch_tq_gemm_decode(const __half* x, const uint8_t* packed, const __half* scale,
                                  const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                  cudaStream_t s);
cudaError_t launch_tq_gemm_decode_group(const __half* x, int count, const uint8_t* const* packed,
                                        const __half* const* scale, const __half* const* bias,
                                        __half* const* y, const int64_t* N, int64_t M, int64_t K,
                                        cudaStream_t s);
cudaError_t launch_w4g_gemm_decode_group(const __half* x, int count, const int32_t* const* qweight,
                                         const __half* const* scales, const __half* const* bias,
                                         __half* const* y, const int64_t* N, int64_t M, int64_t K,
                                         cudaStream_t s);
cudaError_t launch_w4g_gemm_decode(const __half* x, const int32_t* qweight, const __half* scales,
                                   const uint8_t* zeros, const __half* bias, __half* y, int64_t M, int64_t N,
                                   int64_t K, cudaStream_t s);
cudaError_t launch_tq_gemm_prefill(const __half* x, const uint8_t* packed, const __half* scale,
                                   const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                   cudaStream_t s);
cudaError_t launch_w4g_gemm_prefill(const __half* x, const int32_t* qweight, const __half* scales,
                                    const uint8_t* zeros, const __half* bias, __half* y, int64_t M, int64_t N,
                                    int64_t K, cudaStream_t s);
// Up to four matrices that read the same x in ONE tensor-core launch (symmetric W4A16 when int4);
// every matrix must satisfy prefill_supported and the prefill path's alignment.  Worth it when
// prefill_grouping_pays (their tiles together fill at most a few waves).
bool prefill_grouping_pays(int64_t M, const int64_t* N, int count);
cudaError_t launch_gemm_prefill_grouped(bool int4, const __half* x, int count, const void* const* w,
                                        const __half* const* sc, const __half* const* bias, __half* const* y,
                                        const int64_t* N, int64_t M, int64_t K, cudaStream_t s);

// Work list of the persistent batch decode kernel (tq_batch.cu): independent linears sharing M.
struct BatchLinear {
  const __half* x;     // [M, K]
  const void* w;       // ternary uint8 [N, K/4] or W4A16 int32 [N, K/8]
  const __half* sc;    // ternary [N]; W4A16 [N, K/128]
  const __half* bias;  // [N] or null
  __half* y;           // [M, N]
  int64_t N, K;
  const uint8_t* zp;   // W4A16 zero-points [N, K/128], or null (symmetric)
};
constexpr int kBatchMaxItems = 8;
// The call that will follow a batch call on its stream, when the caller names it (its weights
// are then prefetched into L2 during this call; only w, N and K of its items are read).
struct BatchNext {
  const BatchLinear* items = nullptr;
  int count = 0;
  int64_t M = 0;
};
constexpr int64_t kBatchMaxM = 32;        // the tensor-core variant; the mma.sync variant takes M <= 16
// Workspace bytes the batch kernel needs on the current device.
int64_t batch_workspace_bytes();
cudaError_t launch_tq_gemm_batch(const BatchLinear* items, int count, int64_t M, void* ws, int64_t ws_bytes,
                                 cudaStream_t s, bool interleaved = false, const BatchNext& next = BatchNext());
// The pair-interleaved relayout of packed ternary rows (words of 16 codes, flat).
cudaError_t launch_tq_interleave(const uint32_t* in, uint32_t* out, int64_t words, cudaStream_t s);
cudaError_t launch_w4g_gemm_batch(const BatchLinear* items, int count, int64_t M, void* ws, int64_t ws_bytes,
                                  cudaStream_t s, const BatchNext& next = BatchNext());
// The tensor-core variant of the batch kernel (tq_tcbatch.cu), 1 <= M <= 32.
cudaError_t launch_gemm_batch_tc(bool int4, const BatchLinear* items, int count, int64_t M, void* ws,
                                 int64_t ws_bytes, cudaStream_t s);
int64_t tc_batch_workspace_bytes_for(int G);

// Encode a 2-D row-major tensor map (driver entry point fetched through the runtime, so the
// library does not link libcuda).  Returns false on failure.
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                  uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                  CUtensorMapSwizzle swizzle);

// 3-D variant: dims[0] innermost (elements), strides_bytes[i] = stride of dimension i + 1.
bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t dims[3],
                  const uint64_t strides_bytes[2], const uint32_t box[3], CUtensorMapSwizzle swizzle);

// Enqueue the empty kernel that separates a write of model constants from a following GEMM.
cudaError_t after_constants_written(cudaStream_t s);

// Set the dynamic shared-memory limit of `func` on the current device once.
cudaError_t ensure_smem_attr(const void* func, int bytes);

}  // namespace tq
