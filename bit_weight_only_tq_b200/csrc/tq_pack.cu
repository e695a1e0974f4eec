// tq_pack.cu -- quantise-and-pack kernels.
//
// Ternary ([TQ] §1 ternarisation, §3.1 threshold 0.7*mean|w|, code table and byte layout, §3.2
// ceil(K/4) row stride): one CTA per row.  The row sums that decide the threshold and the
// scale are computed EXACTLY (then rounded once to fp64), so the codes and the scale do not
// depend on the order in which the GPU adds:
//   * fp16 input: |w| * 2^24 is an integer below 2^40, so an int64 accumulator is exact for
//     any row length below 2^23;
//   * fp32 input: |w| is binned by its exponent relative to the row's largest exponent; inside
//     a bin of `binw` binades every value is a multiple of the bin's quantum and the bin total
//     stays below 2^53 quanta (binw = 30 - ceil(log2 K)), so fp64 additions in a bin are exact
//     in any order.  Bins 0 and 1 live in registers, deeper (rare) bins in shared memory.  The
//     bins are finally added exactly in fixed point and rounded once.
// W4A16 ([VQ] §4.2, §5: 4-bit, group 128, symmetric, 8 per int32): one warp per (row, group).
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kPackThreads = 256;
constexpr int kMaxBins = 256;

// Load the 4 elements of byte j of a row (k = 4j .. 4j+3), as raw bit patterns widened to
// uint32 (fp32 bits, or fp16 bits in the low half).  Elements past K read as 0.
template <bool kF16>
__device__ __forceinline__ void load4(const void* row, int64_t j, int64_t K, bool vec,
                                      uint32_t (&v)[4]) {
  const int64_t k0 = 4 * j;
  if (vec && k0 + 4 <= K) {
    if (kF16) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(row) + k0));
      v[0] = u.x & 0xFFFFu;
      v[1] = u.x >> 16;
      v[2] = u.y & 0xFFFFu;
      v[3] = u.y >> 16;
    } else {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const float*>(row) + k0));
      v[0] = u.x;
      v[1] = u.y;
      v[2] = u.z;
      v[3] = u.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t k = k0 + i;
      if (k < K) {
        v[i] = kF16 ? static_cast<uint32_t>(__ldg(static_cast<const uint16_t*>(row) + k))
                    : __float_as_uint(__ldg(static_cast<const float*>(row) + k));
      } else {
        v[i] = 0u;
      }
    }
  }
}

__device__ __forceinline__ double elem_to_f64(uint32_t bits, bool f16) {
  return f16 ? static_cast<double>(__half2float(__ushort_as_half(static_cast<uint16_t>(bits))))
             : static_cast<double>(__uint_as_float(bits));
}

// |w| of an fp16 pattern, as an integer multiple of 2^-24 (exact).
__device__ __forceinline__ long long f16_abs_units(uint32_t h) {
  const uint32_t e = (h >> 10) & 0x1Fu, f = h & 0x3FFu;
  return e ? (static_cast<long long>(1024u + f) << (e - 1)) : static_cast<long long>(f);
}

// Accumulator for an exact sum of |w| over part of a row.
template <bool kF16>
struct ExactAcc {
  long long i64 = 0;   // fp16: units of 2^-24
  double b0 = 0.0;     // fp32: bins 0 and 1 (the two bins below the row's top exponent)
  double b1 = 0.0;
  __device__ __forceinline__ void add(uint32_t bits, int emax, int binw, double* s_bins) {
    if (kF16) {
      i64 += f16_abs_units(bits);
    } else {
      const uint32_t a = bits & 0x7FFFFFFFu;
      if (a == 0u) return;
      const int e = max(static_cast<int>(a >> 23), 1);
      const int jb = (emax - e) / binw;
      const double v = static_cast<double>(__uint_as_float(a));
      if (jb == 0)
        b0 += v;
      else if (jb == 1)
        b1 += v;
      else
        atomicAdd(&s_bins[jb], v);
    }
  }
};

// Block-wide exact total of the per-thread accumulators, rounded once to fp64.
// Every thread must call; every thread gets the result.
template <bool kF16>
__device__ double exact_total(const ExactAcc<kF16>& acc, double* s_bins, int nbins,
                              long long* s_red_ll, double* s_red_d, double* s_result) {
  if (kF16) {
    const long long tot = block_sum<long long>(acc.i64, s_red_ll);
    return __ll2double_rn(tot) * 0x1p-24;
  } else {
    const double t0 = block_sum<double>(acc.b0, s_red_d);
    const double t1 = block_sum<double>(acc.b1, s_red_d);
    __syncthreads();  // all deep-bin atomics are done
    if (threadIdx.x == 0) {
      s_bins[0] = t0;
      s_bins[1] = t1;
      *s_result = exact_sum_fixed149(s_bins, nbins);
    }
    __syncthreads();
    return *s_result;
  }
}

template <bool kF16>
__global__ void __launch_bounds__(kPackThreads)
    tq_pack_kernel(const void* __restrict__ w, uint8_t* __restrict__ packed,
                   uint16_t* __restrict__ scale, int64_t N, int64_t K, int binw, int vec) {
  __shared__ double s_bins[kMaxBins];
  __shared__ long long s_red_ll[32];
  __shared__ double s_red_d[32];
  __shared__ int s_red_i[32];
  __shared__ double s_result;

  const int64_t KB = (K + 3) >> 2;
  const int nbins = kF16 ? 0 : min(kMaxBins, 254 / binw + 2);

  for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
    const void* row = kF16 ? static_cast<const void*>(static_cast<const uint16_t*>(w) + n * K)
                           : static_cast<const void*>(static_cast<const float*>(w) + n * K);
    // ---- pass 1 (fp32 only): largest biased exponent of the row
    int emax = 1;
    if (!kF16) {
      int m = 1;
      for (int64_t j = threadIdx.x; j < KB; j += blockDim.x) {
        uint32_t v[4];
        load4<kF16>(row, j, K, vec, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) m = max(m, static_cast<int>((v[i] & 0x7FFFFFFFu) >> 23));
      }
      emax = block_max_int(m, s_red_i);
      for (int i = threadIdx.x; i < nbins; i += blockDim.x) s_bins[i] = 0.0;
      __syncthreads();
    }
    // ---- pass 2: S = exact sum |w|;  t = 0.7 * (S / K)
    ExactAcc<kF16> accS;
#pragma unroll 4
    for (int64_t j = threadIdx.x; j < KB; j += blockDim.x) {
      uint32_t v[4];
      load4<kF16>(row, j, K, vec, v);
#pragma unroll
      for (int i = 0; i < 4; ++i) accS.add(v[i], emax, binw, s_bins);
    }
    const double S = exact_total<kF16>(accS, s_bins, nbins, s_red_ll, s_red_d, &s_result);
    const double t = 0.7 * (S / static_cast<double>(K));
    if (!kF16) {
      for (int i = threadIdx.x; i < nbins; i += blockDim.x) s_bins[i] = 0.0;
      __syncthreads();
    }
    // ---- pass 3: codes, packed bytes, A = exact sum |w| over nonzero codes, nz
    ExactAcc<kF16> accA;
    int nz = 0;
    uint8_t* prow = packed + n * KB;
#pragma unroll 2
    for (int64_t j = threadIdx.x; j < KB; j += blockDim.x) {
      uint32_t v[4];
      load4<kF16>(row, j, K, vec, v);
      uint32_t byte = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t code = 1u;  // padding past K is the zero code 0b01
        if (4 * j + i < K) {
          const double wd = elem_to_f64(v[i], kF16);
          code = (wd < -t) ? 0u : ((wd > t) ? 2u : 1u);
          if (code != 1u) {
            accA.add(v[i], emax, binw, s_bins);
            ++nz;
          }
        }
        byte |= code << (2 * i);
      }
      prow[j] = static_cast<uint8_t>(byte);
    }
    const double A = exact_total<kF16>(accA, s_bins, nbins, s_red_ll, s_red_d, &s_result);
    const int nzt = block_sum<int>(nz, s_red_i);
    if (threadIdx.x == 0) {
      scale[n] = nzt > 0 ? f64_to_f16_rne(A / static_cast<double>(nzt)) : static_cast<uint16_t>(0);
    }
    __syncthreads();  // shared scratch is reused by the next row
  }
}

// ---------------------------------------------------------------------------------------------
// W4A16 pack: one warp per (row n, group g of 128).  Lane l holds k = 128g + 4l .. 4l+3.
// ---------------------------------------------------------------------------------------------
template <bool kF16>
__global__ void __launch_bounds__(256)
    w4g_pack_kernel(const void* __restrict__ w, int32_t* __restrict__ qweight,
                    uint16_t* __restrict__ scales, int64_t N, int64_t K, int vec) {
  const int lane = threadIdx.x & 31;
  const int64_t G = K >> 7;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       item < N * G; item += warps_total) {
    const int64_t n = item / G, g = item - n * G;
    const int64_t k0 = g * 128 + 4 * lane;
    const void* row = kF16 ? static_cast<const void*>(static_cast<const uint16_t*>(w) + n * K)
                           : static_cast<const void*>(static_cast<const float*>(w) + n * K);
    uint32_t v[4];
    load4<kF16>(row, k0 >> 2, K, vec, v);
    float wf[4];
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      wf[i] = kF16 ? __half2float(__ushort_as_half(static_cast<uint16_t>(v[i]))) : __uint_as_float(v[i]);
      mx = fmaxf(mx, fabsf(wf[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    const uint16_t sb = f64_to_f16_rne(static_cast<double>(mx) / 7.0);
    const double sd = f16_bits_to_f64(sb);
    uint32_t nib = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int q = 0;
      if (sd != 0.0) {
        const double r = rint(static_cast<double>(wf[i]) / sd);
        q = static_cast<int>(fmin(fmax(r, -8.0), 7.0));
      }
      nib |= static_cast<uint32_t>(q + 8) << (4 * i);
    }
    const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, nib, 1);
    if ((lane & 1) == 0) {
      qweight[n * (K >> 3) + g * 16 + (lane >> 1)] = static_cast<int32_t>(nib | (other << 16));
    }
    if (lane == 0) scales[n * G + g] = sb;
  }
}

static int ceil_log2_i64(int64_t v) {
  int r = 0;
  while ((int64_t(1) << r) < v) ++r;
  return r;
}

cudaError_t launch_tq_pack(const void* w, bool w_f16, uint8_t* packed, uint16_t* scale, int64_t N,
                           int64_t K, cudaStream_t s) {
  const DeviceInfo di = current_device_info();
  const int64_t grid = N < int64_t(di.num_sms) * 8 ? N : int64_t(di.num_sms) * 8;
  const int binw = 30 - ceil_log2_i64(K);
  const uintptr_t a = reinterpret_cast<uintptr_t>(w);
  const int vec = (K % 4 == 0) && (a % (w_f16 ? 8 : 16) == 0);
  if (w_f16)
    tq_pack_kernel<true><<<static_cast<unsigned>(grid), kPackThreads, 0, s>>>(w, packed, scale, N,
                                                                             K, binw, vec);
  else
    tq_pack_kernel<false><<<static_cast<unsigned>(grid), kPackThreads, 0, s>>>(w, packed, scale,
                                                                              N, K, binw, vec);
  return cudaGetLastError();
}

cudaError_t launch_w4g_pack(const void* w, bool w_f16, int32_t* qweight, uint16_t* scales,
                            int64_t N, int64_t K, cudaStream_t s) {
  const DeviceInfo di = current_device_info();
  const int64_t items = N * (K >> 7);
  int64_t grid = (items + 7) / 8;
  if (grid > int64_t(di.num_sms) * 16) grid = int64_t(di.num_sms) * 16;
  const uintptr_t a = reinterpret_cast<uintptr_t>(w);
  const int vec = (a % (w_f16 ? 8 : 16) == 0);
  if (w_f16)
    w4g_pack_kernel<true><<<static_cast<unsigned>(grid), 256, 0, s>>>(w, qweight, scales, N, K, vec);
  else
    w4g_pack_kernel<false><<<static_cast<unsigned>(grid), 256, 0, s>>>(w, qweight, scales, N, K, vec);
  return cudaGetLastError();
}

}  // namespace tq
