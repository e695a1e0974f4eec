// tq_pack.cu -- quantise-and-pack kernels.
//
// Ternary ([TQ] §1 ternarisation, §3.1 threshold 0.7*mean|w|, code table and byte layout, §3.2
// ceil(K/4) row stride): one warp per row.  The row sums that decide the threshold and the
// scale are computed EXACTLY (then rounded once to fp64), so the codes and the scale do not
// depend on the order in which the GPU adds:
//   * fp16 input: |w| * 2^24 is an integer below 2^40, so an int64 accumulator is exact for
//     any row length below 2^23;
//   * fp32 input: |w| is binned by its exponent relative to the row's largest exponent; inside
//     a bin of `binw` binades every value is a multiple of the bin's quantum and the bin total
//     stays below 2^53 quanta (binw = 30 - ceil(log2 K)), so fp64 additions in a bin are exact
//     in any order.  Bins 0 and 1 live in registers, deeper (rare) bins in the warp's slice of
//     shared memory.  The bins are finally added exactly in fixed point and rounded once.
// The code decision |w| > t is an integer compare of the magnitude's bit pattern against the
// pattern of the largest representable value <= t, which equals the fp64 compare exactly.
// W4A16 ([VQ] §4.2, §5: 4-bit, group 128, symmetric, 8 per int32): one warp per (row, group).
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "tq_common.cuh"

namespace tq {

constexpr int kPackThreads = 256;

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

// Warp-wide exact total of per-lane accumulators, rounded once to fp64 (all lanes get it).
// `wbins` is this warp's shared-memory bin array (fp32 input only).
template <bool kF16>
__device__ double warp_exact_total(const ExactAcc<kF16>& acc, double* wbins, int nbins) {
  if (kF16) {
    long long v = acc.i64;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return __ll2double_rn(v) * 0x1p-24;
  } else {
    double b0 = acc.b0, b1 = acc.b1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {  // exact: every partial sum of one bin is representable
      b0 += __shfl_xor_sync(0xFFFFFFFFu, b0, o);
      b1 += __shfl_xor_sync(0xFFFFFFFFu, b1, o);
    }
    __syncwarp();  // deep-bin atomics of all lanes are done
    double r = 0.0;
    if ((threadIdx.x & 31) == 0) {
      wbins[0] = b0;
      wbins[1] = b1;
      r = exact_sum_fixed149(wbins, nbins);
    }
    return __shfl_sync(0xFFFFFFFFu, r, 0);
  }
}

// Largest magnitude bit pattern whose value is <= t (t >= 0).  Positive IEEE patterns are
// ordered like their values, so for any element |w| > t  <=>  (bits(w) & ~sign) > this.
template <bool kF16>
__device__ __forceinline__ uint32_t magnitude_floor_bits(double t) {
  if (kF16) {
    const uint16_t h = f64_to_f16_rne(t);  // nearest; step down if it rounded up
    const uint32_t m = h & 0x7FFFu;
    if (m != 0u && f16_bits_to_f64(static_cast<uint16_t>(m)) > t) return m - 1u;
    return m >= 0x7C00u ? 0x7BFFu : m;
  } else {
    const float f = __double2float_rd(t);  // round toward -inf: largest float <= t
    const uint32_t m = __float_as_uint(f) & 0x7FFFFFFFu;
    return m >= 0x7F800000u ? 0x7F7FFFFFu : m;
  }
}

// One warp per row.  Pass 1 (fp32 only): largest exponent.  Pass 2: exact sum of |w| -> t.
// Pass 3: codes (an integer compare against the threshold pattern), packed bytes, exact sum of
// the nonzero magnitudes and their count -> scale.  Rows are re-read from L2 between passes.
// fp32 rows read with 16-byte loads first take a fast path: both sums in fp64 (four accumulators
// per lane), used when their error bound decides the threshold's fp32 bucket and the fp16 scale
// (a band of about 1e-14 relative against buckets of 6e-8: practically every row); a row it does
// not decide runs the exact passes.
template <bool kF16>
__global__ void __launch_bounds__(kPackThreads)
    tq_pack_kernel(const void* __restrict__ w, uint8_t* __restrict__ packed,
                   uint16_t* __restrict__ scale, int64_t N, int64_t K, int binw, int vec) {
  constexpr int kWarps = kPackThreads / 32;
  constexpr int kWarpBins = 130;  // fp32 bins per warp: 254 / binw + 2 with binw >= 2 (K <= 2^28)
  __shared__ double s_bins[kF16 ? 1 : kWarps * kWarpBins];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  double* wbins = kF16 ? s_bins : s_bins + wid * kWarpBins;
  const int64_t KB = (K + 3) >> 2;
  const int nbins = kF16 ? 0 : min(kWarpBins, 254 / binw + 2);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;

  // terms per fp64 accumulator, and the relative bound of such sums of nonnegative terms
  // (n u / (1 - n u), u = 2^-53), widened for the fp64 steps after them
  const int64_t n_lane = (KB + 31) / 32;
  const double rel64 = 1.02 * (static_cast<double>(n_lane) * 0x1p-53 / (1.0 - static_cast<double>(n_lane) * 0x1p-53)) +
                       0x1p-48;
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * kWarps + wid; n < N; n += nwarps) {
    const void* row = kF16 ? static_cast<const void*>(static_cast<const uint16_t*>(w) + n * K)
                           : static_cast<const void*>(static_cast<const float*>(w) + n * K);
    if (!kF16 && vec) {
      double s4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
      for (int64_t j = lane; j < KB; j += 32) {
        uint32_t v[4];
        load4<kF16>(row, j, K, vec, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) s4[i] += static_cast<double>(__uint_as_float(v[i] & 0x7FFFFFFFu));
      }
      const double Sh = warp_sum((s4[0] + s4[1]) + (s4[2] + s4[3]));
      const double th = 0.7 * (Sh / static_cast<double>(K));
      const uint32_t tb = magnitude_floor_bits<false>(th * (1.0 - rel64));
      if (Sh < INFINITY && tb == magnitude_floor_bits<false>(th * (1.0 + rel64))) {
        double a4[4] = {0.0, 0.0, 0.0, 0.0};
        int nz = 0;
        uint8_t* prow = packed + n * KB;
#pragma unroll 4
        for (int64_t j = lane; j < KB; j += 32) {
          uint32_t v[4];
          load4<kF16>(row, j, K, vec, v);
          uint32_t byte = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t mag = v[i] & 0x7FFFFFFFu;
            const bool keep = mag > tb;  // |w| > t (K % 4 == 0 on this path: no padding)
            byte |= (keep ? ((v[i] & 0x80000000u) ? 0u : 2u) : 1u) << (2 * i);
            a4[i] += keep ? static_cast<double>(__uint_as_float(mag)) : 0.0;
            nz += keep ? 1 : 0;
          }
          prow[j] = static_cast<uint8_t>(byte);
        }
        const int nzt = warp_sum(nz);
        const double Ah = warp_sum((a4[0] + a4[1]) + (a4[2] + a4[3]));
        uint16_t sc = 0;
        bool done = nzt == 0;
        if (!done) {
          sc = f64_to_f16_rne(Ah * (1.0 - rel64) / static_cast<double>(nzt));
          done = Ah < INFINITY && sc == f64_to_f16_rne(Ah * (1.0 + rel64) / static_cast<double>(nzt));
        }
        if (done) {
          if (lane == 0) scale[n] = sc;
          continue;
        }
      }
    }
    int emax = 1;
    if (!kF16) {
      int m = 1;
      for (int64_t j = lane; j < KB; j += 32) {
        uint32_t v[4];
        load4<kF16>(row, j, K, vec, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) m = max(m, static_cast<int>((v[i] & 0x7FFFFFFFu) >> 23));
      }
      emax = warp_max_int(m);
      __syncwarp();  // lane 0 is done with the previous row's bins
      for (int i = lane; i < nbins; i += 32) wbins[i] = 0.0;
      __syncwarp();
    }
    ExactAcc<kF16> accS;
#pragma unroll 4
    for (int64_t j = lane; j < KB; j += 32) {
      uint32_t v[4];
      load4<kF16>(row, j, K, vec, v);
#pragma unroll
      for (int i = 0; i < 4; ++i) accS.add(v[i], emax, binw, wbins);
    }
    const double S = warp_exact_total<kF16>(accS, wbins, nbins);
    const double t = 0.7 * (S / static_cast<double>(K));
    const uint32_t tb = magnitude_floor_bits<kF16>(t);
    const uint32_t magmask = kF16 ? 0x7FFFu : 0x7FFFFFFFu;
    const uint32_t signbit = kF16 ? 0x8000u : 0x80000000u;
    if (!kF16) {
      __syncwarp();
      for (int i = lane; i < nbins; i += 32) wbins[i] = 0.0;
      __syncwarp();
    }
    ExactAcc<kF16> accA;
    int nz = 0;
    uint8_t* prow = packed + n * KB;
#pragma unroll 4
    for (int64_t j = lane; j < KB; j += 32) {
      uint32_t v[4];
      load4<kF16>(row, j, K, vec, v);
      uint32_t byte = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t code = 1u;  // padding past K is the zero code 0b01
        if (4 * j + i < K && (v[i] & magmask) > tb) {  // |w| > t
          code = (v[i] & signbit) ? 0u : 2u;
          accA.add(v[i], emax, binw, wbins);
          ++nz;
        }
        byte |= code << (2 * i);
      }
      prow[j] = static_cast<uint8_t>(byte);
    }
    const double A = warp_exact_total<kF16>(accA, wbins, nbins);
    const int nzt = warp_sum(nz);
    if (lane == 0)
      scale[n] = nzt > 0 ? f64_to_f16_rne(A / static_cast<double>(nzt)) : static_cast<uint16_t>(0);
  }
}

// ---------------------------------------------------------------------------------------------
// Ternary pack, fp16 rows with K % 8 == 0 and a 16-byte aligned base: the same semantics as
// above with 16-byte loads and cheaper exact sums.  |w| is converted to fp64 by the hardware
// (exact); a lane's fp64 partial sum stays exact while it is below 2^29 (every value is a
// multiple of 2^-24), so it is flushed every 8192 elements into integer units of 2^-24, kept as
// a high (>> 32) and a low part so that no row length overflows; the warp total is the sum of
// the two exact parts, rounded once.  The code decision is a packed 16-bit compare of the
// magnitude patterns against the threshold pattern.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ double f16_mag_f64(uint32_t h) {  // |h| for the fp16 pattern in bits 0..15
  double d;
  const unsigned short m = static_cast<unsigned short>(h & 0x7FFFu);
  asm("{\n\t.reg .f16 t;\n\tmov.b16 t, %1;\n\tcvt.f64.f16 %0, t;\n\t}" : "=d"(d) : "h"(m));
  return d;
}

struct UnitsAcc {  // exact running sum of fp16 magnitudes
  double part = 0.0;
  long long hi = 0, lo = 0;
  __device__ __forceinline__ void flush() {
    const unsigned long long u = static_cast<unsigned long long>(part * 16777216.0);  // exact
    hi += static_cast<long long>(u >> 32);
    lo += static_cast<long long>(u & 0xFFFFFFFFull);
    part = 0.0;
  }
  __device__ __forceinline__ double warp_total() {  // all lanes get the correctly rounded total
    flush();
    long long h = hi, l = lo;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      h += __shfl_xor_sync(0xFFFFFFFFu, h, o);
      l += __shfl_xor_sync(0xFFFFFFFFu, l, o);
    }
    return __ll2double_rn(h) * 256.0 + __ll2double_rn(l) * 0x1p-24;  // two exact terms, one rounding
  }
};

// Fast exact sum of fp16 magnitudes in fp32 (FMA pipe) while the values stay small: each v is
// split into h = v rounded to a multiple of 2^-12 ((v + 2048) - 2048, exact for v < 2^11) and
// l = v - h (exact, |l| <= 2^-13, a multiple of 2^-24).  The h sums are exact while below 2^12
// (multiples of 2^-12) and, h being >= 0, they only grow: a final sum below 2^11 proves every
// partial sum and every v were in range.  The l sums stay exact while fewer than 2^13 values
// are added (|partial| < 1, multiples of 2^-24).  Otherwise the caller recomputes the sum in fp64.
struct FastAcc {
  float hi = 0.0f, lo = 0.0f;
  __device__ __forceinline__ void add(float v) {
    const float h = __fadd_rn(__fadd_rn(v, 2048.0f), -2048.0f);
    hi = __fadd_rn(hi, h);
    lo = __fadd_rn(lo, __fadd_rn(v, -h));
  }
  __device__ __forceinline__ void add_pair(uint32_t mags) {  // two fp16 magnitude patterns
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&mags));
    add(f.x);
    add(f.y);
  }
  __device__ __forceinline__ bool valid() const { return hi < 2048.0f; }
  // This lane's sum in units of 2^-24 (both parts are exact integers in those units).
  __device__ __forceinline__ long long units() const {
    return __double2ll_rn(static_cast<double>(hi) * 16777216.0) + __double2ll_rn(static_cast<double>(lo) * 16777216.0);
  }
};

// Warp total of per-lane unit sums, correctly rounded once to fp64 (all lanes get it).
__device__ __forceinline__ double warp_units_total(long long u) {
  long long h = u >> 32, l = u & 0xFFFFFFFFll;  // two parts, so no row length overflows
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    h += __shfl_xor_sync(0xFFFFFFFFu, h, o);
    l += __shfl_xor_sync(0xFFFFFFFFu, l, o);
  }
  return __ll2double_rn(h) * 256.0 + __ll2double_rn(l) * 0x1p-24;
}

// Relative error bound of a row sum made of fp32 accumulators that each add at most n
// nonnegative terms in order, starting from zero (at most gamma(n) = n u / (1 - n u), u = 2^-24),
// then combined in fp64; the factor and the 2^-45 cover the fp64 roundings of the sum, of the
// value derived from it and of the bounds computed from that value.
__device__ __forceinline__ double fp32_sum_rel_bound(int64_t n) {
  const double nu = static_cast<double>(n) * 0x1p-24;
  return 1.02 * (nu / (1.0 - nu)) + 0x1p-45;
}

// kFast: both row sums are plain fp32 sums (eight accumulators per lane) whose error bound
// decides whether they can be used: the threshold's fp16 bucket and the fp16 scale are taken
// from them only when every value within the bound gives the same bucket / the same fp16 (both
// maps are monotone), which then equals the result from the exact sums; otherwise the row's sum
// is recomputed exactly (FastAcc, fp32 on the FMA pipe, with an fp64 recomputation when its
// values leave its range).  Rows need fewer than 2^13 elements per lane (K < 2^18).
// One warp packs one row: ld(j) returns its 16-byte chunk j (8 elements), prow receives the
// packed bytes; returns the row's fp16 scale (every lane).
template <bool kFast, typename Ld>
__device__ __forceinline__ uint16_t pack_f16_row(Ld ld, uint16_t* prow, int64_t C, int64_t K, double rel, int lane) {
  // exact sum of |w| over the row, fp64 (the fallback, and the path without kFast)
  auto slow_sum = [&]() {
    UnitsAcc acc;
    int cnt = 0;
#pragma unroll 2
    for (int64_t j = lane; j < C; j += 32) {
      const uint4 v = ld(j);
      acc.part += ((f16_mag_f64(v.x) + f16_mag_f64(v.x >> 16)) + (f16_mag_f64(v.y) + f16_mag_f64(v.y >> 16))) +
                  ((f16_mag_f64(v.z) + f16_mag_f64(v.z >> 16)) + (f16_mag_f64(v.w) + f16_mag_f64(v.w >> 16)));
      if (++cnt == 1024) {  // 8192 elements < 2^13: the partial stays below 2^29
        acc.flush();
        cnt = 0;
      }
    }
    return acc.warp_total();
  };
  auto exact_sum = [&]() {
    if (!kFast) return slow_sum();
    FastAcc fa;
#pragma unroll 2
    for (int64_t j = lane; j < C; j += 32) {
      const uint4 v = ld(j);
      fa.add_pair(v.x & 0x7FFF7FFFu);
      fa.add_pair(v.y & 0x7FFF7FFFu);
      fa.add_pair(v.z & 0x7FFF7FFFu);
      fa.add_pair(v.w & 0x7FFF7FFFu);
    }
    return __all_sync(0xFFFFFFFFu, fa.valid()) ? warp_units_total(fa.units()) : slow_sum();
  };
  uint32_t tb;
  bool Sh_finite = false;
  if (kFast) {
    float sa[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 2
    for (int64_t j = lane; j < C; j += 32) {
      const uint4 v = ld(j);
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t m = wd[i] & 0x7FFF7FFFu;
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&m));
        sa[2 * i] += f.x;
        sa[2 * i + 1] += f.y;
      }
    }
    const double Sh = warp_sum(((static_cast<double>(sa[0]) + sa[1]) + (static_cast<double>(sa[2]) + sa[3])) +
                                   ((static_cast<double>(sa[4]) + sa[5]) + (static_cast<double>(sa[6]) + sa[7])));
    const double th = 0.7 * (Sh / static_cast<double>(K));
    const uint32_t lo = magnitude_floor_bits<true>(th * (1.0 - rel));
    const uint32_t hi = magnitude_floor_bits<true>(th * (1.0 + rel));
    Sh_finite = Sh < INFINITY;
    if (Sh_finite && lo == hi) {
      tb = lo;
    } else {
      const double S = exact_sum();
      tb = magnitude_floor_bits<true>(0.7 * (S / static_cast<double>(K)));
    }
  } else {
    const double S = slow_sum();
    tb = magnitude_floor_bits<true>(0.7 * (S / static_cast<double>(K)));
  }
  const uint32_t tb2 = (tb | (tb << 16)) | 0x80008000u;
  // exact sum of the nonzero magnitudes, fp64
  auto slow_nonzero_sum = [&]() {
    UnitsAcc acc;
    int cnt = 0;
    for (int64_t j = lane; j < C; j += 32) {
      const uint4 v = ld(j);
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
      double a2 = 0.0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t D = tb2 - (wd[i] & 0x7FFF7FFFu);
        if (!(D & 0x8000u)) a2 += f16_mag_f64(wd[i]);
        if (!(D & 0x80000000u)) a2 += f16_mag_f64(wd[i] >> 16);
      }
      acc.part += a2;
      if (++cnt == 1024) {
        acc.flush();
        cnt = 0;
      }
    }
    return acc.warp_total();
  };
  // the fp32 sum of the nonzero magnitudes needs a finite row (the fp16 compare below then agrees
  // with the integer one); otherwise the exact path sums them
  const bool fin = kFast && Sh_finite;
  const uint32_t tbh2 = tb | (tb << 16);  // the threshold's fp16 pattern, both halves
  float sa[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  int zeros = 0;  // fewer than 2^18 elements per lane
  int elems = 0;
#pragma unroll 2
  for (int64_t j = lane; j < C; j += 32) {
    const uint4 v = ld(j);
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
    uint32_t dz[4], np[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // per 16-bit half: bit 15 of D is set iff |h| <= t (0x8000 + tb - |h| never borrows
      // across halves): code 01; bit 15 of ~(D | h) is set iff |h| > t and h >= 0: code 10
      const uint32_t m = wd[i] & 0x7FFF7FFFu;
      dz[i] = tb2 - m;
      np[i] = ~(dz[i] | wd[i]);
      if (fin) {  // the magnitudes of the nonzero codes (m > t as fp16; a zero code's half is 0)
        const __half2 mh = *reinterpret_cast<const __half2*>(&m);
        const __half2 keep = __hmul2(mh, __hgt2(mh, *reinterpret_cast<const __half2*>(&tbh2)));
        const float2 f = __half22float2(keep);
        sa[2 * i] += f.x;
        sa[2 * i + 1] += f.y;
      }
    }
    // bytes 1 and 3 of each word carry its two elements' flags in bit 7: one byte permute puts
    // the flags of elements 4q .. 4q + 3 in bit 7 of bytes 0 .. 3; a multiply by
    // 2^24 + 2^18 + 2^12 + 2^6 moves the flag of byte e (bit 8e) to bit 24 + 2e (2G: 25 + 2e),
    // and its other partial products fall on distinct bits below 24 (no carries)
    constexpr uint32_t G = 0x01041040u;
    const uint32_t z0 = (__byte_perm(dz[0], dz[1], 0x7531) >> 7) & 0x01010101u;
    const uint32_t z1 = (__byte_perm(dz[2], dz[3], 0x7531) >> 7) & 0x01010101u;
    const uint32_t p0 = (__byte_perm(np[0], np[1], 0x7531) >> 7) & 0x01010101u;
    const uint32_t p1 = (__byte_perm(np[2], np[3], 0x7531) >> 7) & 0x01010101u;
    const uint32_t lo = z0 * G + p0 * (2u * G), hi = z1 * G + p1 * (2u * G);
    const uint32_t out = (lo >> 24) | ((hi >> 24) << 8);  // element e: code at bits 2e, 2e + 1
    zeros += __popc(out & 0x5555u);                        // code 01
    elems += 8;
    prow[j] = static_cast<uint16_t>(out);
  }
  const int64_t nzt = warp_sum(static_cast<int64_t>(elems - zeros));
  uint16_t sc = 0;
  if (nzt > 0) {
    bool done = false;
    if (fin) {
      const double Ah = warp_sum(((static_cast<double>(sa[0]) + sa[1]) + (static_cast<double>(sa[2]) + sa[3])) +
                                     ((static_cast<double>(sa[4]) + sa[5]) + (static_cast<double>(sa[6]) + sa[7])));
      const uint16_t lo = f64_to_f16_rne(Ah * (1.0 - rel) / static_cast<double>(nzt));
      const uint16_t hi = f64_to_f16_rne(Ah * (1.0 + rel) / static_cast<double>(nzt));
      if (Ah < INFINITY && lo == hi) {
        sc = lo;
        done = true;
      }
    }
    if (!done) sc = f64_to_f16_rne(slow_nonzero_sum() / static_cast<double>(nzt));
  }
  return sc;
}

template <bool kFast>
__global__ void __launch_bounds__(kPackThreads)
    tq_pack_f16_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ packed,
                       uint16_t* __restrict__ scale, int64_t N, int64_t K) {
  constexpr int kWarps = kPackThreads / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t C = K >> 3;  // 16-byte chunks (8 elements) per row
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  const double rel = fp32_sum_rel_bound((C + 31) / 32);  // terms per fp32 accumulator, at most
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * kWarps + wid; n < N; n += nwarps) {
    const uint4* row = reinterpret_cast<const uint4*>(w + n * K);
    const uint16_t sc = pack_f16_row<kFast>([&](int64_t j) { return __ldg(row + j); },
                                            reinterpret_cast<uint16_t*>(packed + n * (K >> 2)), C, K, rel, lane);
    if (lane == 0) scale[n] = sc;
  }
}

// Rows that fit in shared memory: each warp of the CTA brings its row in with one bulk copy
// (global -> shared, completion counted on the warp's mbarrier) and every pass reads it from
// there, so each element crosses HBM once and the warps hold whole rows in flight.
__global__ void __launch_bounds__(kPackThreads)
    tq_pack_f16_smem_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ packed,
                            uint16_t* __restrict__ scale, int64_t N, int64_t K) {
  extern __shared__ __align__(16) uint8_t pk_smem[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, W = static_cast<int>(blockDim.x >> 5);
  const int64_t C = K >> 3;
  const uint4* buf = reinterpret_cast<const uint4*>(pk_smem) + wid * C;
  uint64_t* bar = reinterpret_cast<uint64_t*>(pk_smem + static_cast<int64_t>(W) * C * 16) + wid;
  if (lane == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const double rel = fp32_sum_rel_bound((C + 31) / 32);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * W;
  uint32_t phase = 0;
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * W + wid; n < N; n += nwarps, phase ^= 1u) {
    if (lane == 0) {
      fence_proxy_async_smem();  // the warp's reads of the previous row before the copy's writes
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>(K * 2));
      bulk_load_1d(const_cast<uint4*>(buf), w + n * K, static_cast<uint32_t>(K * 2), bar);
    }
    if (!mbar_wait(bar, phase)) {  // timeout (recorded): give the copy one more bounded wait
      mbar_wait(bar, phase);
      return;
    }
    const uint16_t sc = pack_f16_row<true>([&](int64_t j) { return buf[j]; },
                                           reinterpret_cast<uint16_t*>(packed + n * (K >> 2)), C, K, rel, lane);
    if (lane == 0) scale[n] = sc;
    __syncwarp();
  }
}

// Long rows (more than fit four per 55 KB): the kPackThreads threads of a CTA pack one row
// together, double-buffered in shared memory (the next row's bulk copy runs under this row's
// work).  Thread t takes the 16-byte chunks t, t + kPackThreads, ...; the row sums are reduced
// over the CTA in a fixed order, and the exact fallbacks reduce integer parts (exact).
struct PackCtaRed {
  double d[kPackThreads / 32];
  long long h[kPackThreads / 32], l[kPackThreads / 32];
};

// every thread of the block calls these; every thread gets the result
__device__ __forceinline__ double cta_sum_f64(double v, PackCtaRed* red) {
  v = warp_sum(v);
  __syncthreads();  // the previous reduction's reads are done
  if ((threadIdx.x & 31) == 0) red->d[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int i = 0; i < kPackThreads / 32; ++i) t += red->d[i];
  return t;
}

// Exact total of per-thread parts h (units of 2^8) and l (units of 2^-24), correctly rounded once.
__device__ __forceinline__ double cta_units_total(long long h, long long l, PackCtaRed* red) {
  h = warp_sum(h);
  l = warp_sum(l);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) {
    red->h[threadIdx.x >> 5] = h;
    red->l[threadIdx.x >> 5] = l;
  }
  __syncthreads();
  long long H = 0, L = 0;
#pragma unroll
  for (int i = 0; i < kPackThreads / 32; ++i) {
    H += red->h[i];
    L += red->l[i];
  }
  return __ll2double_rn(H) * 256.0 + __ll2double_rn(L) * 0x1p-24;  // two exact terms, one rounding
}

__global__ void __launch_bounds__(kPackThreads)
    tq_pack_f16_row_cta_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ packed,
                               uint16_t* __restrict__ scale, int64_t N, int64_t K) {
  extern __shared__ __align__(16) uint8_t pk_smem[];
  const int tid = threadIdx.x;
  const int64_t C = K >> 3;
  const uint4* bufs = reinterpret_cast<const uint4*>(pk_smem);  // [2][C]
  uint64_t* bar = reinterpret_cast<uint64_t*>(pk_smem + 2 * C * 16);
  PackCtaRed* red = reinterpret_cast<PackCtaRed*>(bar + 2);
  const uint32_t bytes = static_cast<uint32_t>(K * 2);
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int64_t row, int b) {
    mbar_arrive_expect_tx(&bar[b], bytes);
    bulk_load_1d(const_cast<uint4*>(bufs + b * C), w + row * K, bytes, &bar[b]);
  };
  const int64_t G = gridDim.x;
  int64_t n = blockIdx.x;
  if (tid == 0 && n < N) issue(n, 0);
  const int64_t n_thr = (C + kPackThreads - 1) / kPackThreads;  // terms per fp32 accumulator
  const double rel = fp32_sum_rel_bound(n_thr);
  for (int it = 0; n < N; n += G, ++it) {
    const int b = it & 1;
    if (tid == 0) {
      if (n + G < N) {
        fence_proxy_async_smem();  // buffer b ^ 1 was last read two rows ago (a barrier since)
        issue(n + G, b ^ 1);
      }
    }
    // a wait that runs out (recorded) ends the CTA, the same way in every thread, after a bounded
    // wait for the copy issued into the other buffer
    if (!__syncthreads_and(mbar_wait(&bar[b], static_cast<uint32_t>(it >> 1) & 1u))) {
      if (n + G < N) mbar_wait(&bar[b ^ 1], static_cast<uint32_t>((it + 1) >> 1) & 1u);
      return;
    }
    const uint4* buf = bufs + b * C;
    // ---- threshold: fp32 sums when their bound decides the fp16 bucket, else exact
    float sa[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    for (int64_t j = tid; j < C; j += kPackThreads) {
      const uint4 v = buf[j];
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t m = wd[i] & 0x7FFF7FFFu;
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&m));
        sa[2 * i] += f.x;
        sa[2 * i + 1] += f.y;
      }
    }
    const double Sh = cta_sum_f64(((static_cast<double>(sa[0]) + sa[1]) + (static_cast<double>(sa[2]) + sa[3])) +
                                      ((static_cast<double>(sa[4]) + sa[5]) + (static_cast<double>(sa[6]) + sa[7])),
                                  red);
    const bool fin = Sh < INFINITY;
    const double th = 0.7 * (Sh / static_cast<double>(K));
    uint32_t tb = magnitude_floor_bits<true>(th * (1.0 - rel));
    if (!fin || tb != magnitude_floor_bits<true>(th * (1.0 + rel))) {
      FastAcc fa;
      for (int64_t j = tid; j < C; j += kPackThreads) {
        const uint4 v = buf[j];
        fa.add_pair(v.x & 0x7FFF7FFFu);
        fa.add_pair(v.y & 0x7FFF7FFFu);
        fa.add_pair(v.z & 0x7FFF7FFFu);
        fa.add_pair(v.w & 0x7FFF7FFFu);
      }
      double S;
      if (__syncthreads_and(fa.valid())) {
        const long long u = fa.units();
        S = cta_units_total(u >> 32, u & 0xFFFFFFFFll, red);
      } else {
        UnitsAcc acc;
        int cnt = 0;
        for (int64_t j = tid; j < C; j += kPackThreads) {
          const uint4 v = buf[j];
          acc.part += ((f16_mag_f64(v.x) + f16_mag_f64(v.x >> 16)) + (f16_mag_f64(v.y) + f16_mag_f64(v.y >> 16))) +
                      ((f16_mag_f64(v.z) + f16_mag_f64(v.z >> 16)) + (f16_mag_f64(v.w) + f16_mag_f64(v.w >> 16)));
          if (++cnt == 1024) {
            acc.flush();
            cnt = 0;
          }
        }
        acc.flush();
        S = cta_units_total(acc.hi, acc.lo, red);
      }
      tb = magnitude_floor_bits<true>(0.7 * (S / static_cast<double>(K)));
    }
    const uint32_t tb2 = (tb | (tb << 16)) | 0x80008000u;
    const uint32_t tbh2 = tb | (tb << 16);
    // ---- codes, zero count, fp32 sum of the nonzero magnitudes
    uint16_t* prow = reinterpret_cast<uint16_t*>(packed + n * (K >> 2));
    float sb[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    int zeros = 0, elems = 0;
    for (int64_t j = tid; j < C; j += kPackThreads) {
      const uint4 v = buf[j];
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
      uint32_t dz[4], np[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t m = wd[i] & 0x7FFF7FFFu;
        dz[i] = tb2 - m;
        np[i] = ~(dz[i] | wd[i]);
        if (fin) {
          const __half2 mh = *reinterpret_cast<const __half2*>(&m);
          const __half2 keep = __hmul2(mh, __hgt2(mh, *reinterpret_cast<const __half2*>(&tbh2)));
          const float2 f = __half22float2(keep);
          sb[2 * i] += f.x;
          sb[2 * i + 1] += f.y;
        }
      }
      constexpr uint32_t Gm = 0x01041040u;  // the flag gather of pack_f16_row
      const uint32_t z0 = (__byte_perm(dz[0], dz[1], 0x7531) >> 7) & 0x01010101u;
      const uint32_t z1 = (__byte_perm(dz[2], dz[3], 0x7531) >> 7) & 0x01010101u;
      const uint32_t p0 = (__byte_perm(np[0], np[1], 0x7531) >> 7) & 0x01010101u;
      const uint32_t p1 = (__byte_perm(np[2], np[3], 0x7531) >> 7) & 0x01010101u;
      const uint32_t lo = z0 * Gm + p0 * (2u * Gm), hi = z1 * Gm + p1 * (2u * Gm);
      const uint32_t out = (lo >> 24) | ((hi >> 24) << 8);
      zeros += __popc(out & 0x5555u);
      elems += 8;
      prow[j] = static_cast<uint16_t>(out);
    }
    const int64_t nzt = static_cast<int64_t>(
        cta_sum_f64(static_cast<double>(elems - zeros), red));  // integers below 2^31: exact in fp64
    uint16_t sc = 0;
    if (nzt > 0) {
      const double Ah = cta_sum_f64(((static_cast<double>(sb[0]) + sb[1]) + (static_cast<double>(sb[2]) + sb[3])) +
                                        ((static_cast<double>(sb[4]) + sb[5]) + (static_cast<double>(sb[6]) + sb[7])),
                                    red);
      const uint16_t slo = f64_to_f16_rne(Ah * (1.0 - rel) / static_cast<double>(nzt));
      if (fin && Ah < INFINITY && slo == f64_to_f16_rne(Ah * (1.0 + rel) / static_cast<double>(nzt))) {
        sc = slo;
      } else {
        UnitsAcc acc;
        int cnt = 0;
        for (int64_t j = tid; j < C; j += kPackThreads) {
          const uint4 v = buf[j];
          const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
          double a2 = 0.0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t D = tb2 - (wd[i] & 0x7FFF7FFFu);
            if (!(D & 0x8000u)) a2 += f16_mag_f64(wd[i]);
            if (!(D & 0x80000000u)) a2 += f16_mag_f64(wd[i] >> 16);
          }
          acc.part += a2;
          if (++cnt == 1024) {
            acc.flush();
            cnt = 0;
          }
        }
        acc.flush();
        sc = f64_to_f16_rne(cta_units_total(acc.hi, acc.lo, red) / static_cast<double>(nzt));
      }
    }
    if (tid == 0) scale[n] = sc;
    __syncthreads();  // every thread is done with buffer b before it is refilled
  }
}

// ---------------------------------------------------------------------------------------------
// Pair-interleaved relayout (the post-load repack of [VQ] §4.3, applied to the ternary rows).
// A 32-bit little-endian word holds 16 codes, code slot s at bits 2s..2s+1 (canonical: k = s).
// The interleaved word holds the even slots (k = 0, 2, .., 14) in order in its low 16 bits and
// the odd slots (k = 1, 3, .., 15) in its high 16 bits, so a decode that reads bit position 2p
// of both halves gets k = 2p and 2p + 1.  Each 2-bit field is gathered by a three-step compaction.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t compact_even_fields(uint32_t v) {  // fields at bits 4i..4i+1 -> 2i..2i+1
  v &= 0x33333333u;
  v = (v | (v >> 2)) & 0x0F0F0F0Fu;
  v = (v | (v >> 4)) & 0x00FF00FFu;
  v = (v | (v >> 8)) & 0x0000FFFFu;
  return v;
}

__global__ void __launch_bounds__(256) tq_interleave_kernel(const uint32_t* in, uint32_t* out,  // may be the same buffer
                                                          int64_t words) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words; i += stride) {
    const uint32_t w = in[i];
    out[i] = compact_even_fields(w) | (compact_even_fields(w >> 2) << 16);
  }
}

cudaError_t launch_tq_interleave(const uint32_t* in, uint32_t* out, int64_t words, cudaStream_t s) {
  if (words <= 0) return cudaSuccess;
  const int sms = current_device_info().num_sms;
  int64_t blocks = (words + 255) / 256;
  if (blocks > 8 * static_cast<int64_t>(sms)) blocks = 8 * static_cast<int64_t>(sms);
  tq_interleave_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(in, out, words);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// W4A16 pack.  A warp quantises whole groups of 128; lane l holds weights 4l .. 4l+3 of a group.
// ---------------------------------------------------------------------------------------------
// The group quantiser of the activation-order kernel: this lane's four weights wf of one
// 128-wide group (the warp holds the group).  The contiguous-group kernel below computes the same
// codes, scales and zeros, sixteen groups per warp at a time.  Symmetric ([VQ] §5 "sym": true): s = fp16(max|w|/7),
// q = clamp(rint(w / s), -8, 7), stored u = q + 8.  Asymmetric (zeros requested, the weight_zp of
// the same section): lo = min(0, min w), hi = max(0, max w), s = fp16((hi - lo) / 15),
// z = clamp(rint(-lo / s), 0, 15), stored u = clamp(rint(w / s) + z, 0, 15).  All quotients in
// fp64 with the STORED fp16 s; s == 0 gives u = 0 (asymmetric, z = 0) or u = 8 (symmetric).
__device__ __forceinline__ void w4_quantize_group(const float (&wf)[4], bool asym, uint16_t& sb, int& z,
                                                  int (&u)[4]) {
  float a = 0.0f, b = 0.0f;  // symmetric: a = max|w|; asymmetric: a = min(0, w), b = max(0, w)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (asym) {
      a = fminf(a, wf[i]);
      b = fmaxf(b, wf[i]);
    } else {
      a = fmaxf(a, fabsf(wf[i]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    if (asym) {
      a = fminf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      b = fmaxf(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
    } else {
      a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    }
  }
  sb = asym ? f64_to_f16_rne((static_cast<double>(b) - static_cast<double>(a)) / 15.0)
            : f64_to_f16_rne(static_cast<double>(a) / 7.0);
  const double sd = f16_bits_to_f64(sb);
  // rint(v / s) in fp32 with the same result as the fp64 quotient: r = v * (1 / s) is within a
  // few fp32 ulps of q = v / s, so floor(r) + 1/2 is the half-integer h next to q (r is clamped
  // to +-64 first: every q beyond that saturates the code alike); whether q lies below, at or
  // above h is the sign of h s - v, which one fused multiply-add gives exactly (h s is exact, and
  // h s - v is a multiple of 2^-149, so it never rounds to zero unless it is zero: this needs
  // fp32 subnormals, i.e. no flush-to-zero); at q == h the even neighbour wins, as rint's does.
  // An infinite s or a non-finite v takes the fp64 quotient (clamped alike; a NaN quotient gives
  // the lowest code, as the clamps of the fp64 form do).  The result lies in [-64, 65].
  const float sf = static_cast<float>(sd);
  const bool fin_s = sd != 0.0 && sd < INFINITY;
  const float inv = fin_s ? 1.0f / sf : 0.0f;
  auto q_of = [&](float v) -> int {
    if (!fin_s || !(fabsf(v) < INFINITY))
      return static_cast<int>(fmin(fmax(rint(static_cast<double>(v) / sd), -64.0), 65.0));
    const int fl = static_cast<int>(floorf(fminf(fmaxf(__fmul_rn(v, inv), -64.0f), 64.0f)));
    const float d = __fmaf_rn(static_cast<float>(fl) + 0.5f, sf, -v);
    return d < 0.0f ? fl + 1 : d > 0.0f ? fl : fl + (fl & 1);
  };
  z = asym ? 0 : 8;
  if (asym && sd != 0.0) z = min(max(q_of(-a), 0), 15);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (sd == 0.0) {
      u[i] = asym ? 0 : 8;
    } else {
      const int r = q_of(wf[i]);
      u[i] = asym ? min(max(r + z, 0), 15) : min(max(r, -8), 7) + 8;
    }
  }
}

// Contiguous groups.  Item i = n G + g (row n, group g of 128 columns; K = 128 G) is the 128
// weights at element 128 i of the row-major W, and its outputs are qweight words 16 i .. 16 i + 15,
// scale i and zero i, so W is walked as one flat run of items.  A warp takes kB = 16 consecutive
// items per pass; lane l holds weights 4 l .. 4 l + 3 of each, all sixteen loads issued first.
// The group statistics (max |w|, or min and max) are reduced across the warp for all sixteen
// items at once by recursive halving (each exchange step halves the items a lane still holds, so
// lane l ends with item l mod 16 after 16 shuffles instead of 80), the lane then derives that
// item's scale (and zero) in fp64 as the group quantiser above does, and the quantiser of each
// item reads them back from lane j with one shuffle per item.
//
// Codes in fp32, equal to rint(v / s) of the fp64 quotient: r = v * (1 / s) is within a few fp32
// ulps of q = v / s, so h = floor(r) + 1/2 is a half-integer within one of q; q > h, q = h or
// q < h is the sign of d = h s - v, which one fused multiply-add gives exactly (h s is exact, h s
// - v is a multiple of 2^-149 and so rounds to zero only when it is zero: this needs fp32
// subnormals, i.e. no flush-to-zero), so the code is h + 1/2, h (a tie) or h - 1/2; adding
// 1.5 * 2^23 rounds a tie to even, as rint does, and leaves the code in the low mantissa bits.
// Overflowing or non-finite quotients (huge v, v = +-inf or NaN, s = inf) end at the same clamped
// codes as the fp64 form; s = 0 gives code 8 (symmetric) or 0 (asymmetric), as there.
constexpr int kW4PackItems = 16;

template <bool kF16, bool kAsym>
__global__ void __launch_bounds__(256)
    w4g_pack_kernel(const void* __restrict__ w, int32_t* __restrict__ qweight, uint16_t* __restrict__ scales,
                    uint8_t* __restrict__ zeros, int64_t items, int vec) {
  constexpr int kB = kW4PackItems;
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: integers in the low mantissa bits
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kB;
       base < items; base += warps_total * kB) {
    const int nb = items - base < kB ? static_cast<int>(items - base) : kB;  // the same for the whole warp
    const void* grp0 = kF16 ? static_cast<const void*>(static_cast<const uint16_t*>(w) + base * 128)
                            : static_cast<const void*>(static_cast<const float*>(w) + base * 128);
    // fp32: four values per lane and item; fp16: two half pairs
    constexpr int kWords = kF16 ? 2 : 4;
    uint32_t v[kB][kWords];
#pragma unroll
    for (int j = 0; j < kB; ++j) {
#pragma unroll
      for (int i = 0; i < kWords; ++i) v[j][i] = 0u;
      if (j >= nb) continue;
      if (kF16) {
        const uint16_t* p = static_cast<const uint16_t*>(grp0) + j * 128 + 4 * lane;
        if (vec) {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
          v[j][0] = u.x;
          v[j][1] = u.y;
        } else {
          v[j][0] = static_cast<uint32_t>(__ldg(p)) | (static_cast<uint32_t>(__ldg(p + 1)) << 16);
          v[j][1] = static_cast<uint32_t>(__ldg(p + 2)) | (static_cast<uint32_t>(__ldg(p + 3)) << 16);
        }
      } else {
        const float* p = static_cast<const float*>(grp0) + j * 128 + 4 * lane;
        if (vec) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
          v[j][0] = u.x;
          v[j][1] = u.y;
          v[j][2] = u.z;
          v[j][3] = u.w;
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) v[j][i] = __float_as_uint(__ldg(p + i));
        }
      }
    }
    auto vals = [&](int j, float (&f)[4]) {
      if (kF16) {
        const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&v[j][0]));
        const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&v[j][1]));
        f[0] = f01.x;
        f[1] = f01.y;
        f[2] = f23.x;
        f[3] = f23.y;
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __uint_as_float(v[j][i]);
      }
    };
    // this lane's statistics of every item: symmetric a = max|w|; asymmetric a = min(0, w),
    // b = max(0, w) (fp16: taken on the half pairs, exact; a NaN loses to any number, as in fminf)
    float a[kB], b[kB];
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      if (kF16) {
        const __half2 h0 = *reinterpret_cast<const __half2*>(&v[j][0]);
        const __half2 h1 = *reinterpret_cast<const __half2*>(&v[j][1]);
        if (kAsym) {
          const __half2 lo = __hmin2(h0, h1), hi = __hmax2(h0, h1);
          a[j] = fminf(fminf(0.0f, __low2float(lo)), __high2float(lo));
          b[j] = fmaxf(fmaxf(0.0f, __low2float(hi)), __high2float(hi));
        } else {
          const __half2 m = __hmax2(__habs2(h0), __habs2(h1));
          a[j] = fmaxf(fmaxf(0.0f, __low2float(m)), __high2float(m));
          b[j] = 0.0f;
        }
      } else {
        a[j] = 0.0f;
        b[j] = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (kAsym) {
            a[j] = fminf(a[j], __uint_as_float(v[j][i]));
            b[j] = fmaxf(b[j], __uint_as_float(v[j][i]));
          } else {
            a[j] = fmaxf(a[j], fabsf(__uint_as_float(v[j][i])));
          }
        }
      }
    }
    // recursive halving: after the step over lane bit k, a lane keeps the upper half of the items
    // it held when that bit is set and the lower half otherwise, combined with its partner's copy
#pragma unroll
    for (int k = kB / 2; k >= 1; k >>= 1) {
      const bool up = (lane & k) != 0;
#pragma unroll
      for (int i = 0; i < k; ++i) {
        const float ra = __shfl_xor_sync(0xFFFFFFFFu, up ? a[i] : a[i + k], k);
        a[i] = kAsym ? fminf(up ? a[i + k] : a[i], ra) : fmaxf(up ? a[i + k] : a[i], ra);
        if (kAsym) {
          const float rb = __shfl_xor_sync(0xFFFFFFFFu, up ? b[i] : b[i + k], k);
          b[i] = fmaxf(up ? b[i + k] : b[i], rb);
        }
      }
    }
    a[0] = kAsym ? fminf(a[0], __shfl_xor_sync(0xFFFFFFFFu, a[0], 16))
                 : fmaxf(a[0], __shfl_xor_sync(0xFFFFFFFFu, a[0], 16));
    if (kAsym) b[0] = fmaxf(b[0], __shfl_xor_sync(0xFFFFFFFFu, b[0], 16));
    // item lane mod 16: its scale, 1 / scale and zero point
    const uint16_t sb = kAsym ? f64_to_f16_rne((static_cast<double>(b[0]) - static_cast<double>(a[0])) / 15.0)
                              : f64_to_f16_rne(static_cast<double>(a[0]) / 7.0);
    const float sf = __half2float(__ushort_as_half(sb));
    const float inv = 1.0f / sf;  // +inf for s = 0 (then unused), 0 for s = inf
    auto round_q = [&](float x, float s, float rs) -> float {  // rint(x / s), exact (see above)
      const float h = floorf(__fmul_rn(x, rs)) + 0.5f;
      const float d = __fmaf_rn(h, s, -x);
      return d < 0.0f ? h + 0.5f : d > 0.0f ? h - 0.5f : h;
    };
    int z = kAsym ? 0 : 8;
    if (kAsym && sf != 0.0f) {
      const float n = (round_q(-a[0], sf, inv) + kMagic) - kMagic;  // ties to even; NaN stays NaN
      z = static_cast<int>(fminf(fmaxf(n, 0.0f), 15.0f));
    }
    if (lane < nb) {
      scales[base + lane] = sb;
      if (kAsym) zeros[base + lane] = static_cast<uint8_t>(z);
    }
    const uint32_t sz = static_cast<uint32_t>(sb) | (static_cast<uint32_t>(z) << 16);
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      if (j >= nb) break;
      const uint32_t szj = __shfl_sync(0xFFFFFFFFu, sz, j);
      const float invj = __shfl_sync(0xFFFFFFFFu, inv, j);
      const float sj = __half2float(__ushort_as_half(static_cast<uint16_t>(szj & 0xFFFFu)));
      const float zj = static_cast<float>(szj >> 16);
      float f[4];
      vals(j, f);
      uint32_t nib = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float y = round_q(f[i], sj, invj);
        float t;
        if (kAsym) {
          const float n = (y + kMagic) - kMagic;
          t = fminf(fmaxf(n + zj, 0.0f), 15.0f) + kMagic;
        } else {
          t = fminf(fmaxf(y, -8.0f), 7.0f) + (kMagic + 8.0f);
        }
        nib |= (__float_as_uint(t) & 15u) << (4 * i);
      }
      if (sj == 0.0f) nib = kAsym ? 0u : 0x8888u;
      const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, nib, 1);
      if ((lane & 1) == 0) qweight[(base + j) * 16 + (lane >> 1)] = static_cast<int32_t>(nib | (other << 16));
    }
  }
}

// Activation order: one warp per (row, group), the group being the columns perm[128 g .. +127];
// the nibbles go to the columns' ORIGINAL positions (OR into a zeroed qweight, since one word
// gathers columns of several groups).  The warps of row 0 also write g_idx[perm[j]] = j / 128.
template <bool kF16>
__global__ void __launch_bounds__(256)
    w4g_pack_perm_kernel(const void* __restrict__ w, const int32_t* __restrict__ perm, int32_t* __restrict__ qweight,
                         uint16_t* __restrict__ scales, uint8_t* __restrict__ zeros, int32_t* __restrict__ g_idx,
                         int64_t N, int64_t K) {
  const int lane = threadIdx.x & 31;
  const int64_t G = K >> 7;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t item = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       item < N * G; item += warps_total) {
    const int64_t n = item / G, g = item - n * G;
    int64_t col[4];
    float wf[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      col[i] = __ldg(perm + g * 128 + 4 * lane + i);
      const bool in = col[i] >= 0 && col[i] < K;  // a perm that is not a permutation: no stray access
      wf[i] = !in ? 0.0f
                  : kF16 ? __half2float(__ushort_as_half(__ldg(static_cast<const uint16_t*>(w) + n * K + col[i])))
                         : __ldg(static_cast<const float*>(w) + n * K + col[i]);
    }
    uint16_t sb;
    int z, u[4];
    w4_quantize_group(wf, zeros != nullptr, sb, z, u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (col[i] < 0 || col[i] >= K) continue;
      atomicOr(reinterpret_cast<unsigned int*>(qweight + n * (K >> 3) + (col[i] >> 3)),
               static_cast<unsigned int>(u[i]) << (4 * (col[i] & 7)));
      if (n == 0 && g_idx) g_idx[col[i]] = static_cast<int32_t>(g);
    }
    if (lane == 0) {
      scales[n * G + g] = sb;
      if (zeros) zeros[n * G + g] = static_cast<uint8_t>(z);
    }
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
  const int64_t rows_per_cta = kPackThreads / 32;
  int64_t grid = (N + rows_per_cta - 1) / rows_per_cta;
  if (grid > int64_t(di.num_sms) * 8) grid = int64_t(di.num_sms) * 8;
  const int binw = 30 - ceil_log2_i64(K);
  const uintptr_t a = reinterpret_cast<uintptr_t>(w);
  if (w_f16 && K % 8 == 0 && a % 16 == 0) {
    // rows that fit in shared memory: one bulk copy per row, every pass from shared memory; four
    // to eight warps per CTA, one row each, within 55 KB (four CTAs per SM); longer rows (up to
    // 100 KB) one per CTA, double-buffered; the grid is what stays resident
    const int64_t row_bytes = 2 * K;
    const int W = static_cast<int>(std::min<int64_t>(8, (55 * 1024) / (row_bytes + 8)));
    if (W < 4 && 2 * row_bytes + 1024 <= 200 * 1024) {
      const int smem = static_cast<int>(2 * row_bytes + 16 + sizeof(PackCtaRed));
      const void* kern = reinterpret_cast<const void*>(tq_pack_f16_row_cta_kernel);
      cudaError_t e = ensure_smem_attr(kern, smem);
      if (e != cudaSuccess) return e;
      int bps = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, tq_pack_f16_row_cta_kernel, kPackThreads, smem) !=
              cudaSuccess ||
          bps < 1) {
        (void)cudaGetLastError();
        bps = 1;
      }
      const int64_t g = std::min<int64_t>(N, static_cast<int64_t>(di.num_sms) * bps);
      tq_pack_f16_row_cta_kernel<<<static_cast<unsigned>(g), kPackThreads, smem, s>>>(
          static_cast<const uint16_t*>(w), packed, scale, N, K);
      return cudaGetLastError();
    }
    if (W >= 4) {
      const int smem = static_cast<int>(W * (row_bytes + 8));
      const void* kern = reinterpret_cast<const void*>(tq_pack_f16_smem_kernel);
      cudaError_t e = ensure_smem_attr(kern, smem);
      if (e != cudaSuccess) return e;
      int bps = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, tq_pack_f16_smem_kernel, W * 32, smem) != cudaSuccess ||
          bps < 1) {
        (void)cudaGetLastError();
        bps = 1;
      }
      const int64_t g = std::min<int64_t>((N + W - 1) / W, static_cast<int64_t>(di.num_sms) * bps);
      tq_pack_f16_smem_kernel<<<static_cast<unsigned>(g), W * 32, smem, s>>>(static_cast<const uint16_t*>(w), packed,
                                                                             scale, N, K);
      return cudaGetLastError();
    }
    // the fp32 row sums need fewer than 2^13 elements per lane
    if (K < (int64_t(1) << 18))
      tq_pack_f16_kernel<true><<<static_cast<unsigned>(grid), kPackThreads, 0, s>>>(
          static_cast<const uint16_t*>(w), packed, scale, N, K);
    else
      tq_pack_f16_kernel<false><<<static_cast<unsigned>(grid), kPackThreads, 0, s>>>(
          static_cast<const uint16_t*>(w), packed, scale, N, K);
    return cudaGetLastError();
  }
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
  return launch_w4g_pack_ex(w, w_f16, nullptr, qweight, scales, nullptr, nullptr, N, K, s);
}

cudaError_t launch_w4g_pack_ex(const void* w, bool w_f16, const int32_t* perm, int32_t* qweight, uint16_t* scales,
                               uint8_t* zeros, int32_t* g_idx, int64_t N, int64_t K, cudaStream_t s) {
  const DeviceInfo di = current_device_info();
  const int64_t items = N * (K >> 7);
  int64_t grid = (items + 7) / 8;
  if (grid > int64_t(di.num_sms) * 16) grid = int64_t(di.num_sms) * 16;
  if (perm) {
    cudaError_t e = cudaMemsetAsync(qweight, 0, static_cast<size_t>(N) * static_cast<size_t>(K / 2), s);
    if (e != cudaSuccess) return e;
    if (w_f16)
      w4g_pack_perm_kernel<true><<<static_cast<unsigned>(grid), 256, 0, s>>>(w, perm, qweight, scales, zeros, g_idx, N, K);
    else
      w4g_pack_perm_kernel<false><<<static_cast<unsigned>(grid), 256, 0, s>>>(w, perm, qweight, scales, zeros, g_idx, N, K);
    return cudaGetLastError();
  }
  if (g_idx) {  // contiguous groups: g_idx[k] = k / 128
    cudaError_t e = launch_iota_groups(g_idx, K, s);
    if (e != cudaSuccess) return e;
  }
  const uintptr_t a = reinterpret_cast<uintptr_t>(w);
  const int vec = (a % (w_f16 ? 8 : 16) == 0);
  // eight warps per CTA, each taking 16 items a pass; the grid is what stays resident
  auto go = [&](auto kern) {
    int bps = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, kern, 256, 0) != cudaSuccess || bps < 1) {
      (void)cudaGetLastError();
      bps = 1;
    }
    const int64_t g = std::min<int64_t>((items + 8 * kW4PackItems - 1) / (8 * kW4PackItems),
                                        static_cast<int64_t>(bps) * di.num_sms);
    kern<<<static_cast<unsigned>(g), 256, 0, s>>>(w, qweight, scales, zeros, items, vec);
    return cudaGetLastError();
  };
  if (w_f16) return zeros ? go(w4g_pack_kernel<true, true>) : go(w4g_pack_kernel<true, false>);
  return zeros ? go(w4g_pack_kernel<false, true>) : go(w4g_pack_kernel<false, false>);
}

}  // namespace tq
