// tq_decode.cu -- memory-bound skinny GEMM (M <= 16) for ternary and W4A16 weights.
//
// [TQ] §1: decode time is spent fetching weights, so the kernel is built around the HBM stream
// of packed codes; [TQ] §4.2: codes are decoded into fp16 tensor-core fragments, accumulated in
// fp32, and the per-row scale is applied after the MMA.
//
// Layout of the work (one CTA = 128 output rows x one K-slice; a cluster of S CTAs covers the
// whole K of its 128 rows and reduces through distributed shared memory, in a fixed order):
//   * warp 4 (one lane) streams 128-row x 128-byte tiles of packed weights with TMA (128-byte
//     swizzle, so the 16-byte reads below are bank-conflict free) into a ring of stages; it
//     starts before griddepcontrol.wait, since weights never depend on the previous kernel;
//   * warps 0-3 each own 32 rows (two 16-row MMA tiles).  Weights are the A operand of
//     mma.sync.m16n8k16 ("swap AB") and the tokens are the N=8 operand, so M <= 8 costs one MMA
//     per 256 weights and M <= 16 two.
//
// In-register decode ("subnormal" trick).  Masking a packed word leaves small integers in the
// fraction bits of each fp16 half, i.e. exact subnormal values c * 2^-24 (or c * 2^-22 when the
// code sits two bits higher).  Per 32-bit word of 16 ternary codes: 3 shifts + 8 ANDs give 8
// fp16x2 registers.  The 4x scale of the second mask position is folded into the activation
// fragment (x/4), so every product carries the same 2^-24 and a single fp32 accumulator per
// output suffices; the epilogue multiplies by 2^24 and subtracts sum_k x (codes are c = w + 1).
// The order of k inside an MMA is permuted; the activation fragments are built (once per CTA,
// in shared memory) in the matching order, so the weights are used in their canonical layout.
// W4A16 uses the same scheme with 4-bit fields (masks 0x000F000F / 0x00F000F0, x/16 fold) and
// one 128-wide quantisation group per 64-byte sub-chunk: y += s[n,g] * (2^24 * C_g - 8 sum_g x).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kDRows = 128;                      // output rows per CTA
constexpr int kDConsumers = 4;                   // consumer warps (32 rows each)
constexpr int kDThreads = (kDConsumers + 1) * 32;
constexpr int kDStageBytes = kDRows * 128;       // one TMA box: 128 rows x 128 bytes
constexpr int kDMaxRing = 4;
constexpr int kDMaxCluster = 8;

struct DecodeArgs {
  const __half* x;
  const __half* sc;    // ternary: scale[N]; W4A16: scales[N, K/128]
  const __half* bias;  // may be null
  __half* y;
  int64_t M, N, K;
  int C;          // stages along K (128 packed bytes of every row per stage)
  int S;          // CTAs per cluster (K-slices)
  int ring;       // stages resident in shared memory
  int max_local;  // ceil(C / S)
};

template <bool kInt4>
struct DecFmt {
  static constexpr int kSubK = kInt4 ? 128 : 256;   // codes per 64-byte sub-chunk
  static constexpr int kLaneK = kInt4 ? 32 : 64;     // codes per lane (16 bytes) per sub-chunk
  static constexpr int kMmas = kInt4 ? 8 : 16;       // MMAs per 16-row tile per sub-chunk
  static constexpr int kFragU4 = kMmas / 2;          // uint4 activation fragments per lane
  static constexpr int kFragBytes = kFragU4 * 32 * 16;
};

struct DecodeSmem {
  uint8_t* stage;
  uint4* xf;
  float* sx;
  float* part;
  uint64_t* full;
  uint64_t* empty;
};

template <bool kInt4, int NT>
__device__ __forceinline__ DecodeSmem decode_smem_carve(uint8_t* base, const DecodeArgs& a) {
  DecodeSmem s;
  uint8_t* p = base;
  s.stage = p;
  p += a.ring * kDStageBytes;
  const int nsub = 2 * a.max_local;
  s.xf = reinterpret_cast<uint4*>(p);
  p += nsub * NT * DecFmt<kInt4>::kFragBytes;
  s.sx = reinterpret_cast<float*>(p);
  p += nsub * 16 * sizeof(float);
  s.part = reinterpret_cast<float*>(p);
  p += kDRows * 16 * sizeof(float);
  s.full = reinterpret_cast<uint64_t*>(p);
  p += kDMaxRing * sizeof(uint64_t);
  s.empty = reinterpret_cast<uint64_t*>(p);
  return s;
}

__host__ __device__ constexpr int decode_smem_bytes(bool int4, int NT, int ring, int max_local) {
  return 1024 /* alignment slack */ + ring * kDStageBytes +
         2 * max_local * NT * (int4 ? 8 * 32 * 8 : 16 * 32 * 8) + 2 * max_local * 16 * 4 +
         kDRows * 16 * 4 + 2 * kDMaxRing * 8;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

template <bool kInt4, int NT>
__global__ void __launch_bounds__(kDThreads)
    decode_gemm_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  using F = DecFmt<kInt4>;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const DecodeSmem sm = decode_smem_carve<kInt4, NT>(base, a);

  pdl_allow_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const int rb = blockIdx.y;
  const int st_begin = static_cast<int>((static_cast<int64_t>(rank) * a.C) / a.S);
  const int st_end = static_cast<int>((static_cast<int64_t>(rank + 1) * a.C) / a.S);
  const int nst = st_end - st_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < a.ring; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kDConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDConsumers) {
    // ------------------------------------------------------------- producer: weight tiles
    if (lane == 0) {
      tma_prefetch_desc(&tmap);
      for (int i = 0; i < nst; ++i) {
        const int slot = i % a.ring;
        if (i >= a.ring && !mbar_wait(&sm.empty[slot], static_cast<uint32_t>((i / a.ring) - 1) & 1u)) break;
        mbar_arrive_expect_tx(&sm.full[slot], kDStageBytes);
        tma_load_2d(sm.stage + slot * kDStageBytes, &tmap, &sm.full[slot], (st_begin + i) * 128,
                    rb * kDRows);
      }
    }
    pdl_wait_prior_grids();  // this warp also writes y in the epilogue
  } else {
    // ------------------------------------------------------------- consumers
    const int g = lane >> 2, t = lane & 3;
    pdl_wait_prior_grids();  // x (and y) may belong to the previous kernel in the stream

    // Stage the activation fragments of this CTA's K-slice, in MMA order.
    const int nsub = 2 * nst;
    for (int p = warp; p < nsub * NT; p += kDConsumers) {
      const int scl = p / NT, T = p - scl * NT;
      const int m = 8 * T + g;
      const int64_t kb = static_cast<int64_t>(st_begin * 2 + scl) * F::kSubK + t * F::kLaneK;
      __align__(16) __half X[F::kLaneK];
      if (m < a.M && kb + F::kLaneK <= a.K) {
        const uint4* src = reinterpret_cast<const uint4*>(a.x + m * a.K + kb);
#pragma unroll
        for (int i = 0; i < F::kLaneK / 8; ++i) reinterpret_cast<uint4*>(X)[i] = __ldg(src + i);
      } else {
#pragma unroll
        for (int i = 0; i < F::kLaneK; ++i)
          X[i] = (m < a.M && kb + i < a.K) ? a.x[m * a.K + kb + i] : __float2half_rn(0.0f);
      }
      float sum = 0.0f;
#pragma unroll
      for (int i = 0; i < F::kLaneK; ++i) sum += __half2float(X[i]);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
      if (t == 0) sm.sx[scl * 16 + m] = sum;
      const __half2 q4 = __floats2half2_rn(0.25f, 0.25f);
      const __half2 q16 = __floats2half2_rn(0.0625f, 0.0625f);
#pragma unroll
      for (int ip = 0; ip < F::kFragU4; ++ip) {
        uint32_t r[4];
#pragma unroll
        for (int cls = 0; cls < 2; ++cls) {
          __half2 b01, b23;
          if (!kInt4) {
            const int h = ip >> 2, s = ip & 3, pp = 2 * s + cls;
            b01 = __halves2half2(X[32 * h + pp], X[32 * h + 8 + pp]);
            b23 = __halves2half2(X[32 * h + 16 + pp], X[32 * h + 24 + pp]);
            if (cls) {
              b01 = __hmul2(b01, q4);
              b23 = __hmul2(b23, q4);
            }
          } else {
            const int h = ip >> 1, s = ip & 1, pp = 2 * s + cls;
            b01 = __halves2half2(X[16 * h + pp], X[16 * h + 4 + pp]);
            b23 = __halves2half2(X[16 * h + 8 + pp], X[16 * h + 12 + pp]);
            if (cls) {
              b01 = __hmul2(b01, q16);
              b23 = __hmul2(b23, q16);
            }
          }
          r[2 * cls] = h2_bits(b01);
          r[2 * cls + 1] = h2_bits(b23);
        }
        sm.xf[((scl * NT + T) * F::kFragU4 + ip) * 32 + lane] = make_uint4(r[0], r[1], r[2], r[3]);
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kDConsumers * 32) : "memory");

    float acc[2][NT][4];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
      for (int T = 0; T < NT; ++T)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[rt][T][c] = 0.0f;

    const int64_t G = a.K >> 7;
    for (int i = 0; i < nst; ++i) {
      const int slot = i % a.ring;
      if (!mbar_wait(&sm.full[slot], static_cast<uint32_t>(i / a.ring) & 1u)) break;
      const uint8_t* st = sm.stage + slot * kDStageBytes;
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        const int scl = 2 * i + sub;
        uint4 bf[NT][F::kFragU4];
#pragma unroll
        for (int T = 0; T < NT; ++T)
#pragma unroll
          for (int ip = 0; ip < F::kFragU4; ++ip)
            bf[T][ip] = sm.xf[((scl * NT + T) * F::kFragU4 + ip) * 32 + lane];
        float xg[NT][2];
        int64_t gi = 0;
        if (kInt4) {
          gi = static_cast<int64_t>(st_begin + i) * 2 + sub;
#pragma unroll
          for (int T = 0; T < NT; ++T) {
            xg[T][0] = 8.0f * sm.sx[scl * 16 + 8 * T + 2 * t];
            xg[T][1] = 8.0f * sm.sx[scl * 16 + 8 * T + 2 * t + 1];
          }
        }
        const int chunk = sub * 4 + t;
#pragma unroll
        for (int rt = 0; rt < 2; ++rt) {
          const int r0 = warp * 32 + rt * 16 + g, r1 = r0 + 8;
          const uint4 U0 = *reinterpret_cast<const uint4*>(st + r0 * 128 + ((chunk ^ (r0 & 7)) << 4));
          const uint4 U1 = *reinterpret_cast<const uint4*>(st + r1 * 128 + ((chunk ^ (r1 & 7)) << 4));
          const uint32_t w0[4] = {U0.x, U0.y, U0.z, U0.w};
          const uint32_t w1[4] = {U1.x, U1.y, U1.z, U1.w};
          if (!kInt4) {
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int s = 0; s < 4; ++s) {
                const uint32_t x0 = w0[2 * h] >> (4 * s), x1 = w1[2 * h] >> (4 * s);
                const uint32_t x2 = w0[2 * h + 1] >> (4 * s), x3 = w1[2 * h + 1] >> (4 * s);
#pragma unroll
                for (int cls = 0; cls < 2; ++cls) {
                  const uint32_t mk = cls ? 0x000C000Cu : 0x00030003u;
                  const int ip = h * 4 + s;
#pragma unroll
                  for (int T = 0; T < NT; ++T) {
                    const uint32_t b0 = cls ? bf[T][ip].z : bf[T][ip].x;
                    const uint32_t b1 = cls ? bf[T][ip].w : bf[T][ip].y;
                    mma_16816(acc[rt][T], x0 & mk, x1 & mk, x2 & mk, x3 & mk, b0, b1);
                  }
                }
              }
          } else {
            float cg[NT][4];
#pragma unroll
            for (int T = 0; T < NT; ++T)
#pragma unroll
              for (int c = 0; c < 4; ++c) cg[T][c] = 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int s = 0; s < 2; ++s) {
                const uint32_t x0 = w0[2 * h] >> (8 * s), x1 = w1[2 * h] >> (8 * s);
                const uint32_t x2 = w0[2 * h + 1] >> (8 * s), x3 = w1[2 * h + 1] >> (8 * s);
#pragma unroll
                for (int cls = 0; cls < 2; ++cls) {
                  const uint32_t mk = cls ? 0x00F000F0u : 0x000F000Fu;
                  const int ip = h * 2 + s;
#pragma unroll
                  for (int T = 0; T < NT; ++T) {
                    const uint32_t b0 = cls ? bf[T][ip].z : bf[T][ip].x;
                    const uint32_t b1 = cls ? bf[T][ip].w : bf[T][ip].y;
                    mma_16816(cg[T], x0 & mk, x1 & mk, x2 & mk, x3 & mk, b0, b1);
                  }
                }
              }
            const int64_t n0 = static_cast<int64_t>(rb) * kDRows + r0, n1 = n0 + 8;
            // groups past K (a zero-filled half stage) contribute nothing
            const float s0 = (n0 < a.N && gi < G) ? __half2float(a.sc[n0 * G + gi]) : 0.0f;
            const float s1 = (n1 < a.N && gi < G) ? __half2float(a.sc[n1 * G + gi]) : 0.0f;
#pragma unroll
            for (int T = 0; T < NT; ++T) {
              acc[rt][T][0] = fmaf(s0, fmaf(cg[T][0], 16777216.0f, -xg[T][0]), acc[rt][T][0]);
              acc[rt][T][1] = fmaf(s0, fmaf(cg[T][1], 16777216.0f, -xg[T][1]), acc[rt][T][1]);
              acc[rt][T][2] = fmaf(s1, fmaf(cg[T][2], 16777216.0f, -xg[T][0]), acc[rt][T][2]);
              acc[rt][T][3] = fmaf(s1, fmaf(cg[T][3], 16777216.0f, -xg[T][1]), acc[rt][T][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
    }

    // partial results of this K-slice -> shared memory part[row][token]
    float sxt[NT][2];
#pragma unroll
    for (int T = 0; T < NT; ++T) {
      sxt[T][0] = 0.0f;
      sxt[T][1] = 0.0f;
      if (!kInt4) {
        for (int scl = 0; scl < nsub; ++scl) {
          sxt[T][0] += sm.sx[scl * 16 + 8 * T + 2 * t];
          sxt[T][1] += sm.sx[scl * 16 + 8 * T + 2 * t + 1];
        }
      }
    }
#pragma unroll
    for (int rt = 0; rt < 2; ++rt) {
      const int r0 = warp * 32 + rt * 16 + g, r1 = r0 + 8;
#pragma unroll
      for (int T = 0; T < NT; ++T) {
        const int m0 = 8 * T + 2 * t;
        if (!kInt4) {
          sm.part[r0 * 16 + m0] = fmaf(acc[rt][T][0], 16777216.0f, -sxt[T][0]);
          sm.part[r0 * 16 + m0 + 1] = fmaf(acc[rt][T][1], 16777216.0f, -sxt[T][1]);
          sm.part[r1 * 16 + m0] = fmaf(acc[rt][T][2], 16777216.0f, -sxt[T][0]);
          sm.part[r1 * 16 + m0 + 1] = fmaf(acc[rt][T][3], 16777216.0f, -sxt[T][1]);
        } else {
          sm.part[r0 * 16 + m0] = acc[rt][T][0];
          sm.part[r0 * 16 + m0 + 1] = acc[rt][T][1];
          sm.part[r1 * 16 + m0] = acc[rt][T][2];
          sm.part[r1 * 16 + m0 + 1] = acc[rt][T][3];
        }
      }
    }
  }

  // --------------------------------------------------------------- cluster reduction, epilogue
  cluster_sync_all();
  {
    const int rr0 = (rank * kDRows) / a.S, rr1 = ((rank + 1) * kDRows) / a.S;
    const int nrows = rr1 - rr0;
    const int Mv = static_cast<int>(a.M < 8 * NT ? a.M : 8 * NT);
    const uint32_t part_local = smem_u32(sm.part);
    for (int idx = threadIdx.x; idx < nrows * Mv; idx += kDThreads) {
      const int m = idx / nrows, r = rr0 + (idx - m * nrows);
      const int64_t n = static_cast<int64_t>(rb) * kDRows + r;
      if (n >= a.N) continue;
      float v = 0.0f;
      const uint32_t off = static_cast<uint32_t>((r * 16 + m) * sizeof(float));
      for (int q = 0; q < a.S; ++q) v += ld_shared_cluster_f32(mapa_shared(part_local + off, q));
      if (!kInt4) v *= __half2float(a.sc[n]);
      if (a.bias) v += __half2float(a.bias[n]);
      a.y[m * a.N + n] = __float2half_rn(v);
    }
  }
  cluster_sync_all();
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
struct DecodePlan {
  int S, C, ring, max_local, smem;
};

static bool plan_decode(bool int4, int NT, int64_t N, int64_t K, int num_sms, DecodePlan* p) {
  const int64_t kbytes = int4 ? K / 2 : K / 4;
  const int C = static_cast<int>((kbytes + 127) / 128);
  const int64_t RB = (N + kDRows - 1) / kDRows;
  const int64_t target = 2 * static_cast<int64_t>(num_sms);
  int S = static_cast<int>((target + RB - 1) / RB);
  if (S < 1) S = 1;
  const int smax = C < kDMaxCluster ? C : kDMaxCluster;
  if (S > smax) S = smax;
  for (;; ++S) {
    const int ml = (C + S - 1) / S;
    const int ring = ml < kDMaxRing ? ml : kDMaxRing;
    const int bytes = decode_smem_bytes(int4, NT, ring, ml);
    if (bytes <= 227 * 1024) {
      *p = DecodePlan{S, C, ring, ml, bytes};
      return true;
    }
    if (S >= smax) return false;
  }
}

template <bool kInt4, int NT>
static cudaError_t launch_decode_t(const CUtensorMap& tmap, const DecodeArgs& a, const DecodePlan& p,
                                   cudaStream_t s) {
  auto* kern = decode_gemm_kernel<kInt4, NT>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), p.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.S), static_cast<unsigned>((a.N + kDRows - 1) / kDRows), 1);
  cfg.blockDim = dim3(kDThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (p.S > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(p.S);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, tmap, a);
}

template <bool kInt4>
static cudaError_t launch_decode(const __half* x, const void* w, const __half* sc,
                                 const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                 cudaStream_t s) {
  const DeviceInfo di = current_device_info();
  const int NT = M > 8 ? 2 : 1;
  DecodePlan p;
  if (!plan_decode(kInt4, NT, N, K, di.num_sms, &p)) return cudaErrorInvalidValue;
  const int64_t kbytes = kInt4 ? K / 2 : K / 4;
  CUtensorMap tmap;
  if (!make_tmap_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, static_cast<uint64_t>(kbytes),
                    static_cast<uint64_t>(N), static_cast<uint64_t>(kbytes), 128, kDRows,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  DecodeArgs a;
  a.x = x;
  a.sc = sc;
  a.bias = bias;
  a.y = y;
  a.M = M;
  a.N = N;
  a.K = K;
  a.C = p.C;
  a.S = p.S;
  a.ring = p.ring;
  a.max_local = p.max_local;
  return NT == 1 ? launch_decode_t<kInt4, 1>(tmap, a, p, s) : launch_decode_t<kInt4, 2>(tmap, a, p, s);
}

bool decode_supported(bool int4, int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > 16 || N < 1) return false;
  if (int4 ? (K % 128 != 0) : (K % 64 != 0)) return false;
  DecodePlan p;
  return plan_decode(int4, M > 8 ? 2 : 1, N, K, 148, &p);
}

cudaError_t launch_tq_gemm_decode(const __half* x, const uint8_t* packed, const __half* scale,
                                  const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                  cudaStream_t s) {
  return launch_decode<false>(x, packed, scale, bias, y, M, N, K, s);
}

cudaError_t launch_w4g_gemm_decode(const __half* x, const int32_t* qweight, const __half* scales,
                                   const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                   cudaStream_t s) {
  return launch_decode<true>(x, qweight, scales, bias, y, M, N, K, s);
}

}  // namespace tq
