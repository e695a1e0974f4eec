// tq_prefill.cu -- tensor-core GEMM for large M (prefill), ternary and W4A16 weights.
//
// This path is a dense contraction, so it runs on the 5th-generation tensor cores:
//   y[m, n] = sum_k x[m,k] * What[n,k]   as   D(TMEM, fp32) += A(x tile, smem) * B(What tile, smem)^T
// [TQ] §4.2-4.3 (prior art: decode the codes into fp16 tensor-core operands, accumulate in fp32,
// apply the per-row scale after the MMA; stage weights through shared memory).  On sm_100a:
//   * warp 0, one lane: TMA loads of the x tile (128 tokens x 64 k, fp16, 128-byte swizzle) and
//     of the packed weight tile (256 rows x 16 bytes ternary / 32 bytes W4A16) into a ring;
//   * warps 4-11 (256 threads, one weight row each): decode the packed row into fp16 and store
//     it in the K-major 128-byte-swizzle layout the UMMA descriptor expects -- exactly what TMA
//     would have written for an fp16 matrix, so A and B share one descriptor format;
//       ternary: (c - 1) is exact in fp16; the row scale is applied in the epilogue;
//       W4A16:   fp16(q * s[n, k/128]) (one rounding, <= 2^-11 relative);
//   * warp 1: allocates 256 TMEM columns (the 128 x 256 fp32 accumulator); one lane issues
//     tcgen05.mma (M=128, N=256, K=16, fp16 x fp16 -> fp32) and commits to mbarriers that free
//     the input stages;
//   * warps 0-3: epilogue -- tcgen05.ld the accumulator (lane = token row), apply scale / bias,
//     convert to fp16 and store.
// Every wait is bounded; a wait that runs out records a timeout in the device status word and
// the CTA skips the rest of its work, frees its TMEM and exits (kernels never trap).
//
// Decode of one ternary byte (4 codes c0..c3 at bits 0,2,4,6) to two fp16x2 (natural k order):
// replicate the byte into both 16-bit halves, AND with a mask and OR with an exponent so each
// code lands in the fraction bits where its weight is exactly 1 (bases 1024, 256, 64, 16), then
// one fp16x2 subtraction removes base + 1.  Four integer/fp16 operations per 4 weights.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kPBM = 128;        // tokens per tile (UMMA M)
constexpr int kPBN = 256;        // weight rows per tile (UMMA N)
constexpr int kPBK = 64;         // K per stage: one 128-byte swizzle row of fp16
constexpr int kPRingL = 4;       // stages of (x tile, packed tile)
constexpr int kPRingB = 3;       // stages of decoded weight tiles
constexpr int kPDecThreads = 256;
constexpr int kPThreads = 128 + kPDecThreads;
constexpr int kPTileA = kPBM * kPBK * 2;  // 16 KB
constexpr int kPTileB = kPBN * kPBK * 2;  // 32 KB
constexpr uint32_t kPTmemCols = 256;

template <bool kInt4>
struct PFmt {
  static constexpr int kRowBytes = kInt4 ? 32 : 16;  // packed bytes per row per k-block
  static constexpr int kTileP = kPBN * kRowBytes;
};

template <bool kInt4>
struct PrefillLayout {
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kPRingL * kPTileA;
  static constexpr int kOffP = kOffB + kPRingB * kPTileB;
  static constexpr int kOffScale = kOffP + kPRingL * PFmt<kInt4>::kTileP;
  static constexpr int kOffBias = kOffScale + kPBN * 4;
  static constexpr int kOffBar = kOffBias + kPBN * 4;
  // barriers: fullL[4], emptyA[4], emptyP[4], fullB[3], emptyB[3], accFull, tmem slot
  static constexpr int kNumBars = 3 * kPRingL + 2 * kPRingB + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffTmemSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;  // alignment slack
};

struct PrefillArgs {
  const __half* sc;    // ternary: scale[N]; W4A16: scales[N, K/128]
  const __half* bias;  // may be null
  __half* y;
  int64_t M, N, K;
};

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Byte `bi` of w replicated into bits 0-7 and 16-23.
__device__ __forceinline__ uint32_t byte_to_halves(uint32_t w, int bi) {
  return __byte_perm(w, 0u, static_cast<uint32_t>(bi | (4 << 4) | (bi << 8) | (4 << 12)));
}

// 8 consecutive ternary codes (bytes b0 = byte 2j, b1 = byte 2j+1 of the row) -> 8 fp16 (c - 1).
__device__ __forceinline__ uint4 decode_tq_8(uint32_t w, int bpair) {
  const uint32_t t0 = byte_to_halves(w, 2 * bpair), t1 = byte_to_halves(w, 2 * bpair + 1);
  // (1025, 257) and (65, 17) as fp16x2: 0x5C04'6401 and 0x4C40'5410
  uint4 r;
  r.x = hsub2_u32((t0 & 0x000C0003u) | 0x5C006400u, 0x5C046401u);
  r.y = hsub2_u32((t0 & 0x00C00030u) | 0x4C005400u, 0x4C405410u);
  r.z = hsub2_u32((t1 & 0x000C0003u) | 0x5C006400u, 0x5C046401u);
  r.w = hsub2_u32((t1 & 0x00C00030u) | 0x4C005400u, 0x4C405410u);
  return r;
}

// 8 consecutive INT4 codes (one int32 word) -> 8 fp16 q * s, s2 = (s, s).
__device__ __forceinline__ uint4 decode_w4_8(uint32_t w, uint32_t s2) {
  uint32_t o[4];
#pragma unroll
  for (int bi = 0; bi < 4; ++bi) {
    const uint32_t t = byte_to_halves(w, bi);
    // low nibble -> 1024 + u (0x6400 base), high nibble -> 64 + u (0x5400 base, bits 4-7)
    const uint32_t h = (t & 0x00F0000Fu) | 0x54006400u;
    o[bi] = hmul2_u32(hsub2_u32(h, 0x54806408u /* (1032, 72) */), s2);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <bool kInt4>
__global__ void __launch_bounds__(kPThreads, 1)
    prefill_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ CUtensorMap tmap_w, const PrefillArgs a) {
  using L = PrefillLayout<kInt4>;
  using F = PFmt<kInt4>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned; pointer arithmetic on the __shared__ array keeps the shared address
  // space visible to the compiler (plain ld/st.shared instead of generic accesses)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
  uint64_t* fullL = bars;
  uint64_t* emptyA = bars + kPRingL;
  uint64_t* emptyP = bars + 2 * kPRingL;
  uint64_t* fullB = bars + 3 * kPRingL;
  uint64_t* emptyB = fullB + kPRingB;
  uint64_t* accFull = emptyB + kPRingB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kOffTmemSlot);
  float* sScale = reinterpret_cast<float*>(sm + L::kOffScale);
  float* sBias = reinterpret_cast<float*>(sm + L::kOffBias);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kPBN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kPBM;
  const int nk = static_cast<int>(a.K / kPBK);
  const int64_t G = a.K >> 7;

  pdl_allow_dependents();

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPRingL; ++i) {
      mbar_init(&fullL[i], 1);
      mbar_init(&emptyA[i], 1);
      mbar_init(&emptyP[i], kPDecThreads);
    }
    for (int i = 0; i < kPRingB; ++i) {
      mbar_init(&fullB[i], kPDecThreads);
      mbar_init(&emptyB[i], 1);
    }
    mbar_init(accFull, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kPTmemCols);
    tmem_relinquish();
  }
  if (warp >= 4) {
    const int r = threadIdx.x - 128;
    const int64_t n = n0 + r;
    sScale[r] = (!kInt4 && n < a.N) ? __half2float(a.sc[n]) : 0.0f;
    sBias[r] = (a.bias && n < a.N) ? __half2float(a.bias[n]) : 0.0f;
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_d = *tmem_slot;

  bool ok = true;
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    pdl_wait_prior_grids();
    if (lane == 0) {
      tma_prefetch_desc(&tmap_x);
      tma_prefetch_desc(&tmap_w);
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % kPRingL;
        if (kb >= kPRingL) {
          const uint32_t par = static_cast<uint32_t>((kb / kPRingL) - 1) & 1u;
          ok = mbar_wait(&emptyA[s], par) && mbar_wait(&emptyP[s], par);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(&fullL[s], kPTileA + F::kTileP);
        tma_load_2d(sm + L::kOffA + s * kPTileA, &tmap_x, &fullL[s], kb * kPBK, static_cast<int32_t>(m0));
        tma_load_2d(sm + L::kOffP + s * F::kTileP, &tmap_w, &fullL[s], kb * F::kRowBytes,
                    static_cast<int32_t>(n0));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    pdl_wait_prior_grids();  // x arrives only after the previous kernel: block, do not poll
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kPBM, kPBN);
      const uint32_t a_base = smem_u32(sm + L::kOffA), b_base = smem_u32(sm + L::kOffB);
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % kPRingL, b = kb % kPRingB;
        ok = mbar_wait(&fullL[s], static_cast<uint32_t>(kb / kPRingL) & 1u) &&
             mbar_wait(&fullB[b], static_cast<uint32_t>(kb / kPRingB) & 1u);
        if (!ok) break;
        tc_fence_after_sync();
        const uint64_t adesc = sdesc_kmajor_sw128(a_base + s * kPTileA);
        const uint64_t bdesc = sdesc_kmajor_sw128(b_base + b * kPTileB);
#pragma unroll
        for (int k16 = 0; k16 < kPBK / 16; ++k16) {
          // +32 bytes along K inside the swizzle atom = +2 in the encoded start address
          umma_f16(tmem_d, adesc + 2 * k16, bdesc + 2 * k16, idesc, (kb | k16) != 0 ? 1u : 0u);
        }
        umma_commit(&emptyA[s]);
        umma_commit(&emptyB[b]);
      }
      if (ok) umma_commit(accFull);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ decode warps
    const int r = threadIdx.x - 128;  // weight row within the tile
    const int64_t n = n0 + r;
    uint8_t* brow_base = sm + L::kOffB + (r >> 3) * 1024 + (r & 7) * 128;
    const int sw = r & 7;
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int s = kb % kPRingL, b = kb % kPRingB;
      ok = mbar_wait(&fullL[s], static_cast<uint32_t>(kb / kPRingL) & 1u);
      if (!ok) break;
      const uint8_t* prow = sm + L::kOffP + s * F::kTileP + r * F::kRowBytes;
      uint4 p0 = *reinterpret_cast<const uint4*>(prow);
      uint4 p1 = make_uint4(0u, 0u, 0u, 0u);
      if (kInt4) p1 = *reinterpret_cast<const uint4*>(prow + 16);
      mbar_arrive(&emptyP[s]);
      uint32_t s2 = 0u;
      if (kInt4) {
        const uint16_t sb = (n < a.N) ? __half_as_ushort(a.sc[n * G + (kb >> 1)]) : static_cast<uint16_t>(0);
        s2 = static_cast<uint32_t>(sb) | (static_cast<uint32_t>(sb) << 16);
      }
      if (kb >= kPRingB) {
        ok = mbar_wait(&emptyB[b], static_cast<uint32_t>((kb / kPRingB) - 1) & 1u);
        if (!ok) break;
      }
      uint8_t* brow = brow_base + b * kPTileB;
      const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 v = kInt4 ? decode_w4_8(pw[j], s2) : decode_tq_8(pw[j >> 1], j & 1);
        *reinterpret_cast<uint4*>(brow + ((j ^ sw) << 4)) = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(&fullB[b]);
    }
  }

  // -------------------------------------------------------------------- epilogue (warps 0-3)
  if (warp < 4) {
    if (warp != 0) pdl_wait_prior_grids();
    __syncwarp();
    const bool acc_ok = mbar_wait(accFull, 0u);
    tc_fence_after_sync();
    const int64_t m = m0 + warp * 32 + lane;
    const uint32_t taddr = tmem_d + (static_cast<uint32_t>(warp * 32) << 16);
    if (acc_ok) {
      const bool vec = ((a.N & 7) == 0);
#pragma unroll 1
      for (int c = 0; c < kPBN / 32; ++c) {
        uint32_t rr[32];
        tmem_ld_32x32b_x32(taddr + c * 32, rr);
        tmem_ld_wait();
        if (m < a.M) {
          const int64_t nb = n0 + c * 32;
          __align__(16) __half o[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float v = __uint_as_float(rr[j]);
            const float yv = kInt4 ? (v + sBias[c * 32 + j]) : fmaf(v, sScale[c * 32 + j], sBias[c * 32 + j]);
            o[j] = __float2half_rn(yv);
          }
          __half* dst = a.y + m * a.N + nb;
          if (vec && nb + 32 <= a.N) {
#pragma unroll
            for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(dst)[q] = reinterpret_cast<const uint4*>(o)[q];
          } else {
            for (int j = 0; j < 32; ++j)
              if (nb + j < a.N) dst[j] = o[j];
          }
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_d, kPTmemCols);
  }
}

bool prefill_supported(bool int4, int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1) return false;
  if (K < kPBK) return false;
  if (int4 ? (K % 128 != 0) : (K % 64 != 0)) return false;
  if ((M + kPBM - 1) / kPBM > 65535) return false;
  return true;
}

template <bool kInt4>
static cudaError_t launch_prefill(const __half* x, const void* w, const __half* sc,
                                  const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                  cudaStream_t s) {
  using L = PrefillLayout<kInt4>;
  using F = PFmt<kInt4>;
  CUtensorMap tx, tw;
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, static_cast<uint64_t>(K),
                    static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, kPBK, kPBM,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const uint64_t kbytes = kInt4 ? static_cast<uint64_t>(K) / 2 : static_cast<uint64_t>(K) / 4;
  if (!make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, kbytes, static_cast<uint64_t>(N), kbytes,
                    F::kRowBytes, kPBN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  auto* kern = prefill_gemm_kernel<kInt4>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), L::kAlloc);
  if (e != cudaSuccess) return e;
  PrefillArgs a;
  a.sc = sc;
  a.bias = bias;
  a.y = y;
  a.M = M;
  a.N = N;
  a.K = K;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((N + kPBN - 1) / kPBN), static_cast<unsigned>((M + kPBM - 1) / kPBM), 1);
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tx, tw, a);
}

cudaError_t launch_tq_gemm_prefill(const __half* x, const uint8_t* packed, const __half* scale,
                                   const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                   cudaStream_t s) {
  return launch_prefill<false>(x, packed, scale, bias, y, M, N, K, s);
}

cudaError_t launch_w4g_gemm_prefill(const __half* x, const int32_t* qweight, const __half* scales,
                                    const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                    cudaStream_t s) {
  return launch_prefill<true>(x, qweight, scales, bias, y, M, N, K, s);
}

}  // namespace tq
