// tq_decode.cu -- memory-bound skinny GEMM (M <= 16) for ternary and W4A16 weights.
//
// [TQ] §1: decode time is spent fetching weights, so the kernel is built around the HBM stream
// of packed codes; [TQ] §4.2: codes are decoded into fp16 tensor-core fragments, accumulated in
// fp32, and the per-row scale is applied after the MMA.
//
// Work layout.  One CTA = 128 output rows x one K-slice; a cluster of S CTAs (S <= 8) covers
// the whole K of its 128 rows and reduces through distributed shared memory in a fixed order
// (deterministic, no global scratch).  Per CTA:
//   * warps 0-3 (consumers) each own 32 rows = two 16-row MMA tiles.  Weights are the A operand
//     of mma.sync.m16n8k16 ("swap AB"), the tokens the N = 8 operand: one MMA per 256 weights
//     for M <= 8, two for M <= 16;
//   * warp 4 (producer): lane 0 streams 128-row x 128-byte packed tiles with TMA (128-byte
//     swizzle: the 16-byte fragment reads are bank-conflict free) into a ring, starting before
//     griddepcontrol.wait because weights never depend on the previous kernel; all 32 lanes then
//     copy the activations of each stage (cp.async, padded, conflict-free), rearrange them into
//     ready-made B fragments in the k order the decode produces (byte permutes), and compute the
//     per-token sums of x on the tensor core (an MMA with an all-ones A).
//
// In-register decode ("subnormal" trick).  ANDing a packed 32-bit word with 0x00030003 << 2p
// leaves, in each fp16 half, the code at bits 2p..2p+1: the exact value c * 2^(2p-24) (fp16
// subnormals for p <= 4, and still exactly linear for p = 5 where the code fills the two lowest
// exponent bits).  Positions 6, 7 are shifted down by 12 first.  So one word of 16 codes costs
// 1 shift + 8 ANDs for 8 fp16x2 registers, ~0.56 integer operations per weight.  The odd
// positions carry an extra factor 4, folded into their activation fragments (x / 4); the
// remaining factors 2^-24, 2^-20, 2^-16 are kept apart in separate accumulators and applied
// exactly (powers of two) in the epilogue, which also subtracts sum_k x (codes are c = w + 1).
// One accumulator per position pair keeps the dependent MMA chains short (latency, not issue,
// bounds a skinny GEMM).
// W4A16 uses the same scheme with 4-bit fields (masks 0x000F000F / 0x00F000F0, x / 16 fold) and
// one 128-wide quantisation group per 64-byte sub-chunk: y += s[n,g] * (2^24 * C_g - 8 sum_g x).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kDRows = 128;                 // output rows per CTA
constexpr int kDConsumers = 8;              // consumer warps (16 rows = one MMA tile each)
constexpr int kDRT = kDRows / (16 * kDConsumers);  // 16-row MMA tiles per consumer warp
constexpr int kDBuilders = 2;               // activation warps: one per 64-byte sub-chunk
constexpr int kDBuildWarp0 = kDConsumers;
constexpr int kDTmaWarp = kDConsumers + kDBuilders;  // issues the weight TMA stream
constexpr int kDThreads = (kDConsumers + kDBuilders + 1) * 32;
constexpr int kDStageBytes = kDRows * 128;  // one TMA box: 128 rows x 128 bytes
constexpr int kDMaxRing = 6;                // weight stages resident in shared memory
constexpr int kDXRing = 2;                  // activation-fragment stages
constexpr int kDMaxCluster = 8;
constexpr int kDRedRows = kDRows + kDMaxCluster;  // >= S * ceil(128 / S)
constexpr int kDSmemBudget = 113 * 1024;    // two CTAs per SM

template <bool kInt4>
struct DecFmt {
  static constexpr int kStageK = kInt4 ? 256 : 512;  // codes per stage (128 bytes of a row)
  static constexpr int kSubK = kStageK / 2;          // codes per 64-byte sub-chunk
  static constexpr int kLaneK = kSubK / 4;           // codes per lane (16 bytes) per sub-chunk
  static constexpr int kMmas = kInt4 ? 8 : 16;       // MMAs per 16-row tile per sub-chunk
  static constexpr int kFragU4 = kMmas / 2;          // uint4 B fragments per lane per sub-chunk
  static constexpr int kFragBytes = kFragU4 * 32 * 16;
  static constexpr int kXLaneBytes = kLaneK * 2;     // activation bytes per lane per sub-chunk
  static constexpr int kXStride = kXLaneBytes + 16;  // padded: conflict-free 16-byte reads
};

constexpr int kDMaxGroup = 4;  // weight matrices sharing x in one launch (e.g. q, k, v)

struct DecodeArgs {
  const __half* x;
  int64_t M, K;
  int C;     // stages along K
  int S;     // CTAs per cluster (K-slices)
  int ring;  // weight stages resident in shared memory (all of a CTA's stages when they fit)
  int count;                        // matrices in the group
  int rb_start[kDMaxGroup + 1];     // first 128-row block of each matrix in grid.y
  int64_t N[kDMaxGroup];
  const __half* sc[kDMaxGroup];     // ternary: scale[N]; W4A16: scales[N, K/128]
  const __half* bias[kDMaxGroup];   // may be null
  __half* y[kDMaxGroup];
};

struct DecodeMaps {
  CUtensorMap m[kDMaxGroup];        // packed weights of each matrix
};

template <bool kInt4, int NT>
struct DecLayout {
  using F = DecFmt<kInt4>;
  static constexpr int kXfStage = 2 * NT * F::kFragBytes;      // B fragments of one stage
  static constexpr int kXsSub = NT * 32 * F::kXStride;          // natural x of one sub-chunk
  static constexpr int kXgStage = 2 * 16 * 4;                   // W4A16 group sums [sub][token]
  static constexpr int kRed = kDRedRows * 16 * 4;
  static constexpr int kSxr = kDMaxCluster * 16 * 4;
  __host__ __device__ static constexpr int bytes(int ring) {
    return 1024 + ring * kDStageBytes + kDXRing * (kXfStage + kXgStage) + 2 * kDBuilders * kXsSub +
           kRed + kSxr + 2 * 16 * 4 + (2 * kDMaxRing + 2 * kDXRing) * 8;
  }
};

template <bool kInt4, int NT>
__global__ void __launch_bounds__(kDThreads, 2)
    decode_gemm_kernel(const __grid_constant__ DecodeMaps maps, const __grid_constant__ DecodeArgs a) {
  using F = DecFmt<kInt4>;
  using L = DecLayout<kInt4, NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wst = base;                                                // ring x 16 KB weight tiles
  uint8_t* xf = wst + a.ring * kDStageBytes;                          // 2 x B fragments
  float* xg = reinterpret_cast<float*>(xf + kDXRing * L::kXfStage);   // 2 x [2][16] group sums
  uint8_t* xs = reinterpret_cast<uint8_t*>(xg + kDXRing * 2 * 16);    // [builder][2] natural x
  float* red = reinterpret_cast<float*>(xs + 2 * kDBuilders * L::kXsSub);  // [S][rows/S][16]
  float* sxr = red + kDRedRows * 16;                                  // [S][16] slice sums of x
  float* sxb = sxr + kDMaxCluster * 16;                               // [builder][16] sums of x
  uint64_t* wfull = reinterpret_cast<uint64_t*>(sxb + 2 * 16);
  uint64_t* wempty = wfull + kDMaxRing;
  uint64_t* xfull = wempty + kDMaxRing;     // B fragments of a stage built (builder warps)
  uint64_t* xempty = xfull + kDXRing;       // ... and consumed (consumer warps)

  pdl_allow_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rank = static_cast<int>(cluster_ctarank());
  // which matrix of the group this CTA works on, and its 128-row block within that matrix
  int grp = 0;
#pragma unroll
  for (int q = 1; q < kDMaxGroup; ++q)
    if (q < a.count && static_cast<int>(blockIdx.y) >= a.rb_start[q]) grp = q;
  const int rb = static_cast<int>(blockIdx.y) - a.rb_start[grp];
  const CUtensorMap* tmap = &maps.m[grp];
  const int64_t Nm = a.N[grp];
  const __half* scm = a.sc[grp];
  const __half* biasm = a.bias[grp];
  __half* ym = a.y[grp];
  const int st_begin = static_cast<int>((static_cast<int64_t>(rank) * a.C) / a.S);
  const int st_end = static_cast<int>((static_cast<int64_t>(rank + 1) * a.C) / a.S);
  const int nst = st_end - st_begin;
  const int own_cap = (kDRows + a.S - 1) / a.S;  // row slots per owner in `red`

  if (threadIdx.x == 0) {
    for (int i = 0; i < a.ring; ++i) {
      mbar_init(&wfull[i], 1);
      mbar_init(&wempty[i], kDConsumers);
    }
    for (int i = 0; i < kDXRing; ++i) {
      mbar_init(&xfull[i], kDBuilders * 32);
      mbar_init(&xempty[i], kDConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDTmaWarp) {
    // ================================================================== weight TMA warp
    if (lane == 0) {
      tma_prefetch_desc(tmap);
      const int pre = nst < a.ring ? nst : a.ring;
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&wfull[i], kDStageBytes);
        tma_load_2d(wst + i * kDStageBytes, tmap, &wfull[i], (st_begin + i) * 128, rb * kDRows);
      }
      // refill each weight slot as soon as the consumers release it (they start only once the
      // previous kernel is done, so block in griddepcontrol.wait instead of polling meanwhile)
      if (a.ring < nst) pdl_wait_prior_grids();
      for (int j = a.ring; j < nst; ++j) {
        const int ws = j % a.ring;
        if (!mbar_wait(&wempty[ws], static_cast<uint32_t>((j / a.ring) - 1) & 1u)) break;
        mbar_arrive_expect_tx(&wfull[ws], kDStageBytes);
        tma_load_2d(wst + ws * kDStageBytes, tmap, &wfull[ws], (st_begin + j) * 128, rb * kDRows);
      }
    }
  } else if (warp >= kDBuildWarp0) {
    // ================================================================== builder warps
    // Builder `sub` owns the 64-byte sub-chunk `sub` of every stage: it copies those
    // activations (cp.async, padded), lays them out as B fragments in the k order the decode
    // produces (odd positions pre-scaled by 1/4 or 1/16), and sums x on the CUDA cores.
    const int sub = warp - kDBuildWarp0;
    pdl_wait_prior_grids();  // activations may come from the previous kernel
    uint8_t* mybuf = xs + sub * 2 * L::kXsSub;
    auto issue_x = [&](int i) {
      if (i < nst) {
        uint8_t* buf = mybuf + (i & 1) * L::kXsSub;
#pragma unroll
        for (int T = 0; T < NT; ++T) {
          const int m = 8 * T + g;
          const int64_t k0 = static_cast<int64_t>(st_begin + i) * F::kStageK + sub * F::kSubK + t * F::kLaneK;
          const bool valid = (m < a.M) && (k0 < a.K);
          const __half* src = valid ? a.x + m * a.K + k0 : a.x;
          uint8_t* dst = buf + (T * 32 + lane) * F::kXStride;
#pragma unroll
          for (int j = 0; j < F::kXLaneBytes / 16; ++j)
            cp_async_16(dst + 16 * j, src + (valid ? 8 * j : 0), valid ? 16u : 0u);
        }
      }
      cp_async_commit();  // one group per stage (possibly empty) keeps the accounting uniform
    };
    issue_x(0);
    issue_x(1);
    const __half2 fold = kInt4 ? __floats2half2_rn(0.0625f, 0.0625f) : __floats2half2_rn(0.25f, 0.25f);
    float sxl[NT];  // running sum of this lane's activations (ternary)
#pragma unroll
    for (int T = 0; T < NT; ++T) sxl[T] = 0.0f;
    for (int i = 0; i < nst; ++i) {
      const int xslot = i & 1;
      if (i >= kDXRing && !mbar_wait(&xempty[xslot], static_cast<uint32_t>((i >> 1) - 1) & 1u)) break;
      cp_async_wait<1>();  // this lane's copies of stage i have landed
      const uint8_t* buf = mybuf + (i & 1) * L::kXsSub;
      uint4* xfs = reinterpret_cast<uint4*>(xf + xslot * L::kXfStage);
#pragma unroll
      for (int T = 0; T < NT; ++T) {
        const uint4* src = reinterpret_cast<const uint4*>(buf + (T * 32 + lane) * F::kXStride);
        uint32_t P[F::kLaneK / 2];
#pragma unroll
        for (int j = 0; j < F::kLaneK / 8; ++j) {
          const uint4 v = src[j];
          P[4 * j] = v.x;
          P[4 * j + 1] = v.y;
          P[4 * j + 2] = v.z;
          P[4 * j + 3] = v.w;
        }
        float ps = 0.0f;  // sum of this lane's activations in the sub-chunk (fixed order)
#pragma unroll
        for (int j = 0; j < F::kLaneK / 2; ++j) {
          const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&P[j]));
          ps += f2.x + f2.y;
        }
#pragma unroll
        for (int f = 0; f < F::kFragU4; ++f) {
          uint32_t Pa, Pb, Pc, Pd;
          if (!kInt4) {  // f = h*4 + pp: positions p = 2pp (even), 2pp+1 (odd) of word pair h
            const int h = f >> 2, pp = f & 3;
            Pa = P[16 * h + pp];
            Pb = P[16 * h + 4 + pp];
            Pc = P[16 * h + 8 + pp];
            Pd = P[16 * h + 12 + pp];
          } else {       // f = h*2 + s: nibble positions 2s (class 0), 2s+1 (class 1)
            const int h = f >> 1, s2 = f & 1;
            Pa = P[8 * h + s2];
            Pb = P[8 * h + 2 + s2];
            Pc = P[8 * h + 4 + s2];
            Pd = P[8 * h + 6 + s2];
          }
          const uint32_t e01 = __byte_perm(Pa, Pb, 0x5410), e23 = __byte_perm(Pc, Pd, 0x5410);
          uint32_t o01 = __byte_perm(Pa, Pb, 0x7632), o23 = __byte_perm(Pc, Pd, 0x7632);
          __half2 so01 = __hmul2(*reinterpret_cast<__half2*>(&o01), fold);
          __half2 so23 = __hmul2(*reinterpret_cast<__half2*>(&o23), fold);
          xfs[((sub * NT + T) * F::kFragU4 + f) * 32 + lane] =
              make_uint4(e01, e23, *reinterpret_cast<uint32_t*>(&so01), *reinterpret_cast<uint32_t*>(&so23));
        }
        ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 1);  // the four lanes of one token
        ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 2);
        if (kInt4) {
          if (t == 0) xg[(xslot * 2 + sub) * 16 + 8 * T + g] = ps;
        } else {
          sxl[T] += ps;
        }
      }
      mbar_arrive(&xfull[xslot]);
      issue_x(i + 2);
    }
    cp_async_wait<0>();
    if (!kInt4 && t == 0) {
#pragma unroll
      for (int T = 0; T < NT; ++T) sxb[sub * 16 + 8 * T + g] = sxl[T];
    }
  } else {
    // ================================================================== consumer warps
    constexpr int NG = kInt4 ? 1 : 4;  // accumulator groups: one per position pair (chains)
    float acc[NG][kDRT][NT][4];
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
        for (int T = 0; T < NT; ++T)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[q][rt][T][c] = 0.0f;
    const int64_t G = a.K >> 7;
    pdl_wait_prior_grids();  // block (not poll) until the activations can exist
    for (int i = 0; i < nst; ++i) {
      const int ws = i % a.ring, xslot = i & 1;
      if (!mbar_wait(&wfull[ws], static_cast<uint32_t>(i / a.ring) & 1u) ||
          !mbar_wait(&xfull[xslot], static_cast<uint32_t>(i >> 1) & 1u))
        break;
      const uint8_t* st = wst + ws * kDStageBytes;
      const uint4* xfs = reinterpret_cast<const uint4*>(xf + xslot * L::kXfStage);
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        const int chunk = sub * 4 + t;
        uint32_t w0[kDRT][4], w1[kDRT][4];
#pragma unroll
        for (int rt = 0; rt < kDRT; ++rt) {
          const int r0 = warp * (16 * kDRT) + rt * 16 + g, r1 = r0 + 8;
          const uint4 U0 = *reinterpret_cast<const uint4*>(st + r0 * 128 + ((chunk ^ (r0 & 7)) << 4));
          const uint4 U1 = *reinterpret_cast<const uint4*>(st + r1 * 128 + ((chunk ^ (r1 & 7)) << 4));
          w0[rt][0] = U0.x; w0[rt][1] = U0.y; w0[rt][2] = U0.z; w0[rt][3] = U0.w;
          w1[rt][0] = U1.x; w1[rt][1] = U1.y; w1[rt][2] = U1.z; w1[rt][3] = U1.w;
        }
        if (!kInt4) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t sh[kDRT][4];
#pragma unroll
            for (int rt = 0; rt < kDRT; ++rt) {
              sh[rt][0] = w0[rt][2 * h] >> 12;
              sh[rt][1] = w1[rt][2 * h] >> 12;
              sh[rt][2] = w0[rt][2 * h + 1] >> 12;
              sh[rt][3] = w1[rt][2 * h + 1] >> 12;
            }
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
              uint4 B[NT];
#pragma unroll
              for (int T = 0; T < NT; ++T) B[T] = xfs[((sub * NT + T) * 8 + h * 4 + pp) * 32 + lane];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const int p = 2 * pp + q;
#pragma unroll
                for (int rt = 0; rt < kDRT; ++rt) {
                  uint32_t a0, a1, a2, a3;
                  if (p < 6) {
                    const uint32_t mk = 0x00030003u << (2 * p);
                    a0 = w0[rt][2 * h] & mk;
                    a1 = w1[rt][2 * h] & mk;
                    a2 = w0[rt][2 * h + 1] & mk;
                    a3 = w1[rt][2 * h + 1] & mk;
                  } else {
                    const uint32_t mk = (p == 6) ? 0x00030003u : 0x000C000Cu;
                    a0 = sh[rt][0] & mk;
                    a1 = sh[rt][1] & mk;
                    a2 = sh[rt][2] & mk;
                    a3 = sh[rt][3] & mk;
                  }
#pragma unroll
                  for (int T = 0; T < NT; ++T)
                    mma_16816(acc[pp % NG][rt][T], a0, a1, a2, a3, q ? B[T].z : B[T].x, q ? B[T].w : B[T].y);
                }
              }
            }
          }
        } else {
          const int64_t gi = static_cast<int64_t>(st_begin + i) * 2 + sub;
          float xgt[NT][2];
#pragma unroll
          for (int T = 0; T < NT; ++T) {
            xgt[T][0] = 8.0f * xg[(xslot * 2 + sub) * 16 + 8 * T + 2 * t];
            xgt[T][1] = 8.0f * xg[(xslot * 2 + sub) * 16 + 8 * T + 2 * t + 1];
          }
#pragma unroll
          for (int rt = 0; rt < kDRT; ++rt) {
            float cg[2][NT][4];  // two chains (class 0 / class 1 fields)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
              for (int T = 0; T < NT; ++T)
#pragma unroll
                for (int c = 0; c < 4; ++c) cg[j][T][c] = 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int s2 = 0; s2 < 2; ++s2) {
                const uint32_t x0 = w0[rt][2 * h] >> (8 * s2), x1 = w1[rt][2 * h] >> (8 * s2);
                const uint32_t x2 = w0[rt][2 * h + 1] >> (8 * s2), x3 = w1[rt][2 * h + 1] >> (8 * s2);
                uint4 B[NT];
#pragma unroll
                for (int T = 0; T < NT; ++T) B[T] = xfs[((sub * NT + T) * 4 + h * 2 + s2) * 32 + lane];
#pragma unroll
                for (int cls = 0; cls < 2; ++cls) {
                  const uint32_t mk = cls ? 0x00F000F0u : 0x000F000Fu;
#pragma unroll
                  for (int T = 0; T < NT; ++T)
                    mma_16816(cg[cls][T], x0 & mk, x1 & mk, x2 & mk, x3 & mk, cls ? B[T].z : B[T].x,
                              cls ? B[T].w : B[T].y);
                }
              }
            const int64_t n0 = static_cast<int64_t>(rb) * kDRows + warp * (16 * kDRT) + rt * 16 + g, n1 = n0 + 8;
            // groups past K (a zero-filled half stage) contribute nothing
            const float s0 = (n0 < Nm && gi < G) ? __half2float(scm[n0 * G + gi]) : 0.0f;
            const float s1 = (n1 < Nm && gi < G) ? __half2float(scm[n1 * G + gi]) : 0.0f;
#pragma unroll
            for (int T = 0; T < NT; ++T) {
              float c4[4];
#pragma unroll
              for (int c = 0; c < 4; ++c) c4[c] = cg[0][T][c] + cg[1][T][c];
              acc[0][rt][T][0] = fmaf(s0, fmaf(c4[0], 16777216.0f, -xgt[T][0]), acc[0][rt][T][0]);
              acc[0][rt][T][1] = fmaf(s0, fmaf(c4[1], 16777216.0f, -xgt[T][1]), acc[0][rt][T][1]);
              acc[0][rt][T][2] = fmaf(s1, fmaf(c4[2], 16777216.0f, -xgt[T][0]), acc[0][rt][T][2]);
              acc[0][rt][T][3] = fmaf(s1, fmaf(c4[3], 16777216.0f, -xgt[T][1]), acc[0][rt][T][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&wempty[ws]);
        mbar_arrive(&xempty[xslot]);
      }
    }
    // push this slice's partial results to the CTA that owns each row (the rows of the row block
    // are split evenly over the cluster: owner q holds rows [q*128/S, (q+1)*128/S))
    const uint32_t red_local = smem_u32(red);
#pragma unroll
    for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = warp * (16 * kDRT) + rt * 16 + g + 8 * hr;
        const int q = (r * a.S + a.S - 1) / kDRows;
        const int slot = r - (q * kDRows) / a.S;
        const uint32_t dst = mapa_shared(red_local + ((rank * own_cap + slot) * 16) * 4, static_cast<uint32_t>(q));
#pragma unroll
        for (int T = 0; T < NT; ++T)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int ci = 2 * hr + c;
            float v;
            // factors 2^-24 (pairs 0 and 3), 2^-20 (pair 1), 2^-16 (pair 2): exact rescaling
            if (!kInt4)
              v = fmaf(acc[0][rt][T][ci] + acc[NG - 1][rt][T][ci], 16777216.0f,
                       fmaf(acc[1 % NG][rt][T][ci], 1048576.0f, acc[2 % NG][rt][T][ci] * 65536.0f));
            else
              v = acc[0][rt][T][ci];
            st_shared_cluster_f32(dst + (8 * T + 2 * t + c) * 4, v);
          }
      }
  }

  // ==================================================================== cluster reduction
  __syncthreads();  // the builders' sums of x are in shared memory
  if (!kInt4 && threadIdx.x < 16) {  // push this slice's token sums of x to every owner
    const float sx = sxb[threadIdx.x] + sxb[16 + threadIdx.x];
    const uint32_t loc = smem_u32(sxr + rank * 16 + threadIdx.x);
    for (int q = 0; q < a.S; ++q) st_shared_cluster_f32(mapa_shared(loc, q), sx);
  }
  cluster_sync_all();  // every partial and slice sum has landed in its owner's shared memory
  pdl_wait_prior_grids();
  {
    const int rr0 = (rank * kDRows) / a.S, rr1 = ((rank + 1) * kDRows) / a.S;
    const int nrows = rr1 - rr0;
    const int Mv = static_cast<int>(a.M < 8 * NT ? a.M : 8 * NT);
    for (int idx = threadIdx.x; idx < nrows * Mv; idx += kDThreads) {
      const int m = idx / nrows, slot = idx - m * nrows;
      const int64_t n = static_cast<int64_t>(rb) * kDRows + rr0 + slot;
      if (n >= Nm) continue;
      float v = 0.0f, sx = 0.0f;
      for (int q = 0; q < a.S; ++q) {  // fixed order: deterministic
        v += red[(q * own_cap + slot) * 16 + m];
        if (!kInt4) sx += sxr[q * 16 + m];
      }
      if (!kInt4) v = (v - sx) * __half2float(scm[n]);
      if (biasm) v += __half2float(biasm[n]);
      ym[m * Nm + n] = __float2half_rn(v);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
struct DecodePlan {
  int S, C, ring, smem;
};

template <bool kInt4, int NT>
static bool plan_decode_t(int64_t RB, int64_t K, int num_sms, DecodePlan* p) {
  using F = DecFmt<kInt4>;
  const int C = static_cast<int>((K + F::kStageK - 1) / F::kStageK);
  // weight ring: every stage of the CTA's slice if it fits (then the whole slice is in flight
  // before griddepcontrol.wait), else as many as two CTAs per SM allow
  int ring = kDMaxRing;
  while (ring > 2 && DecLayout<kInt4, NT>::bytes(ring) > kDSmemBudget) --ring;
  const int smem = DecLayout<kInt4, NT>::bytes(ring);
  if (smem > 227 * 1024) return false;
  // one wave of two CTAs per SM, at most 8 K-slices per row block
  int64_t S = (2 * static_cast<int64_t>(num_sms)) / RB;
  if (S < 1) S = 1;
  if (S > kDMaxCluster) S = kDMaxCluster;
  if (S > C) S = C;
  *p = DecodePlan{static_cast<int>(S), C, ring, smem};
  return true;
}

static bool plan_decode(bool int4, int NT, int64_t RB, int64_t K, int num_sms, DecodePlan* p) {
  if (int4) return NT == 1 ? plan_decode_t<true, 1>(RB, K, num_sms, p) : plan_decode_t<true, 2>(RB, K, num_sms, p);
  return NT == 1 ? plan_decode_t<false, 1>(RB, K, num_sms, p) : plan_decode_t<false, 2>(RB, K, num_sms, p);
}

template <bool kInt4, int NT>
static cudaError_t launch_decode_t(const DecodeMaps& maps, const DecodeArgs& a, const DecodePlan& p,
                                   cudaStream_t s) {
  auto* kern = decode_gemm_kernel<kInt4, NT>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), p.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.S), static_cast<unsigned>(a.rb_start[a.count]), 1);
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
  return cudaLaunchKernelEx(&cfg, kern, maps, a);
}

// One launch for `count` matrices that share x (same M and K): y_g = x . What_g^T (+ bias_g).
template <bool kInt4>
static cudaError_t launch_decode_group(const __half* x, int count, const void* const* w,
                                       const __half* const* sc, const __half* const* bias,
                                       __half* const* y, const int64_t* N, int64_t M, int64_t K,
                                       cudaStream_t s) {
  if (count < 1 || count > kDMaxGroup) return cudaErrorInvalidValue;
  const DeviceInfo di = current_device_info();
  const int NT = M > 8 ? 2 : 1;
  DecodeArgs a = {};
  DecodeMaps maps;
  a.x = x;
  a.M = M;
  a.K = K;
  a.count = count;
  int64_t rbs = 0;
  const int64_t kbytes = kInt4 ? K / 2 : K / 4;
  for (int g = 0; g < count; ++g) {
    a.rb_start[g] = static_cast<int>(rbs);
    rbs += (N[g] + kDRows - 1) / kDRows;
    a.N[g] = N[g];
    a.sc[g] = sc[g];
    a.bias[g] = bias ? bias[g] : nullptr;
    a.y[g] = y[g];
    if (!make_tmap_2d(&maps.m[g], CU_TENSOR_MAP_DATA_TYPE_UINT8, w[g], static_cast<uint64_t>(kbytes),
                      static_cast<uint64_t>(N[g]), static_cast<uint64_t>(kbytes), 128, kDRows,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  for (int g = count; g < kDMaxGroup; ++g) maps.m[g] = maps.m[0];
  a.rb_start[count] = static_cast<int>(rbs);
  if (rbs > 65535) return cudaErrorInvalidValue;
  DecodePlan p;
  if (!plan_decode(kInt4, NT, rbs, K, di.num_sms, &p)) return cudaErrorInvalidValue;
  a.C = p.C;
  a.S = p.S;
  a.ring = p.ring;
  return NT == 1 ? launch_decode_t<kInt4, 1>(maps, a, p, s) : launch_decode_t<kInt4, 2>(maps, a, p, s);
}

bool decode_supported(bool int4, int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > 16 || N < 1) return false;
  if (int4 ? (K % 128 != 0) : (K % 64 != 0)) return false;
  DecodePlan p;
  return plan_decode(int4, M > 8 ? 2 : 1, (N + kDRows - 1) / kDRows, K, 148, &p);
}

cudaError_t launch_tq_gemm_decode(const __half* x, const uint8_t* packed, const __half* scale,
                                  const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                  cudaStream_t s) {
  const void* w = packed;
  return launch_decode_group<false>(x, 1, &w, &scale, &bias, &y, &N, M, K, s);
}

cudaError_t launch_w4g_gemm_decode(const __half* x, const int32_t* qweight, const __half* scales,
                                   const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                   cudaStream_t s) {
  const void* w = qweight;
  return launch_decode_group<true>(x, 1, &w, &scales, &bias, &y, &N, M, K, s);
}

cudaError_t launch_tq_gemm_decode_group(const __half* x, int count, const uint8_t* const* packed,
                                        const __half* const* scale, const __half* const* bias,
                                        __half* const* y, const int64_t* N, int64_t M, int64_t K,
                                        cudaStream_t s) {
  const void* w[kDMaxGroup];
  for (int g = 0; g < count && g < kDMaxGroup; ++g) w[g] = packed[g];
  return launch_decode_group<false>(x, count, w, scale, bias, y, N, M, K, s);
}

cudaError_t launch_w4g_gemm_decode_group(const __half* x, int count, const int32_t* const* qweight,
                                         const __half* const* scales, const __half* const* bias,
                                         __half* const* y, const int64_t* N, int64_t M, int64_t K,
                                         cudaStream_t s) {
  const void* w[kDMaxGroup];
  for (int g = 0; g < count && g < kDMaxGroup; ++g) w[g] = qweight[g];
  return launch_decode_group<true>(x, count, w, scales, bias, y, N, M, K, s);
}

}  // namespace tq
