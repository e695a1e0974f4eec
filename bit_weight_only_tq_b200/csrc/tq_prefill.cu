// tq_prefill.cu -- tensor-core GEMM for large M (prefill), ternary and W4A16 weights.
//
// This path is a dense contraction, so it runs on the 5th-generation tensor cores.  [TQ] §4.2-4.3
// (prior art): decode the codes into fp16 tensor-core operands, accumulate in fp32, apply the
// per-row scale after the MMA.  On sm_100a the decoded weights never touch shared memory: they
// are the A operand of tcgen05.mma, written straight into tensor memory, and the activations are
// the B operand:
//   D[n, m] (TMEM, fp32) += A[n, k] (TMEM, fp16 decoded weights) * B[m, k]^T (smem, x tile)
// One CTA = 128 weight rows (the TMEM lanes, UMMA M) x TN tokens (UMMA N = 256, or 128 for
// small M):
//   * warp 0, one lane: TMA loads of the x tile (TN tokens x 64 k, fp16, 128-byte swizzle, the
//     K-major layout the UMMA descriptor expects) into a ring; warp 2, one lane: TMA loads of the
//     packed weights, 128 rows x 128 bytes per tile (8 ternary / 4 W4A16 stages, 128-byte
//     swizzle) into a ring of three;
//   * warp 1: allocates the tensor memory (accumulator + a ring of decoded-weight slots); one
//     lane issues tcgen05.mma (M=128, N=TN, K=16, A from tensor memory) and commits to
//     mbarriers that free the input stages;
//   * warps 4-11, two groups of four taking alternate stages (thread r % 128 = weight row r =
//     TMEM lane r): decode the packed row into 32 fp16x2 registers in natural k order and store
//     them with one tcgen05.st per stage;
//       ternary: (c - 1) is exact in fp16; the row scale is applied in the epilogue;
//       W4A16:   fp16(q * s[n, k/128]) (one rounding, <= 2^-11 relative);
//   * the epilogue, all twelve warps in three groups of four taking 32-token chunks in turn:
//     tcgen05.ld 32 tokens of a row at a time, scale / bias, fp16, staged through shared memory
//     for coalesced 16-byte stores of y.
// Shared-memory traffic per MMA is the x tile only (read by the MMA, written by TMA); decoding
// into shared memory would add the weight tile twice (written, then read).
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

#include <atomic>

#include "tq_common.cuh"

namespace tq {

constexpr int kQM = 128;         // weight rows per CTA (UMMA M, TMEM lanes)
constexpr int kQK = 64;          // K per stage: one 128-byte swizzle row of fp16
constexpr int kQMaxRing = 12;    // stages of (x tile, packed tile), at most
constexpr int kQMaxARing = 8;    // tensor-memory slots of decoded weights (32 columns each)
constexpr int kQDecGroups = 2;   // groups of four decode warps, taking alternate stages
constexpr int kQThreads = 128 * (1 + kQDecGroups);  // warps 0-3: TMA, MMA; then the decode groups
constexpr int kQEpiGroups = 1 + kQDecGroups;        // every group of four warps runs the epilogue
constexpr bool kMergeStageBarriers = true;

// kKS: K per stage, 64 (one 128-byte swizzle row of fp16 per operand row) or 128 (two of them,
// eight MMAs per barrier test and commit instead of four)
template <bool kInt4, int kKS>
struct PFmt {
  static constexpr int kSub = kKS / kQK;                       // 64-k sub-tiles per stage
  static constexpr int kRowBytes = (kInt4 ? 32 : 16) * kSub;  // packed bytes per row per stage
  // the packed weights arrive in tiles of 128 bytes per row (512 ternary / 256 W4A16 k),
  // 128-byte swizzled: one DRAM burst per row instead of one small piece per stage
  static constexpr int kSPP = 128 / kRowBytes;                 // stages per packed tile
  static constexpr int kTileP = kQM * 128;
  static constexpr int kPRing = 3;
  static_assert(kSPP % kQDecGroups == 0, "the decode groups alternate within a packed tile");
};

// kSS: the decoded weights go to shared memory (128-byte-swizzled K-major tiles, the layout TMA
// gives the x tile) and the MMA reads both operands from there; otherwise they go to tensor
// memory.
template <bool kInt4, int TN, bool kSS, int kKS>
struct PrefillLayout {
  static_assert(kSS || kKS == kQK, "tensor-memory A slots hold 64 k");
  static constexpr int kSub = kKS / kQK;
  static constexpr int kTileXs = TN * kQK * 2;   // x sub-tile: TN rows x 128 bytes
  static constexpr int kTileAs = kQM * kQK * 2;  // decoded-weight sub-tile (kSS): 128 rows x 128 bytes
  static constexpr int kTileX = kSub * kTileXs;  // x tile of one stage
  static constexpr int kTileA = kSub * kTileAs;  // decoded-weight tile of one stage (kSS)
  // ring depths: narrow tiles move little data per stage, so they keep more stages in flight
  static constexpr int kRing = kSS ? (kSub == 2 ? (TN == 64 ? 3 : 2) : (TN == 64 ? 6 : 4))
                                   : (TN == 256 ? 4 : (TN == 128 ? 6 : 10));
  static constexpr int kARing = kSS ? kRing : (TN == 256 ? 4 : kQMaxARing);
  // equal rings: one barrier per stage for "x tile landed and weights decoded" and one for
  // "stage consumed", so the MMA thread tests one barrier and commits once per stage
  static constexpr bool kMergedBars = kMergeStageBarriers && kRing == kARing;
  static constexpr int kOffX = 0;
  static constexpr int kOffP = kOffX + kRing * kTileX;
  static constexpr int kOffA = kOffP + PFmt<kInt4, kKS>::kPRing * PFmt<kInt4, kKS>::kTileP;
  static constexpr int kOffBar = kOffA + (kSS ? kARing * kTileA : 0);
  // barriers: fullX[R], emptyX[R], fullP[RP], emptyP[RP], afull[RA], aempty[RA], accFull; then
  // the TMEM slot
  static constexpr int kNumBars = 2 * kRing + 2 * PFmt<kInt4, kKS>::kPRing + 2 * kARing + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffTmemSlot + 16;
  // alignment slack; at least 116 KB so that one CTA runs per SM: a CTA never waits in
  // tcgen05.alloc for tensor memory held by another CTA (which may itself wait at a cluster
  // barrier for a CTA that waits for tensor memory)
  static constexpr int kAlloc = kBytes + 1024 > 116 * 1024 ? kBytes + 1024 : 116 * 1024;
  // split-K partials [S][TN / S / 4][128 rows][4] fp32 reuse the x and packed rings after the
  // main loop
  static_assert(kQM * (TN + 8) * 4 <= kRing * kTileX + PFmt<kInt4, kKS>::kPRing * PFmt<kInt4, kKS>::kTileP,
                "split-K partials fit");
  // tensor memory: accumulator columns [0, TN), decoded-weight slots after it (not kSS)
  static constexpr uint32_t kColA = TN;
  static constexpr uint32_t kTmemCols = kSS ? static_cast<uint32_t>(TN) : (TN + 32 * kARing <= 256 ? 256u : 512u);
  // epilogue staging (reuses the x ring): one buffer of 32 tokens x 128 rows fp16 per group
  static_assert(kQEpiGroups * 32 * kQM * 2 <= kRing * kTileX, "staging fits in the x ring");
  static_assert(kRing <= kQMaxRing && kARing <= kQMaxARing && (kSS || TN + 32 * kARing <= 512), "rings");
  static_assert(kAlloc <= 227 * 1024, "shared memory");
};

// One launch covers up to kQMaxGroup matrices that share x (a serving engine's fused q/k/v or
// gate/up): grid x runs over the row tiles of all of them, matrix g owning tiles
// [tile0[g], tile0[g + 1]).
constexpr int kQMaxGroup = 4;

struct PrefillArgs {
  const __half* sc[kQMaxGroup];    // ternary: scale[N]; W4A16: scales[N, K/128]
  const uint8_t* zp[kQMaxGroup];   // W4A16 zero-points [N, K/128], or null (symmetric)
  const __half* bias[kQMaxGroup];  // may be null
  __half* y[kQMaxGroup];
  int64_t N[kQMaxGroup];
  int64_t ldy[kQMaxGroup];         // y row stride (elements): N, or more for a block of y's columns
  int tile0[kQMaxGroup + 1];
  int count;
  int64_t M, K;
  int S;               // K-slices: CTAs per cluster (grid z), reduced through DSMEM
};

struct PrefillWeightMaps {
  CUtensorMap m[kQMaxGroup];  // packed weights of each matrix
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

// The fp16 pair (1024 + z, 64 + z) that decode_w4_8 subtracts for zero-point z (0..15): 1024 + z
// has unit 1, 64 + z unit 1/16, so both are exact patterns.  z = 8 is the symmetric format.
__device__ __forceinline__ uint32_t w4_zero_pair(uint32_t z) { return ((0x5400u + 16u * z) << 16) | (0x6400u + z); }

// 8 consecutive INT4 codes (one int32 word) -> 8 fp16 (u - z) * s, s2 = (s, s), zsub =
// w4_zero_pair(z).
__device__ __forceinline__ uint4 decode_w4_8(uint32_t w, uint32_t s2, uint32_t zsub) {
  uint32_t o[4];
#pragma unroll
  for (int bi = 0; bi < 4; ++bi) {
    const uint32_t t = byte_to_halves(w, bi);
    // low nibble -> 1024 + u (0x6400 base), high nibble -> 64 + u (0x5400 base, bits 4-7)
    const uint32_t h = (t & 0x00F0000Fu) | 0x54006400u;
    o[bi] = hmul2_u32(hsub2_u32(h, zsub), s2);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <bool kInt4, int TN, bool kSS, int kKS>
__global__ void __launch_bounds__(kQThreads, 1)
    prefill_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ PrefillWeightMaps tmaps_w, const PrefillArgs a) {
  using L = PrefillLayout<kInt4, TN, kSS, kKS>;
  using F = PFmt<kInt4, kKS>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned; pointer arithmetic on the __shared__ array keeps the shared address
  // space visible to the compiler (plain ld/st.shared instead of generic accesses)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
  uint64_t* full = bars;                       // x tile landed (TMA)
  uint64_t* emptyX = bars + L::kRing;          // x tile consumed (MMA commit)
  uint64_t* fullP = bars + 2 * L::kRing;       // packed tile landed (TMA)
  uint64_t* emptyP = fullP + F::kPRing;        // packed tile consumed (decode warps)
  // decoded weights written / consumed (MMA commit); with merged barriers the same barriers as
  // the x tile's (stage s of both rings), `full` then also counts the four decode warps
  uint64_t* afull = L::kMergedBars ? full : emptyP + F::kPRing;
  uint64_t* aempty = L::kMergedBars ? emptyX : emptyP + F::kPRing + L::kARing;
  uint64_t* accFull = emptyP + F::kPRing + 2 * L::kARing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kOffTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int g = 0;  // matrix of this row tile
  while (g + 1 < a.count && static_cast<int>(blockIdx.x) >= a.tile0[g + 1]) ++g;
  const int64_t n0 = static_cast<int64_t>(static_cast<int>(blockIdx.x) - a.tile0[g]) * kQM;  // first weight row
  const int64_t Ng = a.N[g];
  const __half* const gsc = a.sc[g];
  const uint8_t* const gzp = a.zp[g];
  const __half* const gbias = a.bias[g];
  __half* const gy = a.y[g];
  const int64_t gldy = a.ldy[g];
  const CUtensorMap* const tmap_w = &tmaps_w.m[g];
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * TN;   // first token
  const int nk_all = static_cast<int>((a.K + kKS - 1) / kKS);  // a last half stage reads zeros
  const int rank = static_cast<int>(blockIdx.z);              // K-slice = rank in the cluster
  const int kb0 = static_cast<int>((static_cast<int64_t>(rank) * nk_all) / a.S);
  const int nk = static_cast<int>((static_cast<int64_t>(rank + 1) * nk_all) / a.S) - kb0;  // >= 1
  const int64_t G = a.K >> 7;

  pdl_allow_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kRing; ++i) {
      mbar_init(&full[i], L::kMergedBars ? 5 : 1);
      mbar_init(&emptyX[i], 1);
    }
    for (int i = 0; i < F::kPRing; ++i) {
      mbar_init(&fullP[i], 1);
      mbar_init(&emptyP[i], 4 * kQDecGroups);
    }
    for (int i = 0; i < L::kARing && !L::kMergedBars; ++i) {
      mbar_init(&afull[i], 4);
      mbar_init(&aempty[i], 1);
    }
    mbar_init(accFull, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  bool acc_flag = false;  // decode warps: the accumulator is complete
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer: x
    pdl_wait_prior_grids();
    if (lane == 0) {
      tma_prefetch_desc(&tmap_x);
      const bool skipx = skip_x_loads();  // failure-path test hook: never set in normal use
      for (int kb = 0; kb < nk && ok && !skipx; ++kb) {
        const int s = kb % L::kRing;
        if (kb >= L::kRing) {
          ok = mbar_wait(&emptyX[s], static_cast<uint32_t>((kb / L::kRing) - 1) & 1u);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(&full[s], L::kTileX);
#pragma unroll
        for (int q = 0; q < L::kSub; ++q)
          tma_load_2d(sm + L::kOffX + s * L::kTileX + q * L::kTileXs, &tmap_x, &full[s], (kb0 + kb) * kKS + q * kQK,
                      static_cast<int32_t>(m0));
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------------ TMA producer: weights
    // (model constants: issued before the wait for the previous kernel)
    if (lane == 0) {
      tma_prefetch_desc(tmap_w);
      const int npt = (nk + F::kSPP - 1) / F::kSPP;
      for (int pt = 0; pt < npt && ok; ++pt) {
        const int s = pt % F::kPRing;
        if (pt >= F::kPRing) {
          ok = mbar_wait(&emptyP[s], static_cast<uint32_t>((pt / F::kPRing) - 1) & 1u);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(&fullP[s], F::kTileP);
        tma_load_2d(sm + L::kOffP + s * F::kTileP, tmap_w, &fullP[s], (kb0 + pt * F::kSPP) * F::kRowBytes,
                    static_cast<int32_t>(n0));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    pdl_wait_prior_grids();  // x arrives only after the previous kernel: block, do not poll
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kQM, TN);
      const uint32_t x_base = smem_u32(sm + L::kOffX);
      const uint32_t a_base = smem_u32(sm + L::kOffA);
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % L::kRing, as = kb % L::kARing;
        ok = mbar_wait(&full[s], static_cast<uint32_t>(kb / L::kRing) & 1u) &&
             (L::kMergedBars || mbar_wait(&afull[as], static_cast<uint32_t>(kb / L::kARing) & 1u));
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t a_tmem = tmem + L::kColA + 32 * as;
#pragma unroll
        for (int q = 0; q < L::kSub; ++q) {
          const uint64_t bdesc = sdesc_kmajor_sw128(x_base + s * L::kTileX + q * L::kTileXs);
          const uint64_t adesc = sdesc_kmajor_sw128(a_base + as * L::kTileA + q * L::kTileAs);
#pragma unroll
          for (int k16 = 0; k16 < kQK / 16; ++k16) {
            // A in tensor memory: 8 columns (16 fp16) per K=16 step; in shared memory (and B):
            // +32 bytes along K = +2 in the descriptor
            const uint32_t accum = (kb | q | k16) != 0 ? 1u : 0u;
            if (kSS)
              umma_f16(tmem, adesc + 2 * k16, bdesc + 2 * k16, idesc, accum);
            else
              umma_f16_ts(tmem, a_tmem + 8 * k16, bdesc + 2 * k16, idesc, accum);
          }
        }
        umma_commit(&emptyX[s]);
        if (!L::kMergedBars) umma_commit(&aempty[as]);
      }
      if (ok) umma_commit(accFull);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ decode warps
    // group dg decodes stages dg, dg + 2, ...: two warps per SM sub-partition hide each other's
    // waits and tensor-memory store latency
    const int dg = (warp >> 2) - 1;
    const int r = threadIdx.x & (kQM - 1);  // weight row within the tile = TMEM lane
    const int64_t n = n0 + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    // W4A16 group scales of this row: the next group's is loaded when a group starts, a stage
    // or two before it is needed, so the load latency stays off the decode
    auto group_scale = [&](int64_t gi) -> uint16_t {
      return (n < Ng && gi < G) ? __half_as_ushort(gsc[n * G + gi]) : static_cast<uint16_t>(0);
    };
    auto group_zero = [&](int64_t gi) -> uint32_t {
      return (gzp && n < Ng && gi < G) ? static_cast<uint32_t>(gzp[n * G + gi]) : 8u;
    };
    int64_t g_cur = -1, g_nxt = -1;
    uint16_t sc_cur = 0, sc_nxt = 0;
    uint32_t zp_cur = 8u, zp_nxt = 8u;
    for (int kb = dg; kb < nk && ok; kb += kQDecGroups) {
      const int as = kb % L::kARing, pt = kb / F::kSPP, ci = kb - pt * F::kSPP, ps = pt % F::kPRing;
      if (ci == dg) {  // this group's first stage of the packed tile (kSPP is even)
        ok = mbar_wait(&fullP[ps], static_cast<uint32_t>(pt / F::kPRing) & 1u);
        if (!ok) break;
      }
      // this stage's 16 (ternary) or 32 (W4A16) bytes per 64 k of row r: 16-byte chunks of the
      // 128-byte swizzled row (chunk c at position c ^ (r & 7): conflict free)
      constexpr int kCh = (kInt4 ? 2 : 1) * L::kSub;  // chunks per stage
      const uint8_t* prow = sm + L::kOffP + ps * F::kTileP + r * 128;
      uint4 pc[kCh];
#pragma unroll
      for (int c = 0; c < kCh; ++c)
        pc[c] = *reinterpret_cast<const uint4*>(prow + (((kCh * ci + c) ^ (r & 7)) << 4));
      // done with this packed tile: both groups arrive on every tile but a CTA's last, which
      // no later load waits for
      if (ci + kQDecGroups >= F::kSPP || kb + kQDecGroups >= nk) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&emptyP[ps]);
      }
      uint32_t s2 = 0u;
      if (kInt4) {
        const int64_t gi = (static_cast<int64_t>(kb0 + kb) * kKS) >> 7;  // 128-wide group of this stage
        if (gi != g_cur) {
          sc_cur = gi == g_nxt ? sc_nxt : group_scale(gi);
          zp_cur = gi == g_nxt ? zp_nxt : group_zero(gi);
          // the group of this decode group's next stage (kQDecGroups stages on)
          g_nxt = (static_cast<int64_t>(kb0 + kb + kQDecGroups) * kKS) >> 7;
          sc_nxt = group_scale(g_nxt);
          zp_nxt = group_zero(g_nxt);
          g_cur = gi;
        }
        s2 = static_cast<uint32_t>(sc_cur) | (static_cast<uint32_t>(sc_cur) << 16);
      }
      const uint32_t zsub = w4_zero_pair(zp_cur);
      // the packed words of 64-k sub-tile q
      auto words = [&](int q, uint32_t (&pw)[8]) {
        const uint4 u0 = pc[(kInt4 ? 2 : 1) * q];
        const uint4 u1 = kInt4 ? pc[2 * q + 1] : make_uint4(0u, 0u, 0u, 0u);
        pw[0] = u0.x;
        pw[1] = u0.y;
        pw[2] = u0.z;
        pw[3] = u0.w;
        pw[4] = u1.x;
        pw[5] = u1.y;
        pw[6] = u1.z;
        pw[7] = u1.w;
      };
      if (kSS) {
        if (kb >= L::kARing) {
          ok = mbar_wait(&aempty[as], static_cast<uint32_t>((kb / L::kARing) - 1) & 1u);
          if (!ok) break;
        }
        // 16-byte chunk j (k = 8j .. 8j + 7) of row r at chunk position j ^ (r & 7) of the
        // 128-byte row: the 128-byte swizzle; eight consecutive rows fill all 32 banks
#pragma unroll
        for (int q = 0; q < L::kSub; ++q) {
          uint32_t pw[8];
          words(q, pw);
          uint8_t* arow = sm + L::kOffA + as * L::kTileA + q * L::kTileAs + r * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 d = kInt4 ? decode_w4_8(pw[j], s2, zsub) : decode_tq_8(pw[j >> 1], j & 1);
            *reinterpret_cast<uint4*>(arow + ((j ^ (r & 7)) << 4)) = d;
          }
        }
        fence_proxy_async_smem();  // visible to the tensor core's operand reads
      } else {
        uint32_t pw[8];
        words(0, pw);
        uint32_t v[32];  // column j = fp16 pair (k = 2j, 2j + 1) of this row
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 d = kInt4 ? decode_w4_8(pw[j], s2, zsub) : decode_tq_8(pw[j >> 1], j & 1);
          v[4 * j] = d.x;
          v[4 * j + 1] = d.y;
          v[4 * j + 2] = d.z;
          v[4 * j + 3] = d.w;
        }
        if (kb >= L::kARing) {
          ok = mbar_wait(&aempty[as], static_cast<uint32_t>((kb / L::kARing) - 1) & 1u);
          if (!ok) break;
          tc_fence_after_sync();
        }
        tmem_st_32x32b_x32(lane_base + L::kColA + 32 * as, v);
        tmem_st_wait();
        tc_fence_before_sync();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[as]);
    }
    acc_flag = ok && mbar_wait(accFull, 0u);
  }

  // ------------------------------------------------------------------ epilogue (all warps)
  // The groups of four warps (the decode groups, then warps 0-3) take 32-token chunks of the
  // accumulator in turn; warp w reads tensor-memory lanes 32 (w % 4) .. + 31, i.e. weight row
  // r = threadIdx.x % 128.  The decode warps saw the accumulator complete (or the wait run out).
  if (threadIdx.x == 128) tmem_slot[1] = acc_flag ? 1u : 0u;
  pdl_wait_prior_grids();  // y may still be read by the previous kernel
  __syncwarp();            // the single-lane producer and MMA loops have ended
  named_barrier_sync(1 + kQEpiGroups, kQThreads);
  const bool acc_ok = tmem_slot[1] != 0u;
  tc_fence_after_sync();
  {
    const int grp = ((warp >> 2) + kQEpiGroups - 1) % kQEpiGroups;  // chunks grp, grp + kQEpiGroups, ...
    const int r = threadIdx.x & (kQM - 1);
    const int64_t n = n0 + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    float ep_s = 1.0f, ep_b = 0.0f;  // scale / bias of this row
    if (n < Ng) {
      if (!kInt4) ep_s = __half2float(gsc[n]);
      if (gbias) ep_b = __half2float(gbias[n]);
    }
    const bool vec = ((Ng | gldy) & 7) == 0 && (reinterpret_cast<uintptr_t>(gy) & 15u) == 0;
    // y[m0 + t0 + t, n0 + 0..127] for t < cnt (<= 32) from a staging buffer [cnt][128 rows]
    // fp16 of this group (named barrier 1 + grp): 16 chunks of 16 bytes per token, four per
    // thread, then the buffer is free again
    auto store_staged = [&](const __half* stage, int t0, int cnt) {
      named_barrier_sync(1 + grp, 128);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int idx = r + 128 * q, tok = idx >> 4, ch = idx & 15;
        const int64_t m = m0 + t0 + tok, nb = n0 + ch * 8;
        if (tok < cnt && m < a.M && nb < Ng) {
          const uint4 val = *reinterpret_cast<const uint4*>(stage + tok * kQM + ch * 8);
          __half* dst = gy + m * gldy + nb;
          if (vec && nb + 8 <= Ng) {
            *reinterpret_cast<uint4*>(dst) = val;
          } else {
            const __half* hv = reinterpret_cast<const __half*>(&val);
            for (int e = 0; e < 8 && nb + e < Ng; ++e) dst[e] = hv[e];
          }
        }
      }
      named_barrier_sync(1 + grp, 128);
    };
    auto out_h = [&](float v) { return __float2half_rn(kInt4 ? v + ep_b : fmaf(v, ep_s, ep_b)); };
    auto load_chunk = [&](int c, uint32_t (&rr)[32]) {
      if (acc_ok) {
        tmem_ld_32x32b_x32(lane_base + c * 32, rr);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) rr[j] = 0u;
      }
    };
    if (a.S == 1) {
      __half* stage = reinterpret_cast<__half*>(sm + L::kOffX) + grp * 32 * kQM;  // [32 tokens][128 rows]
#pragma unroll 1
      for (int c = grp; c < TN / 32 && acc_ok; c += kQEpiGroups) {
        uint32_t rr[32];
        load_chunk(c, rr);
#pragma unroll
        for (int j = 0; j < 32; ++j) stage[j * kQM + r] = out_h(__uint_as_float(rr[j]));
        store_staged(stage, c * 32, 32);
      }
    } else {
      // split K: the tokens of the tile are split evenly over the S CTAs of the cluster (tpo =
      // TN / S each, a multiple of 8).  Each CTA sends its partial sums of the other CTAs'
      // tokens into their shared memory, laid out [source rank][token / 4][row][token % 4] fp32
      // in the freed x and packed rings: one 16-byte store per thread of four tokens of its row,
      // 512 contiguous bytes per warp.  Its own tokens stay in tensor memory; it adds the S
      // partials of each of them in rank order (the same order on every run) and writes y
      // through staging buffers in the slot of its own rank (no CTA writes there).
      const int tpo = TN / a.S, own0 = rank * tpo, own1 = own0 + tpo;
      float* red = reinterpret_cast<float*>(sm + L::kOffX);
      const uint32_t red_local = smem_u32(red);
      auto slot = [&](int src, int tl) { return ((src * (tpo >> 2) + (tl >> 2)) * kQM + r) * 4; };  // floats
      cluster_sync_all();  // every CTA of the cluster is past its main loop: the x rings are free
#pragma unroll 1
      for (int c = grp; c < TN / 32; c += kQEpiGroups) {
        if (c * 32 >= own0 && c * 32 + 32 <= own1) continue;  // all 32 tokens are this CTA's
        uint32_t rr[32];
        load_chunk(c, rr);
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const int tok = c * 32 + j, q = tok / tpo;  // four consecutive tokens share an owner
          if (q != rank) {
            const uint32_t dst = red_local + 4u * static_cast<uint32_t>(slot(rank, tok - q * tpo));
            st_shared_cluster_v4_f32(mapa_shared(dst, static_cast<uint32_t>(q)), rr[j], rr[j + 1], rr[j + 2],
                                     rr[j + 3]);
          }
        }
      }
      cluster_sync_all();  // all partials have landed
      // own chunks go to the groups in turn; group g's staging buffer (8 KB at 8 g KB) is used
      // only when there are more than g own chunks (tpo > 32 g: the own slot holds 16 g KB or more)
      const int oc0 = own0 / 32;
      __half* stage = reinterpret_cast<__half*>(red + static_cast<size_t>(own0) * kQM) + grp * 32 * kQM;
#pragma unroll 1
      for (int c = oc0 + grp; c * 32 < own1; c += kQEpiGroups) {
        const int b0 = max(c * 32, own0), b1 = min(c * 32 + 32, own1);  // own tokens of chunk c
        uint32_t rr[32];
        load_chunk(c, rr);
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.0f;
        for (int src = 0; src < a.S; ++src) {
          if (src == rank) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += __uint_as_float(rr[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const int tok = c * 32 + j;
              if (tok >= b0 && tok < b1) {
                const float4 p = *reinterpret_cast<const float4*>(red + slot(src, tok - own0));
                v[j] += p.x;
                v[j + 1] += p.y;
                v[j + 2] += p.z;
                v[j + 3] += p.w;
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int tok = c * 32 + j;
          if (tok >= b0 && tok < b1) stage[(tok - b0) * kQM + r] = out_h(v[j]);
        }
        store_staged(stage, b0, b1 - b0);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

bool prefill_supported(bool int4, int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1) return false;
  if (K < kQK) return false;
  if (int4 ? (K % 128 != 0) : (K % 64 != 0)) return false;
  if ((M + 127) / 128 > 65535) return false;
  return true;
}

// The matrices of one launch (all read the same x[M, K]).
struct PrefillProblem {
  int count;
  const void* w[kQMaxGroup];
  const __half* sc[kQMaxGroup];
  const uint8_t* zp[kQMaxGroup];
  const __half* bias[kQMaxGroup];
  __half* y[kQMaxGroup];
  int64_t N[kQMaxGroup];
  int64_t ldy[kQMaxGroup];  // 0: N
};

template <bool kInt4, int TN, bool kSS, int kKS>
static cudaError_t launch_prefill_t(const __half* x, const PrefillProblem& pb, int64_t M, int64_t K, int S,
                                    cudaStream_t s) {
  using L = PrefillLayout<kInt4, TN, kSS, kKS>;
  CUtensorMap tx;
  PrefillWeightMaps tw;
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, static_cast<uint64_t>(K),
                    static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, kQK, TN,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const uint64_t kbytes = kInt4 ? static_cast<uint64_t>(K) / 2 : static_cast<uint64_t>(K) / 4;
  PrefillArgs a = {};
  a.count = pb.count;
  a.tile0[0] = 0;
  for (int g = 0; g < kQMaxGroup; ++g) {
    if (g < pb.count) {
      if (!make_tmap_2d(&tw.m[g], CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.w[g], kbytes, static_cast<uint64_t>(pb.N[g]),
                        kbytes, 128, kQM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
      a.sc[g] = pb.sc[g];
      a.zp[g] = pb.zp[g];
      a.bias[g] = pb.bias[g];
      a.y[g] = pb.y[g];
      a.N[g] = pb.N[g];
      a.ldy[g] = pb.ldy[g] > 0 ? pb.ldy[g] : pb.N[g];
      a.tile0[g + 1] = a.tile0[g] + static_cast<int>((pb.N[g] + kQM - 1) / kQM);
    } else {
      tw.m[g] = tw.m[0];
      a.tile0[g + 1] = a.tile0[g];
    }
  }
  auto* kern = prefill_gemm_kernel<kInt4, TN, kSS, kKS>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), L::kAlloc);
  if (e != cudaSuccess) return e;
  a.M = M;
  a.K = K;
  a.S = S;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.tile0[pb.count]), static_cast<unsigned>((M + TN - 1) / TN),
                     static_cast<unsigned>(S));
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int na = 1;
  if (S > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = static_cast<unsigned>(S);
    na = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, tx, tw, a);
}

// Clusters of S CTAs of this kernel that can be resident at once (a cluster's CTAs share one
// GPC, so the GPCs bound it below SMs / S), queried once per device and S; 0 when unknown.
constexpr int kPfMaxDevices = 64;

template <bool kInt4, int TN, bool kSS, int kKS>
static int prefill_cluster_capacity(int device, int S) {
  using L = PrefillLayout<kInt4, TN, kSS, kKS>;
  static std::atomic<int> cache[kPfMaxDevices][4];
  if (device < 0 || device >= kPfMaxDevices || S < 2 || S > 8) return 0;
  const int li = S == 2 ? 1 : (S == 4 ? 2 : 3);
  int n = cache[device][li].load(std::memory_order_relaxed);
  if (n > 0) return n;
  auto* kern = prefill_gemm_kernel<kInt4, TN, kSS, kKS>;
  if (ensure_smem_attr(reinterpret_cast<const void*>(kern), L::kAlloc) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, static_cast<unsigned>(S));
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kAlloc;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 1;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = static_cast<unsigned>(S);
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    return 0;
  }
  cache[device][li].store(n, std::memory_order_relaxed);
  return n;
}

// Tile choice: 64 tokens for M <= 64 (an N < 64 MMA costs as much as N = 64), 128 for M <= 128,
// else 256: a stage of 256 tokens takes about as long as one of 128 (the issuing thread, not the
// tensor pipe, sets the narrow tiles' stage time), so the wide tile does twice the work per SM
// and stage; K split over a cluster of S CTAs (1, 2, 4 or 8) while the tiles alone leave SMs
// idle and all the clusters fit on the GPU at once (a second wave of clusters costs more than
// the narrower split saves).
constexpr int kPrefillSSMaxTN = 128;  // token tiles up to this width read A from shared memory
constexpr int kPrefillSSStageK = 128;  // and take 128 k per stage (eight MMAs per barrier test)

static int prefill_tile_tokens(int64_t M) { return M <= 64 ? 64 : (M <= 128 ? 128 : 256); }

// One launch for several matrices fills the GPU when each alone would leave SMs idle or end in
// a part-empty wave; past a few waves each matrix's own launch keeps its weights' reuse across
// token tiles closer together in L2 (measured: W4A16 gate+up at M = 4096 4 % slower grouped).
bool prefill_grouping_pays(int64_t M, const int64_t* N, int count) {
  int64_t rt = 0;
  for (int g = 0; g < count; ++g) rt += (N[g] + kQM - 1) / kQM;
  const int TN = prefill_tile_tokens(M);
  return rt * ((M + TN - 1) / TN) <= 4 * static_cast<int64_t>(current_device_info().num_sms);
}

// Row tiles [r0, r1) of a problem (numbered matrix by matrix, as the grid runs over them) as a
// problem of its own: each matrix's part starts at its weights', scales', zeros', bias' and y's
// row offset, and y keeps its row stride.
template <bool kInt4>
static PrefillProblem sub_rows(const PrefillProblem& pb, int64_t K, int64_t r0, int64_t r1) {
  PrefillProblem out = {};
  const int64_t kbytes = kInt4 ? K / 2 : K / 4, G = K >> 7;
  int64_t t0 = 0;  // first row tile of matrix g
  for (int g = 0; g < pb.count; ++g) {
    const int64_t nt = (pb.N[g] + kQM - 1) / kQM;
    const int64_t lo = r0 > t0 ? r0 : t0, hi = r1 < t0 + nt ? r1 : t0 + nt;
    if (lo < hi) {
      const int64_t row = (lo - t0) * kQM, end = (hi - t0) * kQM < pb.N[g] ? (hi - t0) * kQM : pb.N[g];
      const int i = out.count++;
      out.w[i] = static_cast<const uint8_t*>(pb.w[g]) + row * kbytes;
      out.sc[i] = pb.sc[g] + (kInt4 ? row * G : row);
      out.zp[i] = pb.zp[g] ? pb.zp[g] + row * G : nullptr;
      out.bias[i] = pb.bias[g] ? pb.bias[g] + row : nullptr;
      out.y[i] = pb.y[g] + row;
      out.N[i] = end - row;
      out.ldy[i] = pb.ldy[g] > 0 ? pb.ldy[g] : pb.N[g];
    }
    t0 += nt;
  }
  return out;
}

// A launch whose tiles end in a part-empty wave (tiles = W waves + a few) leaves most SMs idle for
// a whole tile time.  Split instead: the row tiles that fill whole waves (of CTAs, with K split
// over Sm when that makes the waves come out whole) in one launch, the few row tiles left in a
// second launch with K split over a cluster of St, which then takes about 1 / St of a tile time.
// Cost model, in units of one full-K tile's time: a wave of CTAs that each take 1 / S of K costs
// 1 / S + 0.12 (a CTA's fixed prologue and epilogue, about 3 us against about 25 us for a tile
// of K = 4096) + 0.08 when S > 1 (the cluster's partial-sum exchange).
struct PrefillTailPlan {
  int64_t rows_main = 0;  // row tiles of the first launch; 0: no split
  int Sm = 1, St = 1;
};

template <typename Cap>
static PrefillTailPlan prefill_tail_plan(int64_t rt, int64_t TT, int nk, int sms, Cap capacity) {
  PrefillTailPlan best;
  const int64_t base = rt * TT;
  if (base <= sms) return best;
  auto waves_cost = [&](int64_t ctas, int S) {
    return static_cast<double>((ctas + sms - 1) / sms) * (1.0 / S + 0.12 + (S > 1 ? 0.08 : 0.0));
  };
  double best_cost = waves_cost(base, 1) * 0.92;  // a split must save 8 % by this model
  for (int Sm = 1; Sm <= 4; Sm *= 2) {
    if (Sm > nk || (Sm > 1 && capacity(Sm) <= 0)) break;
    const int64_t W = base * Sm / sms;  // whole waves of CTAs
    const int64_t rows_main = W * sms / (static_cast<int64_t>(Sm) * TT);
    if (rows_main <= 0 || rows_main >= rt) continue;
    const int64_t tail = (rt - rows_main) * TT;
    int St = 8;
    while (St > 1 && (tail * St > sms || St > nk || capacity(St) < tail)) St /= 2;
    const double cost = waves_cost(rows_main * TT * Sm, Sm) + waves_cost(tail * St, St);
    if (cost < best_cost) {
      best_cost = cost;
      best.rows_main = rows_main;
      best.Sm = Sm;
      best.St = St;
    }
  }
  return best;
}

template <bool kInt4>
static cudaError_t launch_prefill(const __half* x, const PrefillProblem& pb, int64_t M, int64_t K, cudaStream_t s) {
  const DeviceInfo di = current_device_info();
  int64_t rt = 0;
  for (int g = 0; g < pb.count; ++g) rt += (pb.N[g] + kQM - 1) / kQM;
  const int TN = prefill_tile_tokens(M);
  const int KS = TN <= kPrefillSSMaxTN ? kPrefillSSStageK : kQK;
  const int nk = static_cast<int>((K + KS - 1) / KS);
  const int64_t TT = (M + TN - 1) / TN;
  const int64_t base = rt * TT;
  auto capacity = [&](int cs) {
    if (TN == 64) return prefill_cluster_capacity<kInt4, 64, true, kPrefillSSStageK>(di.device, cs);
    if (TN == 128) return prefill_cluster_capacity<kInt4, 128, true, kPrefillSSStageK>(di.device, cs);
    return prefill_cluster_capacity<kInt4, 256, false, kQK>(di.device, cs);
  };
  auto run = [&](const PrefillProblem& p, int S) {
    if (TN == 64) return launch_prefill_t<kInt4, 64, true, kPrefillSSStageK>(x, p, M, K, S, s);
    if (TN == 128) return launch_prefill_t<kInt4, 128, true, kPrefillSSStageK>(x, p, M, K, S, s);
    return launch_prefill_t<kInt4, 256, false, kQK>(x, p, M, K, S, s);
  };
  int S = 1;
  while (S < 8 && base * S * 2 <= di.num_sms && S * 2 <= nk) {
    const int cap = capacity(S * 2);
    if (cap > 0 && base > cap) break;
    S *= 2;
  }
  if (S == 1) {
    const PrefillTailPlan tp = prefill_tail_plan(rt, TT, nk, di.num_sms, capacity);
    if (tp.rows_main > 0) {
      const cudaError_t e = run(sub_rows<kInt4>(pb, K, 0, tp.rows_main), tp.Sm);
      if (e != cudaSuccess) return e;
      return run(sub_rows<kInt4>(pb, K, tp.rows_main, rt), tp.St);
    }
  }
  return run(pb, S);
}

static PrefillProblem one_matrix(const void* w, const __half* sc, const uint8_t* zp, const __half* bias, __half* y,
                                 int64_t N) {
  PrefillProblem pb = {};
  pb.count = 1;
  pb.w[0] = w;
  pb.sc[0] = sc;
  pb.zp[0] = zp;
  pb.bias[0] = bias;
  pb.y[0] = y;
  pb.N[0] = N;
  return pb;
}

cudaError_t launch_tq_gemm_prefill(const __half* x, const uint8_t* packed, const __half* scale,
                                   const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                   cudaStream_t s) {
  return launch_prefill<false>(x, one_matrix(packed, scale, nullptr, bias, y, N), M, K, s);
}

cudaError_t launch_w4g_gemm_prefill(const __half* x, const int32_t* qweight, const __half* scales,
                                    const uint8_t* zeros, const __half* bias, __half* y, int64_t M, int64_t N,
                                    int64_t K, cudaStream_t s) {
  return launch_prefill<true>(x, one_matrix(qweight, scales, zeros, bias, y, N), M, K, s);
}

cudaError_t launch_gemm_prefill_grouped(bool int4, const __half* x, int count, const void* const* w,
                                        const __half* const* sc, const __half* const* bias, __half* const* y,
                                        const int64_t* N, int64_t M, int64_t K, cudaStream_t s) {
  if (count < 1 || count > kQMaxGroup) return cudaErrorInvalidValue;
  PrefillProblem pb = {};
  pb.count = count;
  for (int g = 0; g < count; ++g) {
    pb.w[g] = w[g];
    pb.sc[g] = sc[g];
    pb.zp[g] = nullptr;
    pb.bias[g] = bias[g];
    pb.y[g] = y[g];
    pb.N[g] = N[g];
  }
  return int4 ? launch_prefill<true>(x, pb, M, K, s) : launch_prefill<false>(x, pb, M, K, s);
}

}  // namespace tq
