// tq_tcbatch.cu -- persistent work-list GEMM on the 5th-generation tensor cores for 1 <= M <= 32.
//
// The same work split as tq_batch.cu (stages = item, 128-row block, 128 bytes of every row; CTA
// c owns the contiguous stages [c T / G, (c + 1) T / G); split row blocks summed through the
// workspace in K order), with the multiply on tcgen05 instead of mma.sync:
//   D[row, token] (TMEM, fp32) += A[row, k] (TMEM, decoded fp16 weights) * B[token, k] (smem, x)
// M = 128 weight rows (TMEM lanes), N = TN tokens (16 or 32), K = 16 per instruction.  One
// instruction covers 2048 weights for all the tokens at once, so the multiply stays off the
// issue slots; what is left per weight is the decode ([TQ] §4.2: decode to fp16 tensor-core
// operands, fp32 accumulation, scale after the MMA).
//
// One CTA per SM, twelve warps:
//   warp 0       TMA producer: per stage the 128 x 128-byte packed tile and the stage's x as one
//                box [sub-stage][TN tokens][64 k] (128-byte swizzle); weights requested before
//                griddepcontrol.wait, x after it;
//   warp 1       allocates tensor memory; one lane issues the MMAs: four per 64-k sub-stage into
//                the row block's accumulator (two accumulators, so one row block's epilogue
//                overlaps the next one's MMAs);
//   warps 2-3    ternary: reorder each 16-k block of x in place to the k order of the decode
//                (below); W4A16 needs no reorder;
//   warps 4-7    decode: thread r = weight row r = TMEM lane r; per sub-stage its 16 (ternary) or
//                32 (W4A16) bytes become 32 registers of fp16 pairs, stored with one tcgen05.st
//                into a ring of A slots (32 columns each);
//   warps 8-11   epilogue: tcgen05.ld of a finished accumulator, scale / bias, fp16 y, or the
//                fp32 partial of a split row block to the workspace and the arrival count.
//
// Ternary decode: code position p (0..7) of a 32-bit word holds the codes of k = p and p + 8;
// ~(word << (14 - 2p)) & 0xC000C000 is exactly 2 (c - 1) in each fp16 half (the high code bit on
// the sign, the low one on the top exponent bit).  So TMEM column 8q + p of a sub-stage holds
// the pair (k = 16q + p, 16q + p + 8), which the MMA takes as its k = 16q + 2p, +1: the helper
// warps store x the same way (x'[16q + 2p + h] = x[16q + p + 8h]).  The accumulator holds
// 2 (c - 1) x sums, halved in the epilogue.  W4A16: natural k order, fp16((u - z) * s) per
// pair (as the prefill kernel).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kTcThreads = 384;
constexpr int kTcARing = 12;       // TMEM A slots (sub-stages of 64 k, 32 columns each)
constexpr int kTcMaxRing = 8;      // stages resident in shared memory
constexpr int kTcSlotTokens = 32;  // workspace slot: [32 tokens][128 rows] fp32

template <bool kInt4, int TN>
struct TcLayout {
  static constexpr int kSubs = kInt4 ? 4 : 8;          // 64-k sub-stages per stage
  static constexpr int kRowSub = kInt4 ? 32 : 16;      // packed bytes per row per sub-stage
  static constexpr int kW = 128 * 128;                 // packed tile of a stage
  static constexpr int kXSub = TN * 128;               // x of one sub-stage: TN rows x 64 fp16
  static constexpr int kStage = kW + kSubs * kXSub;
  static constexpr uint32_t kColA = 2 * TN;            // two accumulators, then the A ring
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kColA + 32 * kTcARing <= kTmemCols, "tensor memory");
  static_assert(kXSub % 1024 == 0, "x sub-stages stay on 1024-byte swizzle atoms");
  // barriers: full, xready, empty [kTcMaxRing]; afull, aempty [kTcARing]; dfull, dempty [2]; fin
  static constexpr int kBars = 3 * kTcMaxRing + 2 * kTcARing + 5;
  __host__ __device__ static constexpr int fixed() { return 1024 + 8 * kBars + 16; }
  __host__ __device__ static constexpr int bytes(int ring) { return fixed() + ring * kStage; }
};

struct TcItem {
  const __half* sc;    // ternary: scale[N]; W4A16: scales[N, K/128]
  const uint8_t* zp;   // W4A16 zero-points or null
  const __half* bias;  // may be null
  __half* y;           // [M, N]
  int64_t N, K;
  int64_t begin;       // first stage of this item
  int C;               // stages per row block
  int RB;              // row blocks
};

struct TcParams {
  CUtensorMap w[kBatchMaxItems];  // packed weights [N rows][row bytes], box 128 B x 128 rows
  CUtensorMap x[kBatchMaxItems];  // x viewed as [K/64][M][64], box 64 x TN x sub-stages
  TcItem it[kBatchMaxItems];
  int count, M, G, ring;
  int64_t T;
  int* counters;                  // [G]
  float* slots;                   // [2G][32][128]
};

// (The host keeps T * G below 2^32, so both are exact in 32-bit arithmetic.)
__device__ __forceinline__ int64_t tc_range_begin(int c, int64_t T, int G) {
  return static_cast<int64_t>(static_cast<uint32_t>(c) * static_cast<uint32_t>(T) / static_cast<uint32_t>(G));
}
__device__ __forceinline__ int tc_range_owner(int64_t s, int64_t T, int G) {
  return static_cast<int>((static_cast<uint32_t>(s + 1) * static_cast<uint32_t>(G) - 1u) / static_cast<uint32_t>(T));
}

// Position (item, row block, stage within the row block) walked stage by stage.
struct TcPos {
  int it, rb, kst;
  __device__ __forceinline__ void advance(const TcParams& P) {
    if (++kst == P.it[it].C) {
      kst = 0;
      if (++rb == P.it[it].RB) {
        rb = 0;
        ++it;
      }
    }
  }
};

__device__ __forceinline__ uint32_t tc_dec_tq(uint32_t w, int p) {
  const uint32_t s = p == 7 ? w : (w << (14 - 2 * p));
  return ~s & 0xC000C000u;
}

__device__ __forceinline__ uint32_t tc_byte_halves(uint32_t w, int bi) {
  return __byte_perm(w, 0u, static_cast<uint32_t>(bi | (4 << 4) | (bi << 8) | (4 << 12)));
}

// 8 consecutive INT4 codes (one word) -> 4 registers of fp16 pairs (u - z) * s in k order.
__device__ __forceinline__ void tc_dec_w4(uint32_t w, uint32_t s2, uint32_t zsub, uint32_t* o) {
#pragma unroll
  for (int bi = 0; bi < 4; ++bi) {
    const uint32_t t = tc_byte_halves(w, bi);
    uint32_t h = (t & 0x00F0000Fu) | 0x54006400u;  // (1024 + u_lo, 64 + u_hi)
    __half2 d = __hsub2(*reinterpret_cast<__half2*>(&h), *reinterpret_cast<const __half2*>(&zsub));
    d = __hmul2(d, *reinterpret_cast<const __half2*>(&s2));
    o[bi] = *reinterpret_cast<uint32_t*>(&d);
  }
}

template <bool kInt4, int TN>
__global__ void __launch_bounds__(kTcThreads, 1) tc_batch_kernel(const __grid_constant__ TcParams P) {
  using L = TcLayout<kInt4, TN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stg = sm;                                                   // ring x [weights | x]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P.ring * L::kStage);
  uint64_t* full = bars;                         // stage landed (TMA)           count 1
  uint64_t* xready = full + kTcMaxRing;          // x reordered (helpers)        count 2
  uint64_t* empty = xready + kTcMaxRing;         // stage consumed               count 4 + 1 commit
  uint64_t* afull = empty + kTcMaxRing;          // A slot written (decode)      count 4
  uint64_t* aempty = afull + kTcARing;           // A slot consumed (commit)     count 1
  uint64_t* dfull = aempty + kTcARing;           // accumulator done (commit)    count 1, [2]
  uint64_t* dempty = dfull + 2;                  // accumulator read (epilogue)  count 4, [2]
  uint64_t* fin = dempty + 2;                    // every MMA done (commit)      count 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [0] abort, [1] last

  pdl_allow_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = static_cast<int>(blockIdx.x);
  const int64_t s0 = tc_range_begin(c, P.T, P.G), s1 = tc_range_begin(c + 1, P.T, P.G);
  const int nst = static_cast<int>(s1 - s0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < P.ring; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&xready[i], 2);
      mbar_init(&empty[i], 5);
    }
    for (int i = 0; i < kTcARing; ++i) {
      mbar_init(&afull[i], 4);
      mbar_init(&aempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&dfull[i], 1);
      mbar_init(&dempty[i], 4);
    }
    mbar_init(fin, 1);
    flags[0] = 0;
    flags[1] = 0;
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

  TcPos pos0{0, 0, 0};
  if (nst > 0) {
    while (pos0.it + 1 < P.count && P.it[pos0.it + 1].begin <= s0) ++pos0.it;
    const uint32_t off0 = static_cast<uint32_t>(s0 - P.it[pos0.it].begin);
    pos0.rb = static_cast<int>(off0 / static_cast<uint32_t>(P.it[pos0.it].C));
    pos0.kst = static_cast<int>(off0 % static_cast<uint32_t>(P.it[pos0.it].C));
  }
  auto unit_end = [&](const TcPos& p, int i) { return p.kst == P.it[p.it].C - 1 || i == nst - 1; };

  if (warp == 0) {
    // ==================================================================== TMA producer
    if (lane == 0 && nst > 0) {
      const uint32_t tx = static_cast<uint32_t>(L::kStage);
      for (int q = 0; q < P.count; ++q) {
        tma_prefetch_desc(&P.w[q]);
        tma_prefetch_desc(&P.x[q]);
      }
      const bool skipx = skip_x_loads();  // failure-path test hook: never set in normal use
      TcPos p = pos0;
      const int pre = nst < P.ring ? nst : P.ring;
      for (int i = 0; i < pre; ++i) {  // model constants: before the wait
        mbar_arrive_expect_tx(&full[i], tx);
        tma_load_2d(stg + i * L::kStage, &P.w[p.it], &full[i], p.kst * 128, p.rb * 128);
        p.advance(P);
      }
      pdl_wait_prior_grids();
      p = pos0;
      for (int i = 0; i < nst; ++i) {
        const int slot = i % P.ring;
        if (i >= pre) {
          if (!mbar_wait(&empty[slot], static_cast<uint32_t>((i / P.ring) - 1) & 1u)) {
            flags[0] = 1;
            break;
          }
          mbar_arrive_expect_tx(&full[slot], tx);
          tma_load_2d(stg + slot * L::kStage, &P.w[p.it], &full[slot], p.kst * 128, p.rb * 128);
        }
        if (!skipx)
          tma_load_3d(stg + slot * L::kStage + L::kW, &P.x[p.it], &full[slot], 0, 0, p.kst * L::kSubs);
        p.advance(P);
      }
    }
  } else if (warp == 1) {
    // ==================================================================== MMA issuer
    if (lane == 0) {
      bool ok = true;
      const uint32_t idesc = idesc_f16_f32(128, TN);
      TcPos p = pos0;
      int a = 0;        // sub-stages issued
      int u = 0;        // row blocks (units) started
      bool first = true;
      for (int i = 0; i < nst; ++i) {
        const int slot = i % P.ring;
        const uint32_t ph = static_cast<uint32_t>(i / P.ring) & 1u;
        if (ok) ok = mbar_wait(&full[slot], ph) && (kInt4 || mbar_wait(&xready[slot], ph));
        if (ok && first && u >= 2) ok = mbar_wait(&dempty[u & 1], static_cast<uint32_t>((u >> 1) - 1) & 1u);
        const uint32_t d_tmem = tmem + static_cast<uint32_t>((u & 1) * TN);
        const uint32_t x_base = smem_u32(stg + slot * L::kStage + L::kW);
        for (int sub = 0; sub < L::kSubs; ++sub, ++a) {
          const int as = a % kTcARing;
          if (ok) ok = mbar_wait(&afull[as], static_cast<uint32_t>(a / kTcARing) & 1u);
          if (ok) {
            tc_fence_after_sync();
            const uint64_t bdesc = sdesc_kmajor_sw128(x_base + sub * L::kXSub);
            const uint32_t a_tmem = tmem + L::kColA + 32 * as;
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16)
              umma_f16_ts(d_tmem, a_tmem + 8 * k16, bdesc + 2 * k16, idesc, (first && sub == 0 && k16 == 0) ? 0u : 1u);
            umma_commit(&aempty[as]);
          }
        }
        if (ok) umma_commit(&empty[slot]);
        first = false;
        if (unit_end(p, i)) {
          if (ok) umma_commit(&dfull[u & 1]);
          ++u;
          first = true;
        }
        p.advance(P);
      }
      if (!ok) flags[0] = 1;
      umma_commit(fin);  // every MMA issued above has completed when this arrives
      (void)mbar_wait(fin, 0u);
    }
  } else if (warp < 4) {
    // ==================================================================== x reorder (ternary)
    if (!kInt4) {
      bool ok = true;
      const int ht = threadIdx.x - 64;  // 0..63
      for (int i = 0; i < nst; ++i) {
        const int slot = i % P.ring;
        if (ok) ok = mbar_wait_warp(&full[slot], static_cast<uint32_t>(i / P.ring) & 1u);
        if (ok) {
          uint8_t* xs = stg + slot * L::kStage + L::kW;
          // items: (sub-stage, token, 16-k block q): chunks 2q and 2q + 1 of the token's row
          for (int e = ht; e < L::kSubs * TN * 4; e += 64) {
            const int q = e & 3, row = e >> 2;  // row = sub * TN + token
            uint8_t* rp = xs + row * 128;
            const int sw = row & 7;
            uint4* c0 = reinterpret_cast<uint4*>(rp + (((2 * q) ^ sw) << 4));
            uint4* c1 = reinterpret_cast<uint4*>(rp + (((2 * q + 1) ^ sw) << 4));
            const uint4 lo = *c0, hi = *c1;  // x[16q + 0..7], x[16q + 8..15]
            const uint32_t L0[4] = {lo.x, lo.y, lo.z, lo.w}, H0[4] = {hi.x, hi.y, hi.z, hi.w};
            uint32_t o[8];
#pragma unroll
            for (int pp = 0; pp < 8; ++pp)
              o[pp] = __byte_perm(L0[pp >> 1], H0[pp >> 1], (pp & 1) ? 0x7632u : 0x5410u);  // (x[p], x[p + 8])
            *c0 = make_uint4(o[0], o[1], o[2], o[3]);
            *c1 = make_uint4(o[4], o[5], o[6], o[7]);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) mbar_arrive(&xready[slot]);
      }
    }
  } else if (warp < 8) {
    // ==================================================================== decode
    bool ok = true;
    const int r = threadIdx.x - 128;  // weight row of the block = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp - 4) * 32) << 16);
    TcPos p = pos0;
    int a = 0;
    // W4A16: the scales and zero-points of a stage's two groups, fetched one stage ahead so that
    // their latency stays off the decode
    uint32_t scv[2] = {0u, 0u}, zv[2] = {8u, 8u}, scn[2] = {0u, 0u}, zn[2] = {8u, 8u};
    auto fetch_groups = [&](const TcPos& q, uint32_t (&sc)[2], uint32_t (&z)[2]) {
      const TcItem& J = P.it[q.it];
      const int64_t nn = static_cast<int64_t>(q.rb) * 128 + r, G = J.K >> 7;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int64_t gi = static_cast<int64_t>(q.kst) * 2 + j;
        const bool in = nn < J.N && gi < G;
        sc[j] = in ? static_cast<uint32_t>(__half_as_ushort(J.sc[nn * G + gi])) : 0u;
        z[j] = (in && J.zp) ? static_cast<uint32_t>(J.zp[nn * G + gi]) : 8u;
      }
    };
    if (kInt4 && nst > 0) fetch_groups(pos0, scv, zv);
    for (int i = 0; i < nst; ++i) {
      const int slot = i % P.ring;
      if (kInt4 && i + 1 < nst) {
        TcPos q = p;
        q.advance(P);
        fetch_groups(q, scn, zn);
      }
      if (ok) ok = mbar_wait_warp(&full[slot], static_cast<uint32_t>(i / P.ring) & 1u);
      const uint8_t* prow = stg + slot * L::kStage + r * 128;
      for (int sub = 0; sub < L::kSubs; ++sub, ++a) {
        const int as = a % kTcARing;
        uint32_t v[32];
        if (!kInt4) {
          const uint4 pw = *reinterpret_cast<const uint4*>(prow + ((sub ^ (r & 7)) << 4));
          const uint32_t wq[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int pp = 0; pp < 8; ++pp) v[8 * q + pp] = tc_dec_tq(wq[q], pp);
        } else {
          const uint32_t sg = scv[sub >> 1], zg = zv[sub >> 1];
          const uint32_t s2 = sg | (sg << 16);
          const uint32_t zsub = ((0x5400u + 16u * zg) << 16) | (0x6400u + zg);
          const uint4 p0 = *reinterpret_cast<const uint4*>(prow + (((2 * sub) ^ (r & 7)) << 4));
          const uint4 p1 = *reinterpret_cast<const uint4*>(prow + (((2 * sub + 1) ^ (r & 7)) << 4));
          const uint32_t wq[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) tc_dec_w4(wq[q], s2, zsub, v + 4 * q);
        }
        if (ok && a >= kTcARing) {
          ok = mbar_wait_warp(&aempty[as], static_cast<uint32_t>((a / kTcARing) - 1) & 1u);
          tc_fence_after_sync();
        }
        if (ok) {
          tmem_st_32x32b_x32(lane_base + L::kColA + 32 * as, v);
          tmem_st_wait();
          tc_fence_before_sync();
        }
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&afull[as]);
      }
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&empty[slot]);
      if (!ok) flags[0] = 1;
      p.advance(P);
      if (kInt4) {
        scv[0] = scn[0];
        scv[1] = scn[1];
        zv[0] = zn[0];
        zv[1] = zn[1];
      }
    }
  } else {
    // ==================================================================== epilogue
    bool ok = true;
    const int e = threadIdx.x - 256;  // 0..127: row e of the block
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp - 8) * 32) << 16);
    pdl_wait_prior_grids();           // y and the workspace belong to the previous kernel until now
    TcPos p = pos0;
    int u = 0;
    int64_t ustart = s0;              // first stage of the current row block within the range
    for (int i = 0; i < nst; ++i) {
      if (unit_end(p, i)) {
        const TcItem& I = P.it[p.it];
        const int64_t n = static_cast<int64_t>(p.rb) * 128 + e;
        float ep_s = 1.0f, ep_b = 0.0f;
        if (n < I.N) {
          if (!kInt4) ep_s = 0.5f * __half2float(I.sc[n]);  // the decode doubled the weights
          if (I.bias) ep_b = __half2float(I.bias[n]);
        }
        if (ok) ok = mbar_wait_warp(&dfull[u & 1], static_cast<uint32_t>(u >> 1) & 1u);
        uint32_t acc[TN];
        if (ok) {
          tc_fence_after_sync();
          if (TN == 16) {
            uint32_t (&a16)[16] = *reinterpret_cast<uint32_t(*)[16]>(acc);
            tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>((u & 1) * TN), a16);
          } else {
            uint32_t (&a32)[32] = *reinterpret_cast<uint32_t(*)[32]>(acc);
            tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>((u & 1) * TN), a32);
          }
          tmem_ld_wait();
          tc_fence_before_sync();
        }
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&dempty[u & 1]);
        if (!ok) flags[0] = 1;
        named_barrier_sync(2, 128);
        const bool abort = flags[0] != 0;
        const int64_t gB0 = I.begin + static_cast<int64_t>(p.rb) * I.C, gB1 = gB0 + I.C;
        const int Mt = P.M;
        if (!abort && gB0 >= s0 && gB1 <= s1) {
          if (n < I.N)
#pragma unroll
            for (int tok = 0; tok < TN; ++tok)
              if (tok < Mt)
                I.y[static_cast<int64_t>(tok) * I.N + n] = __float2half_rn(fmaf(__uint_as_float(acc[tok]), ep_s, ep_b));
        } else if (!abort) {
          const int cf = tc_range_owner(gB0, P.T, P.G), cl = tc_range_owner(gB1 - 1, P.T, P.G);
          float* mine = P.slots + (2 * static_cast<int64_t>(c) + (gB0 <= s0 ? 0 : 1)) * kTcSlotTokens * 128;
#pragma unroll
          for (int tok = 0; tok < TN; ++tok)
            if (tok < Mt) mine[tok * 128 + e] = __uint_as_float(acc[tok]);
          named_barrier_sync(2, 128);
          if (e == 0) {
            // the barrier orders the 128 threads' partials before this release; the acquire
            // orders the other contributors' partials before the reads after the next barrier
            const int old = atom_add_acq_rel_gpu(&P.counters[cf], 1);
            flags[1] = old == cl - cf;
          }
          named_barrier_sync(2, 128);
          if (flags[1]) {
            // eight tokens at a time: every load of a slot for them is in flight before the first
            // add (one L2 round trip per contributor, not one per token)
            if (n < I.N)
#pragma unroll
              for (int q0 = 0; q0 < TN; q0 += 8) {
                if (q0 >= Mt) break;
                float v[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] = 0.0f;
                for (int cc = cf; cc <= cl; ++cc) {  // K order: deterministic
                  const int64_t sl = 2 * static_cast<int64_t>(cc) + (gB0 <= tc_range_begin(cc, P.T, P.G) ? 0 : 1);
                  const float* src = P.slots + sl * kTcSlotTokens * 128 + e;
                  float t[8];
#pragma unroll
                  for (int q = 0; q < 8; ++q)
                    if (q0 + q < Mt) t[q] = __ldcg(src + (q0 + q) * 128);
#pragma unroll
                  for (int q = 0; q < 8; ++q)
                    if (q0 + q < Mt) v[q] += t[q];
                }
#pragma unroll
                for (int q = 0; q < 8; ++q)
                  if (q0 + q < Mt) I.y[static_cast<int64_t>(q0 + q) * I.N + n] = __float2half_rn(fmaf(v[q], ep_s, ep_b));
              }
            if (e == 0) P.counters[cf] = 0;
          }
        }
        named_barrier_sync(2, 128);  // the flag is free again
        ++u;
        ustart = s0 + i + 1;
      }
      p.advance(P);
    }
    (void)ustart;
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
// Workspace: the counter region of the mma.sync variant (sized for two CTAs per SM, so that one
// layout serves both variants), then [2 G][32][128] fp32 slots.
int64_t tc_batch_workspace_bytes_for(int G) {
  return batch_counter_bytes(kBCtasPerSm * G) + 2 * static_cast<int64_t>(G) * kTcSlotTokens * 128 * 4;
}

template <bool kInt4, int TN>
static cudaError_t launch_tc_t(const BatchLinear* items, int count, int64_t M, void* ws, int64_t ws_bytes,
                               cudaStream_t s) {
  using L = TcLayout<kInt4, TN>;
  const DeviceInfo di = current_device_info();
  TcParams P;
  P.count = count;
  P.M = static_cast<int>(M);
  int64_t T = 0;
  for (int q = 0; q < count; ++q) {
    const BatchLinear& b = items[q];
    TcItem& I = P.it[q];
    I.sc = b.sc;
    I.zp = b.zp;
    I.bias = b.bias;
    I.y = b.y;
    I.N = b.N;
    I.K = b.K;
    I.C = static_cast<int>((b.K + (kInt4 ? 256 : 512) - 1) / (kInt4 ? 256 : 512));
    I.RB = static_cast<int>((b.N + 127) / 128);
    I.begin = T;
    T += static_cast<int64_t>(I.C) * I.RB;
    const int64_t kbytes = kInt4 ? b.K / 2 : b.K / 4;
    if (!make_tmap_2d(&P.w[q], CU_TENSOR_MAP_DATA_TYPE_UINT8, b.w, static_cast<uint64_t>(kbytes),
                      static_cast<uint64_t>(b.N), static_cast<uint64_t>(kbytes), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    // x[M][K] viewed as [K/64][M][64]: dimension 0 = 64 k, 1 = token (stride K), 2 = k block (stride 128 B)
    const uint64_t dims[3] = {64, static_cast<uint64_t>(M), static_cast<uint64_t>(b.K / 64)};
    const uint64_t strides[2] = {static_cast<uint64_t>(b.K) * 2, 128};
    const uint32_t box[3] = {64, static_cast<uint32_t>(TN), static_cast<uint32_t>(L::kSubs)};
    if (!make_tmap_3d(&P.x[q], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, b.x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  for (int q = count; q < kBatchMaxItems; ++q) {
    P.w[q] = P.w[0];
    P.x[q] = P.x[0];
    P.it[q] = P.it[0];
    P.it[q].begin = T;
  }
  const int Gmax = di.num_sms;
  if (ws_bytes < tc_batch_workspace_bytes_for(Gmax)) return cudaErrorInvalidValue;
  P.T = T;
  P.G = static_cast<int>(T < Gmax ? T : Gmax);
  if (T * P.G >= (static_cast<int64_t>(1) << 32)) return cudaErrorInvalidValue;  // 32-bit range arithmetic
  int ring = kTcMaxRing;
  while (ring > 2 && L::bytes(ring) > 227 * 1024) --ring;
  P.ring = ring;
  const int smem = L::bytes(ring);
  P.counters = reinterpret_cast<int*>(ws);
  P.slots = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + batch_counter_bytes(kBCtasPerSm * Gmax));
  auto* kern = tc_batch_kernel<kInt4, TN>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(P.G), 1, 1);
  cfg.blockDim = dim3(kTcThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

cudaError_t launch_gemm_batch_tc(bool int4, const BatchLinear* items, int count, int64_t M, void* ws,
                                 int64_t ws_bytes, cudaStream_t s) {
  if (count < 1 || count > kBatchMaxItems || M < 1 || M > 32) return cudaErrorInvalidValue;
  if (int4) return M <= 16 ? launch_tc_t<true, 16>(items, count, M, ws, ws_bytes, s)
                           : launch_tc_t<true, 32>(items, count, M, ws, ws_bytes, s);
  return M <= 16 ? launch_tc_t<false, 16>(items, count, M, ws, ws_bytes, s)
                 : launch_tc_t<false, 32>(items, count, M, ws, ws_bytes, s);
}

}  // namespace tq
