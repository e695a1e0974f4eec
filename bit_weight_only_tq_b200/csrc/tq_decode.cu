// tq_decode.cu -- memory-bound skinny GEMM (M <= 64) for ternary and W4A16 weights.
//
// A CTA computes at most 16 tokens; 17 <= M <= 64 runs ceil(M / 16) token chunks over grid z
// in the same launch (the chunks of a row block stream the same weights at about the same time,
// so all but the first mostly read them from L2).
//
// [TQ] §1: decode time is spent fetching weights, so the kernel is built around the HBM stream
// of packed codes; [TQ] §4.2: codes are decoded into fp16 tensor-core fragments, accumulated in
// fp32, and the per-row scale is applied after the MMA.
//
// Work layout.  One CTA = one block of output rows (127 ternary rows plus one virtual row, or 128
// W4A16 rows) x one K-slice; a cluster of S CTAs (S <= 8) covers the whole K of its rows and
// reduces through distributed shared memory in a fixed order (deterministic, no global scratch).
// A stage is 128 bytes of every packed row (512 ternary or 256 INT4 codes) plus the activations
// of those k for all M tokens.  Per CTA:
//   * the last warp (producer) streams each stage with TMA into a ring: the 128-row x 128-byte packed
//     tile (issued before griddepcontrol.wait, weights never depend on the previous kernel) and
//     the activations, one 64-element block x M tokens per box (issued after it), both
//     128-byte swizzled so that every 16-byte read below is bank-conflict free.  For W4A16 it
//     also sums each 128-wide group of x per token;
//   * consumers: warp w owns rows 32 (w & 3) .. +31 (two 16-row MMA tiles).  For M <= 8 there
//     are eight, warp w taking the K half w >> 2 of every stage (the two halves are added in
//     shared memory, in a fixed order, at the end); for M > 8 there are four, each holding both
//     token groups, so that every decoded weight fragment feeds two MMAs.  Weights are the A
//     operand of mma.sync.m16n8k16 ("swap AB"), the tokens the N = 8 operand: one MMA per 256
//     weights and token group.  Each lane builds its B fragments from the activations in
//     shared memory (byte permutes into the k order the decode produces, see below); with two
//     row tiles per warp one fragment feeds four MMAs.
//
// In-register decode ("subnormal" trick).  ANDing a packed 32-bit word with 0x00030003 << 2p
// leaves, in each fp16 half, the code at bits 2p..2p+1: the exact value c * 2^(2p-24) (fp16
// subnormals for p <= 4, and still exactly linear for p = 5 where the code fills the two lowest
// exponent bits).  Positions 6, 7 are shifted down by 12 first.  So one word of 16 codes costs
// 1 shift + 8 ANDs for 8 fp16x2 registers, ~0.56 integer operations per weight.  The odd
// positions carry an extra factor 4, folded into their activation fragments (x / 4); the
// factors 2^-24 (position pairs 0 and 3), 2^-20 (pair 1) and 2^-16 (pair 2) are kept in three
// accumulators and applied exactly (powers of two) after the loop.  The codes are c = w + 1, so
// the result is sum_k c x - sum_k x; sum_k x comes out of the same MMAs as a virtual 128th row
// whose codes are all 01 (c = 1).
// W4A16 uses the same scheme with 4-bit fields (masks 0x000F000F / 0x00F000F0, x / 16 fold) and
// one 128-wide quantisation group per 64-byte sub-chunk: y += s[n,g] * (2^24 * C_g - 8 sum_g x).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kDTile = 128;                 // rows of one packed TMA tile
constexpr int kDRowSets = 4;                // 32 rows = two 16-row MMA tiles per consumer warp
constexpr int kDRT = 2;                     // 16-row MMA tiles per consumer warp

// Consumer warps per CTA, for NT token groups of which each warp holds TW: M <= 8 (NT = 1):
// eight, the two K halves of every stage split between warps w and w + 4; M > 8 with TW = 2:
// four, each holding both token groups (the decoded weights then feed two MMAs); M > 8 with
// TW = 1: eight, warp w holding token group w >> 2 (more warps to hide latency when a CTA has a
// single stage).  The producer is the warp after them.
template <int NT, int TW>
struct DecWarps {
  static constexpr int kCons = (NT == 2 && TW == 2) ? 4 : 8;
  static constexpr int kThreads = (kCons + 1) * 32;
};
constexpr int kDWBytes = kDTile * 128;      // weights of one stage: 128 rows x 128 bytes
constexpr int kDMaxRing = 8;                // stages resident in shared memory
constexpr int kDMaxCluster = 8;
constexpr int kDRedRows = kDTile + kDMaxCluster;  // >= S * ceil(rows / S): red holds [S][16][ceil(rows / S)]
constexpr int kDSmemBudget = 113 * 1024;    // two CTAs per SM

template <bool kInt4>
struct DecFmt {
  static constexpr int kStageK = kInt4 ? 256 : 512;  // codes per stage (128 bytes of a row)
  static constexpr int kKB = kStageK / 64;           // 64-element activation blocks per stage
  static constexpr int kRows = kInt4 ? 128 : 127;    // real output rows per CTA
};

constexpr int kDMaxGroup = 4;  // weight matrices sharing x in one launch (e.g. q, k, v)

struct DecodeArgs {
  int64_t M, K;
  int Mbox;       // tokens per CTA: M, or 16 when M > 16 (grid z = token chunks of 16)
  int C;          // stages along K
  int S;          // CTAs per cluster (K-slices)
  int ring;       // stages resident in shared memory
  int stage;      // bytes of one stage (weights + activations, multiple of 1024)
  int xhalf;      // bytes of one activation box [M][4 blocks][64] (multiple of 1024)
  int count;                        // matrices in the group
  int rb_start[kDMaxGroup + 1];     // first row block of each matrix in grid.y
  int64_t N[kDMaxGroup];
  const __half* sc[kDMaxGroup];     // ternary: scale[N]; W4A16: scales[N, K/128]
  const __half* bias[kDMaxGroup];   // may be null
  __half* y[kDMaxGroup];
};

struct DecodeMaps {
  CUtensorMap m[kDMaxGroup];        // packed weights of each matrix
  CUtensorMap x;                    // activations viewed as [M][K/64][64], box 64 x 4 x M,
                                    // 128-byte swizzle
};

template <bool kInt4>
struct DecLayout {
  static constexpr int kXg = kInt4 ? 2 * 16 * 4 : 0;  // W4A16 group sums of a stage [2][16]
  static constexpr int kRed = kDRedRows * 16 * 4;
  static constexpr int kSxr = kDMaxCluster * 16 * 4;
  static constexpr int kPart = kDTile * 8 * 4;        // second K half's partials (M <= 8)
  __host__ __device__ static constexpr int fixed() { return 1024 + kRed + kSxr + kPart + 3 * kDMaxRing * 8; }
  __host__ __device__ static constexpr int bytes(int ring, int stage) { return fixed() + ring * (stage + kXg); }
};

// Activations of a stage: one TMA box per four 64-element blocks (a ternary stage has two, a
// W4A16 stage one), laid out token-major: 128-byte row 4 m + b for token m, block b.  128-byte
// swizzle: 16-byte chunk c of row r sits at chunk position c ^ (r & 7).  128-bit shared loads
// are served eight lanes at a time; the eight lanes g in {2j, 2j+1}, t in 0..3 read rows
// 4 (8T + g) + t (+ const), whose swizzle phases 4 (g & 1) + t are all different, so every read
// is bank-conflict free.
__device__ __forceinline__ uint4 ld_x_chunk(const uint8_t* box, int row, int c) {
  return *reinterpret_cast<const uint4*>(box + row * 128 + ((c ^ (row & 7)) << 4));
}

// B fragments of one MMA pair from four activation words: even positions (x) and odd positions
// (x times `fold`), in the k order of the decode.
__device__ __forceinline__ void make_frag(uint32_t Pa, uint32_t Pb, uint32_t Pc, uint32_t Pd,
                                          __half2 fold, uint32_t& e0, uint32_t& e1, uint32_t& o0,
                                          uint32_t& o1) {
  e0 = __byte_perm(Pa, Pb, 0x5410);
  e1 = __byte_perm(Pc, Pd, 0x5410);
  uint32_t u01 = __byte_perm(Pa, Pb, 0x7632), u23 = __byte_perm(Pc, Pd, 0x7632);
  __half2 s01 = __hmul2(*reinterpret_cast<__half2*>(&u01), fold);
  __half2 s23 = __hmul2(*reinterpret_cast<__half2*>(&u23), fold);
  o0 = *reinterpret_cast<uint32_t*>(&s01);
  o1 = *reinterpret_cast<uint32_t*>(&s23);
}

template <bool kInt4, int NT, int TW>
__device__ __forceinline__ void decode_gemm_body(const DecodeMaps& maps, const DecodeArgs& a) {
  using F = DecFmt<kInt4>;
  using W = DecWarps<NT, TW>;
  using L = DecLayout<kInt4>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned; pointer arithmetic on the __shared__ array keeps the shared address
  // space visible to the compiler (plain ld/st.shared instead of generic accesses)
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stg = base;                                                  // ring x [weights | x]
  float* xg = reinterpret_cast<float*>(stg + a.ring * a.stage);         // ring x [2][16]
  float* red = xg + a.ring * (L::kXg / 4);                              // [S][16][own_cap]
  float* sxr = red + kDRedRows * 16;                                    // [S][16] slice sums of x
  float* part = sxr + kDMaxCluster * 16;                                // [128 rows][8 tokens]
  uint64_t* full = reinterpret_cast<uint64_t*>(part + kDTile * 8);
  uint64_t* xready = full + kDMaxRing;  // W4A16 group sums of the stage written
  uint64_t* empty = xready + kDMaxRing;

  pdl_allow_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rank = static_cast<int>(cluster_ctarank());
  // which matrix of the group this CTA works on, and its row block within that matrix
  int grp = 0;
#pragma unroll
  for (int q = 1; q < kDMaxGroup; ++q)
    if (q < a.count && static_cast<int>(blockIdx.y) >= a.rb_start[q]) grp = q;
  const int rb = static_cast<int>(blockIdx.y) - a.rb_start[grp];
  const int64_t row0 = static_cast<int64_t>(rb) * F::kRows;  // first output row of the block
  const CUtensorMap* tmap = &maps.m[grp];
  const int64_t Nm = a.N[grp];
  const __half* scm = a.sc[grp];
  const __half* biasm = a.bias[grp];
  __half* ym = a.y[grp] + static_cast<int64_t>(blockIdx.z) * 16 * a.N[grp];
  const int st_begin = static_cast<int>((static_cast<int64_t>(rank) * a.C) / a.S);
  const int st_end = static_cast<int>((static_cast<int64_t>(rank + 1) * a.C) / a.S);
  const int nst = st_end - st_begin;
  const int own_cap = (F::kRows + a.S - 1) / a.S;  // row slots per owner in `red`
  // token chunk of this CTA (M > 16 runs ceil(M / 16) chunks of 16 tokens over grid z: the CTAs
  // of one row block read the same weights at about the same time, so the chunks after the
  // first mostly hit L2)
  const int64_t tok0 = static_cast<int64_t>(blockIdx.z) * 16;
  const int Mi = static_cast<int>(a.M - tok0 < a.Mbox ? a.M - tok0 : a.Mbox);

  if (threadIdx.x == 0) {
    for (int i = 0; i < a.ring; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&xready[i], 32);
      mbar_init(&empty[i], W::kCons);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // this thread's output row of the epilogue and its scale / bias, fetched before any wait
  // (they never depend on the previous kernel) so that the epilogue does not wait on them
  const int rr0 = (rank * F::kRows) / a.S, rr1 = ((rank + 1) * F::kRows) / a.S;
  const int nrows = rr1 - rr0;
  const int ep_row = threadIdx.x;
  const int64_t ep_n = row0 + rr0 + ep_row;
  const bool ep_on = ep_row < nrows && ep_n < Nm;
  float ep_s = 1.0f, ep_b = 0.0f;
  if (ep_on) {
    if (!kInt4) ep_s = __half2float(scm[ep_n]);
    if (biasm) ep_b = __half2float(biasm[ep_n]);
  }

  if (warp == W::kCons) {
    // ================================================================== producer warp
    const uint32_t tx = static_cast<uint32_t>(kDWBytes + F::kKB * a.Mbox * 128);  // whole boxes
    auto load_w = [&](int i) {
      tma_load_2d(stg + (i % a.ring) * a.stage, tmap, &full[i % a.ring], (st_begin + i) * 128,
                  static_cast<int>(row0));
    };
    auto load_x = [&](int i) {
      uint8_t* dst = stg + (i % a.ring) * a.stage + kDWBytes;
#pragma unroll
      for (int hb = 0; hb < F::kKB / 4; ++hb)
        tma_load_3d(dst + hb * a.xhalf, &maps.x, &full[i % a.ring], 0, (st_begin + i) * F::kKB + 4 * hb,
                    static_cast<int32_t>(tok0));
    };
    const int pre = nst < a.ring ? nst : a.ring;
    if (lane == 0) {
      tma_prefetch_desc(tmap);
      tma_prefetch_desc(&maps.x);
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], tx);
        load_w(i);
      }
    }
    pdl_wait_prior_grids();  // the activations may come from the previous kernel
    if (lane == 0)
      for (int i = 0; i < pre; ++i) load_x(i);
    if (!kInt4) {
      if (lane == 0)
        for (int j = a.ring; j < nst; ++j) {
          const int slot = j % a.ring;
          if (!mbar_wait(&empty[slot], static_cast<uint32_t>((j / a.ring) - 1) & 1u)) break;
          mbar_arrive_expect_tx(&full[slot], tx);
          load_w(j);
          load_x(j);
        }
    } else {
      // group sums: lane -> token m = lane % (8*NT), block part = lane / (8*NT)
      constexpr int MP = 8 * NT, PARTS = 32 / MP, KBL = F::kKB / PARTS;
      const int m = lane % MP, part = lane / MP;
      for (int i = 0; i < nst; ++i) {
        const int slot = i % a.ring;
        const uint32_t ph = static_cast<uint32_t>(i / a.ring) & 1u;
        if (!mbar_wait_warp(&full[slot], ph)) break;  // warp-uniform exit
        const uint8_t* xs = stg + slot * a.stage + kDWBytes;
        float ps = 0.0f;
        if (m < Mi) {
#pragma unroll
          for (int bb = 0; bb < KBL; ++bb) {
            const int b = part * KBL + bb;  // W4A16: one box, rows 4 m + b
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 v = ld_x_chunk(xs, 4 * m + b, c);
              const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&u[j]));
                ps += f2.x + f2.y;
              }
            }
          }
        }
        // a group is 128 elements = 2 blocks: combine the two parts of one group
        if (KBL == 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, MP);
        const int gq = (part * KBL) >> 1;
        if (KBL == 2 || (part & 1) == 0) xg[(slot * 2 + gq) * 16 + m] = ps;
        mbar_arrive(&xready[slot]);
        const int j = i + a.ring;
        if (j < nst) {
          if (!mbar_wait_warp(&empty[slot], ph)) break;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[slot], tx);
            load_w(j);
            load_x(j);
          }
        }
      }
    }
  } else {
    // ================================================================== consumer warps
    // accumulator groups by exact power-of-two factor: pairs 0 and 3 (2^-24), 1 (2^-20), 2 (2^-16)
    constexpr int NG = kInt4 ? 1 : 3;
    const int rs = warp & (kDRowSets - 1), hi = warp / kDRowSets;  // hi: K half or token group
    const int sub_lo = NT == 1 ? hi : 0, sub_hi = NT == 1 ? hi + 1 : 2;
    const int Tb = TW < NT ? hi : 0;  // first token group of this warp
    bool tokv[TW];  // this lane's token 8(Tb+T) + g (B column g of token group Tb+T) exists
#pragma unroll
    for (int T = 0; T < TW; ++T) tokv[T] = 8 * (Tb + T) + g < Mi;
    float acc[NG][kDRT][TW][4];
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
        for (int T = 0; T < TW; ++T)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[q][rt][T][c] = 0.0f;
    const __half2 fold = kInt4 ? __floats2half2_rn(0.0625f, 0.0625f) : __floats2half2_rn(0.25f, 0.25f);
    // MMA tile row g is stored row gp of its group of eight, gp = (g >> 1) | (g & 1) << 2: the
    // eight lanes of a quarter warp then read rows of different swizzle phases (conflict free)
    const int gp = (g >> 1) | ((g & 1) << 2);
    const int rw = rs * 16 * kDRT + gp;  // row of tile 0, lower half; tile rt adds 16 rt, upper +8
    // ternary: tile row 127 is the virtual all-01 row (its result is sum_k x)
    const bool virt = !kInt4 && rw + 16 * (kDRT - 1) + 8 == kDTile - 1;
    const int64_t G = a.K >> 7;
    pdl_wait_prior_grids();  // block (not poll) until the previous kernel is done
    for (int i = 0; i < nst; ++i) {
      const int slot = i % a.ring;
      const uint32_t ph = static_cast<uint32_t>(i / a.ring) & 1u;
      if (!mbar_wait_warp(&full[slot], ph)) break;  // warp-uniform exit
      const uint8_t* st = stg + slot * a.stage;
      const uint8_t* xs = st + kDWBytes;
#pragma unroll 1
      for (int sub = sub_lo; sub < sub_hi; ++sub) {
        const int chunk = sub * 4 + t;  // this lane's 16 bytes of the packed rows
        // rows rw + 16 rt + 8 hr all have (row & 7) == gp: swizzled chunk position chunk ^ gp
        uint32_t w[kDRT][2][4];
#pragma unroll
        for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            uint4 U = *reinterpret_cast<const uint4*>(st + (rw + 16 * rt + 8 * hr) * 128 + ((chunk ^ gp) << 4));
            if (virt && rt == kDRT - 1 && hr == 1) U = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
            w[rt][hr][0] = U.x;
            w[rt][hr][1] = U.y;
            w[rt][hr][2] = U.z;
            w[rt][hr][3] = U.w;
          }
        if (!kInt4) {
          // the 64 codes of the chunk are k = 64*chunk + 0..63: activation block `chunk`, i.e.
          // block t of the box of sub-chunk `sub`
          const uint8_t* xbox = xs + sub * a.xhalf;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // P[T][j] = x[8(Tb+T)+g][64*chunk + 32h + 2j .. +1]
            uint32_t P[TW][16];
#pragma unroll
            for (int T = 0; T < TW; ++T)
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (tokv[T]) v = ld_x_chunk(xbox, 4 * (8 * (Tb + T) + g) + t, 4 * h + jj);
                P[T][4 * jj] = v.x;
                P[T][4 * jj + 1] = v.y;
                P[T][4 * jj + 2] = v.z;
                P[T][4 * jj + 3] = v.w;
              }
            uint32_t sh[kDRT][4];
#pragma unroll
            for (int rt = 0; rt < kDRT; ++rt) {
              sh[rt][0] = w[rt][0][2 * h] >> 12;
              sh[rt][1] = w[rt][1][2 * h] >> 12;
              sh[rt][2] = w[rt][0][2 * h + 1] >> 12;
              sh[rt][3] = w[rt][1][2 * h + 1] >> 12;
            }
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
              uint32_t be0[TW], be1[TW], bo0[TW], bo1[TW];
#pragma unroll
              for (int T = 0; T < TW; ++T)
                make_frag(P[T][pp], P[T][4 + pp], P[T][8 + pp], P[T][12 + pp], fold, be0[T], be1[T], bo0[T], bo1[T]);
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const int p = 2 * pp + q;
#pragma unroll
                for (int rt = 0; rt < kDRT; ++rt) {
                  uint32_t a0, a1, a2, a3;
                  if (p < 6) {
                    const uint32_t mk = 0x00030003u << (2 * p);
                    a0 = w[rt][0][2 * h] & mk;
                    a1 = w[rt][1][2 * h] & mk;
                    a2 = w[rt][0][2 * h + 1] & mk;
                    a3 = w[rt][1][2 * h + 1] & mk;
                  } else {
                    const uint32_t mk = (p == 6) ? 0x00030003u : 0x000C000Cu;
                    a0 = sh[rt][0] & mk;
                    a1 = sh[rt][1] & mk;
                    a2 = sh[rt][2] & mk;
                    a3 = sh[rt][3] & mk;
                  }
#pragma unroll
                  for (int T = 0; T < TW; ++T)
                    mma_16816(acc[pp == 3 ? 0 : pp][rt][T], a0, a1, a2, a3, q ? bo0[T] : be0[T], q ? bo1[T] : be1[T]);
                }
              }
            }
          }
        } else {
          // the 32 codes of the chunk are k = 32*chunk + 0..31: half (chunk & 1) of activation
          // block chunk / 2, its 16-byte chunks 4*(chunk & 1) + 0..3
          uint32_t P[TW][16];
#pragma unroll
          for (int T = 0; T < TW; ++T)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              uint4 v = make_uint4(0u, 0u, 0u, 0u);
              if (tokv[T]) v = ld_x_chunk(xs, 4 * (8 * (Tb + T) + g) + (chunk >> 1), 4 * (chunk & 1) + jj);
              P[T][4 * jj] = v.x;
              P[T][4 * jj + 1] = v.y;
              P[T][4 * jj + 2] = v.z;
              P[T][4 * jj + 3] = v.w;
            }
          float cg[2][kDRT][TW][4];  // two chains (class 0 / class 1 fields)
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
              for (int T = 0; T < TW; ++T)
#pragma unroll
                for (int c = 0; c < 4; ++c) cg[j][rt][T][c] = 0.0f;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
              uint32_t be0[TW], be1[TW], bo0[TW], bo1[TW];
#pragma unroll
              for (int T = 0; T < TW; ++T)
                make_frag(P[T][8 * h + s2], P[T][8 * h + 2 + s2], P[T][8 * h + 4 + s2], P[T][8 * h + 6 + s2], fold,
                          be0[T], be1[T], bo0[T], bo1[T]);
#pragma unroll
              for (int rt = 0; rt < kDRT; ++rt) {
                const uint32_t x0 = w[rt][0][2 * h] >> (8 * s2), x1 = w[rt][1][2 * h] >> (8 * s2);
                const uint32_t x2 = w[rt][0][2 * h + 1] >> (8 * s2), x3 = w[rt][1][2 * h + 1] >> (8 * s2);
#pragma unroll
                for (int cls = 0; cls < 2; ++cls) {
                  const uint32_t mk = cls ? 0x00F000F0u : 0x000F000Fu;
#pragma unroll
                  for (int T = 0; T < TW; ++T)
                    mma_16816(cg[cls][rt][T], x0 & mk, x1 & mk, x2 & mk, x3 & mk, cls ? bo0[T] : be0[T],
                              cls ? bo1[T] : be1[T]);
                }
              }
            }
          if (sub == sub_lo) (void)mbar_wait_warp(&xready[slot], ph);
          const int64_t gi = static_cast<int64_t>(st_begin + i) * 2 + sub;
#pragma unroll
          for (int rt = 0; rt < kDRT; ++rt) {
            const int64_t n0 = row0 + rw + 16 * rt, n1 = n0 + 8;
            // groups past K (a zero-filled half stage) contribute nothing
            const float s0 = (n0 < Nm && gi < G) ? __half2float(scm[n0 * G + gi]) : 0.0f;
            const float s1 = (n1 < Nm && gi < G) ? __half2float(scm[n1 * G + gi]) : 0.0f;
#pragma unroll
            for (int T = 0; T < TW; ++T) {
              const float xg0 = 8.0f * xg[(slot * 2 + sub) * 16 + 8 * (Tb + T) + 2 * t];
              const float xg1 = 8.0f * xg[(slot * 2 + sub) * 16 + 8 * (Tb + T) + 2 * t + 1];
              float c4[4];
#pragma unroll
              for (int c = 0; c < 4; ++c) c4[c] = cg[0][rt][T][c] + cg[1][rt][T][c];
              acc[0][rt][T][0] = fmaf(s0, fmaf(c4[0], 16777216.0f, -xg0), acc[0][rt][T][0]);
              acc[0][rt][T][1] = fmaf(s0, fmaf(c4[1], 16777216.0f, -xg1), acc[0][rt][T][1]);
              acc[0][rt][T][2] = fmaf(s1, fmaf(c4[2], 16777216.0f, -xg0), acc[0][rt][T][2]);
              acc[0][rt][T][3] = fmaf(s1, fmaf(c4[3], 16777216.0f, -xg1), acc[0][rt][T][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    // this warp's results: factors 2^-24 (pairs 0 and 3), 2^-20 (pair 1), 2^-16 (pair 2) applied
    // exactly; rows rw + 16 rt + 8 hr, tokens 8 (Tb + T) + 2t + c
    float v[kDRT][TW][4];
#pragma unroll
    for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
      for (int T = 0; T < TW; ++T)
#pragma unroll
        for (int ci = 0; ci < 4; ++ci)
          v[rt][T][ci] = kInt4 ? acc[0][rt][T][ci]
                               : fmaf(acc[0][rt][T][ci], 16777216.0f,
                                      fmaf(acc[1 % NG][rt][T][ci], 1048576.0f, acc[2 % NG][rt][T][ci] * 65536.0f));
    if (NT == 1) {  // M <= 8: add the second K half (warps 4-7) to the first, fixed order
      if (hi == 1) {
#pragma unroll
        for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
          for (int ci = 0; ci < 4; ++ci)
            part[(rw + 16 * rt + 8 * (ci >> 1)) * 8 + 2 * t + (ci & 1)] = v[rt][0][ci];
      }
      named_barrier_sync(1, W::kCons * 32);
      if (hi == 1) goto consumers_done;
#pragma unroll
      for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
        for (int ci = 0; ci < 4; ++ci) v[rt][0][ci] += part[(rw + 16 * rt + 8 * (ci >> 1)) * 8 + 2 * t + (ci & 1)];
    }
    {
      // push this slice's partial results to the CTA that owns each row (owner q holds rows
      // [q*R/S, (q+1)*R/S) of the R real rows); the virtual row goes to every owner
      const uint32_t red_local = smem_u32(red), sxr_local = smem_u32(sxr);
#pragma unroll
      for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int r = rw + 16 * rt + 8 * hr;
          const bool vrow = virt && rt == kDRT - 1 && hr == 1;
          const int q = ((r + 1) * a.S - 1) / F::kRows;
          const int slot = r - (q * F::kRows) / a.S;
#pragma unroll
          for (int T = 0; T < TW; ++T)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const float val = v[rt][T][2 * hr + c];
              const int tok = 8 * (Tb + T) + 2 * t + c;
              if (vrow) {
                for (int o = 0; o < a.S; ++o)
                  st_shared_cluster_f32(mapa_shared(sxr_local + (rank * 16 + tok) * 4, static_cast<uint32_t>(o)), val);
              } else if (r < F::kRows) {
                st_shared_cluster_f32(
                    mapa_shared(red_local + ((rank * 16 + tok) * own_cap + slot) * 4, static_cast<uint32_t>(q)), val);
              }
            }
        }
    }
  consumers_done:;
  }

  // ==================================================================== cluster reduction
  cluster_sync_all();  // every partial and slice sum has landed in its owner's shared memory
  pdl_wait_prior_grids();
  if (ep_on) {
    const int Mv = Mi < 8 * NT ? Mi : 8 * NT;
    for (int mm = 0; mm < Mv; ++mm) {
      float v = 0.0f, sx = 0.0f;
      for (int q = 0; q < a.S; ++q) {  // fixed order: deterministic
        v += red[(q * 16 + mm) * own_cap + ep_row];  // consecutive rows: conflict free
        if (!kInt4) sx += sxr[q * 16 + mm];
      }
      if (!kInt4) v = (v - sx) * ep_s;
      ym[mm * Nm + ep_n] = __float2half_rn(v + ep_b);
    }
  }
}

// M <= 8: two CTAs of nine warps per SM; five warps share one SM sub-partition's 16K registers,
// so a thread may use at most 102 (96 it is).
template <bool kInt4>
__global__ void __maxnreg__(96)
    decode_gemm_kernel_m8(const __grid_constant__ DecodeMaps maps, const __grid_constant__ DecodeArgs a) {
  decode_gemm_body<kInt4, 1, 1>(maps, a);
}

// M <= 16, both token groups per warp: two CTAs of five warps per SM (at most 168 registers).
template <bool kInt4>
__global__ void __launch_bounds__(DecWarps<2, 2>::kThreads, 2)
    decode_gemm_kernel_m16(const __grid_constant__ DecodeMaps maps, const __grid_constant__ DecodeArgs a) {
  decode_gemm_body<kInt4, 2, 2>(maps, a);
}

// M <= 16, one token group per warp: two CTAs of nine warps per SM (96 registers, as above).
template <bool kInt4>
__global__ void __maxnreg__(96)
    decode_gemm_kernel_m16s(const __grid_constant__ DecodeMaps maps, const __grid_constant__ DecodeArgs a) {
  decode_gemm_body<kInt4, 2, 1>(maps, a);
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
struct DecodePlan {
  int S, C, ring, stage, xhalf, smem;
};

// Stage ring and cluster size for RB row blocks x `chunks` token chunks of M tokens each.
template <bool kInt4>
static bool plan_decode_t(int64_t RB, int64_t M, int64_t K, int num_sms, DecodePlan* p, int64_t chunks) {
  using F = DecFmt<kInt4>;
  using L = DecLayout<kInt4>;
  const int C = static_cast<int>((K + F::kStageK - 1) / F::kStageK);
  const int xhalf = ((static_cast<int>(M) * 4 * 128 + 1023) / 1024) * 1024;
  const int xbytes = (F::kKB / 4) * xhalf;  // activation boxes of one stage
  const int stage = kDWBytes + xbytes;
  // as many stages as two CTAs per SM allow (a CTA's whole slice when it fits, so that all its
  // weights are in flight before griddepcontrol.wait)
  int ring = kDMaxRing;
  while (ring > 2 && L::bytes(ring, stage) > kDSmemBudget) --ring;
  const int smem = L::bytes(ring, stage);
  if (smem > kDSmemBudget) return false;
  // one wave of two CTAs per SM, at most 8 K-slices per row block
  int64_t S = (2 * static_cast<int64_t>(num_sms)) / (RB * chunks);
  if (S < 1) S = 1;
  if (S > kDMaxCluster) S = kDMaxCluster;
  if (S > C) S = C;
  *p = DecodePlan{static_cast<int>(S), C, ring, stage, xhalf, smem};
  return true;
}

static bool plan_decode(bool int4, int64_t RB, int64_t M, int64_t K, int num_sms, DecodePlan* p,
                        int64_t chunks = 1) {
  return int4 ? plan_decode_t<true>(RB, M, K, num_sms, p, chunks) : plan_decode_t<false>(RB, M, K, num_sms, p, chunks);
}

template <bool kInt4, int NT, int TW>
static cudaError_t launch_decode_t(const DecodeMaps& maps, const DecodeArgs& a, const DecodePlan& p,
                                   cudaStream_t s) {
  auto* kern = NT == 1 ? decode_gemm_kernel_m8<kInt4>
                       : (TW == 2 ? decode_gemm_kernel_m16<kInt4> : decode_gemm_kernel_m16s<kInt4>);
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kDSmemBudget);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.S), static_cast<unsigned>(a.rb_start[a.count]),
                     static_cast<unsigned>((a.M + 15) / 16));
  cfg.blockDim = dim3(DecWarps<NT, TW>::kThreads, 1, 1);
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
  using F = DecFmt<kInt4>;
  if (count < 1 || count > kDMaxGroup) return cudaErrorInvalidValue;
  const DeviceInfo di = current_device_info();
  const int64_t Mbox = M > 16 ? 16 : M;
  const int64_t chunks = (M + 15) / 16;
  const int NT = Mbox > 8 ? 2 : 1;
  DecodeArgs a = {};
  DecodeMaps maps;
  a.M = M;
  a.Mbox = static_cast<int>(Mbox);
  a.K = K;
  a.count = count;
  int64_t rbs = 0;
  const int64_t kbytes = kInt4 ? K / 2 : K / 4;
  for (int g = 0; g < count; ++g) {
    a.rb_start[g] = static_cast<int>(rbs);
    rbs += (N[g] + F::kRows - 1) / F::kRows;
    a.N[g] = N[g];
    a.sc[g] = sc[g];
    a.bias[g] = bias ? bias[g] : nullptr;
    a.y[g] = y[g];
    if (!make_tmap_2d(&maps.m[g], CU_TENSOR_MAP_DATA_TYPE_UINT8, w[g], static_cast<uint64_t>(kbytes),
                      static_cast<uint64_t>(N[g]), static_cast<uint64_t>(kbytes), 128, kDTile,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  for (int g = count; g < kDMaxGroup; ++g) maps.m[g] = maps.m[0];
  {  // activations viewed as [M][K/64][64]: one box = four 64-element blocks x Mbox tokens
    const uint64_t dims[3] = {64, static_cast<uint64_t>(K / 64), static_cast<uint64_t>(M)};
    const uint64_t strides[2] = {128, static_cast<uint64_t>(K) * 2};
    const uint32_t box[3] = {64, 4, static_cast<uint32_t>(Mbox)};
    if (!make_tmap_3d(&maps.x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  a.rb_start[count] = static_cast<int>(rbs);
  if (rbs > 65535) return cudaErrorInvalidValue;
  DecodePlan p;
  if (!plan_decode(kInt4, rbs, Mbox, K, di.num_sms, &p, chunks)) return cudaErrorInvalidValue;
  a.C = p.C;
  a.S = p.S;
  a.ring = p.ring;
  a.stage = p.stage;
  a.xhalf = p.xhalf;
  if (NT == 1) return launch_decode_t<kInt4, 1, 1>(maps, a, p, s);
  // a CTA with a single stage and two CTAs per SM: more, lighter warps hide the latency better
  const bool single = (p.C + p.S - 1) / p.S <= 1 && static_cast<int64_t>(p.S) * rbs * chunks > di.num_sms;
  return single ? launch_decode_t<kInt4, 2, 1>(maps, a, p, s) : launch_decode_t<kInt4, 2, 2>(maps, a, p, s);
}

bool decode_supported(bool int4, int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > kDecodeMaxM || N < 1) return false;
  if (int4 ? (K % 128 != 0) : (K % 64 != 0)) return false;
  DecodePlan p;
  const int64_t rows = int4 ? DecFmt<true>::kRows : DecFmt<false>::kRows;
  return plan_decode(int4, (N + rows - 1) / rows, M > 16 ? 16 : M, K, 148, &p, (M + 15) / 16);
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
