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
// Work layout.  One CTA = one block of 128 output rows x one K-slice; a cluster of S CTAs (S <= 8) covers the whole K of its rows and
// reduces through distributed shared memory in a fixed order (deterministic, no global scratch).
// A stage is 128 bytes of every packed row (512 ternary or 256 INT4 codes) plus the activations
// of those k for all M tokens.  Per CTA:
//   * the last warp (producer) streams each stage with TMA into a ring: the 128-row x 128-byte packed
//     tile (issued before griddepcontrol.wait, weights never depend on the previous kernel) and
//     the activations, one 64-element block x M tokens per box (issued after it), both
//     128-byte swizzled so that every 16-byte read below is bank-conflict free;
//   * consumers: warp w owns rows 32 (w & 3) .. +31 (two 16-row MMA tiles).  For M <= 8 there
//     are eight, warp w taking the K half w >> 2 of every stage (the two halves are added in
//     shared memory, in a fixed order, at the end); for M > 8 there are four, each holding both
//     token groups, so that every decoded weight fragment feeds two MMAs.  Weights are the A
//     operand of mma.sync.m16n8k16 ("swap AB"), the tokens the N = 8 operand: one MMA per 256
//     weights and token group.  Each lane builds its B fragments from the activations in
//     shared memory (byte permutes into the k order the decode produces, see below); with two
//     row tiles per warp one fragment feeds four MMAs.
//
// In-register decode, exact.  The MMA multiplies the weight values themselves, so the fp32
// accumulators only ever hold partial sums of x * What (no large sum of x is formed and
// subtracted at the end: that cancellation would cost accuracy on rows with few nonzero codes).
//   ternary: code position p (0..7) of a 32-bit word holds the codes of k = p and k = p + 8 in
//     its two fp16 halves.  Shifting them to bits 14-15 of each half and keeping the complement
//     of those two bits gives the fp16 values -2 / -0 / +2 = 2 (c - 1) (the code's high bit lands
//     on the sign): one shift and one LOP3 per register of two weights; the result is halved
//     after the loop.  The activation fragments are x pairs (p, p + 8), picked with byte permutes.
//   W4A16: ANDing a word with 0x000F000F (nibbles at bits 0-3) or 0x00F000F0 (bits 4-7) leaves
//     u * 2^-24 or u * 2^-20 in each half (fp16 subnormals, exactly linear in u); one fp16x2
//     subtraction of z units gives (u - z) times that power of two exactly.  The two fields
//     accumulate in separate chains, combined with an exact factor 1/16, and each 128-wide
//     quantisation group (one 64-byte sub-chunk) is scaled as y += s[n,g] * 2^24 * sum_g (u - 8) x.
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
  static constexpr int kRows = 128;                   // output rows per CTA
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
  uint32_t four;  // 4 (decode multiplier, see DecLane)
  int count;                        // matrices in the group
  int rb_start[kDMaxGroup + 1];     // first row block of each matrix in grid.y
  int64_t N[kDMaxGroup];
  const __half* sc[kDMaxGroup];     // ternary: scale[N]; W4A16: scales[N, K/128]
  const uint8_t* zp[kDMaxGroup];    // W4A16 zero-points [N, K/128], or null (symmetric: 8)
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
  static constexpr int kRed = kDRedRows * 16 * 4;
  static constexpr int kPart = kDTile * 8 * 4;        // second K half's partials (M <= 8)
  __host__ __device__ static constexpr int fixed() { return 1024 + kRed + kPart + 2 * kDMaxRing * 8; }
  __host__ __device__ static constexpr int bytes(int ring, int stage) { return fixed() + ring * stage; }
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

// B fragments of one MMA pair from four activation words: the low fp16 halves (even positions)
// and the high halves (odd positions) of (Pa, Pb) and of (Pc, Pd), in the k order of the decode.
__device__ __forceinline__ void make_frag(uint32_t Pa, uint32_t Pb, uint32_t Pc, uint32_t Pd, uint32_t& e0,
                                          uint32_t& e1, uint32_t& o0, uint32_t& o1) {
  e0 = __byte_perm(Pa, Pb, 0x5410);
  e1 = __byte_perm(Pc, Pd, 0x5410);
  o0 = __byte_perm(Pa, Pb, 0x7632);
  o1 = __byte_perm(Pc, Pd, 0x7632);
}

// One A-fragment register.  `mask` selects one code field in each fp16 half, which then holds
// the code times the field's unit (a power of two: the pattern 0x0001 << field offset);
// subtracting `unit` (the offset times that field unit: 1 for ternary, 8 for W4A16) leaves
// (code - offset) * field unit, i.e. the weight value -1 / 0 / +1 or -8..7 times a power of two.
// fp16 arithmetic is exact here: operands and result are multiples of the subnormal quantum
// 2^-24 below 2^-12.
__device__ __forceinline__ uint32_t dec_field(uint32_t w, uint32_t mask, uint32_t unit) {
  uint32_t a = w & mask;
  __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&unit));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Lane constants of a consumer warp: MMA fragment coordinates (g = lane / 4, t = lane % 4), the
// stored row of tile row g (gp) and of this warp's first tile row (rw), the sub-chunks of a stage
// this warp covers and its first token group.
struct DecLane {
  int g, t, gp, rw, sub_lo, sub_hi, Tb;
  uint32_t four;  // 4, from the launch parameters: the compiler cannot turn `x * four` into a shift
};

// One stage of the consumer loop: this warp's rows (two 16-row tiles) x its sub-chunks of the
// stage's 128 bytes per row, for its token groups, accumulated into `acc` (ternary: three
// exact power-of-two classes; W4A16: one, the group scales already applied).  `st` is the
// stage's weight tile, followed by its activation boxes (`xhalf` bytes each).  W4A16 needs the
// first quantisation group of the stage (`gi_base`), the block's first row and the scales.
// One ternary A-fragment register: code position p (0..7) of a packed word, i.e. the codes of
// k = p (low fp16 half) and k = p + 8 (high half) of the word's 16.  Shifting the code to bits
// 14-15 of each half puts its high bit b1 at the sign bit and its low bit b0 at the top exponent
// bit; complementing both and clearing the rest leaves the fp16 value
//   c = 0b00 -> 0xC000 = -2,  c = 0b01 -> 0x8000 = -0,  c = 0b10 -> 0x4000 = +2,
// i.e. exactly 2 (c - 1): one shift and one LOP3 per two weights, no arithmetic.  (Code 0b11 is
// invalid and decodes to +0.)

// kIL: the ternary weights are in the pair-interleaved layout (slot j of a word holds k = 2j,
// slot 8 + j holds k = 2j + 1), so the activation pair of code position p is the p-th 32-bit
// word of x as it lies in shared memory: no byte permutes.
template <bool kInt4, int NT, int TW, bool kIL = false>
__device__ __forceinline__ void dec_stage(float (&acc)[kDRT][TW][4], const uint8_t* st, int xhalf,
                                          const DecLane& L, const int (&xrow)[TW], int64_t gi_base,
                                          int64_t row0, int64_t Nm, const __half* scm, const uint8_t* zpm,
                                          int64_t G) {
  const int t = L.t, gp = L.gp, rw = L.rw, sub_lo = L.sub_lo, sub_hi = L.sub_hi;
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
        w[rt][hr][0] = U.x;
        w[rt][hr][1] = U.y;
        w[rt][hr][2] = U.z;
        w[rt][hr][3] = U.w;
      }
    if (!kInt4) {
      // the 64 codes of the chunk are k = 64*chunk + 0..63: activation block `chunk`, i.e.
      // block t of the box of sub-chunk `sub`
      const uint8_t* xbox = xs + sub * xhalf;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // P[T][j] = x[8(Tb+T)+g][64*chunk + 32h + 2j .. +1]
        uint32_t P[TW][16];
#pragma unroll
        for (int T = 0; T < TW; ++T)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint4 v = ld_x_chunk(xbox, xrow[T] + t, 4 * h + jj);
            P[T][4 * jj] = v.x;
            P[T][4 * jj + 1] = v.y;
            P[T][4 * jj + 2] = v.z;
            P[T][4 * jj + 3] = v.w;
          }
        // position p of words 2h (k = 64 chunk + 32h + p, + p + 8) and 2h + 1 (+ 16 + p, + 24 + p):
        // x pairs (p, p + 8) are the even (p even) or odd halves of P[p / 2] and P[p / 2 + 4].
        // Positions run 7 .. 0 on running copies of the words moved two bits left per step
        // (code p at bits 14-15 / 30-31); the move is a multiply by four, which runs on the FMA
        // pipe and leaves the integer ALU pipe to the masks and the x permutes.
        uint32_t sw[kDRT][4];
#pragma unroll
        for (int rt = 0; rt < kDRT; ++rt) {
          sw[rt][0] = w[rt][0][2 * h];
          sw[rt][1] = w[rt][1][2 * h];
          sw[rt][2] = w[rt][0][2 * h + 1];
          sw[rt][3] = w[rt][1][2 * h + 1];
        }
#pragma unroll
        for (int pp = 0; pp < 8; ++pp) {
          const int p = 7 - pp;
          const uint32_t sel = (p & 1) ? 0x7632u : 0x5410u;
          uint32_t b0[TW], b1[TW];
#pragma unroll
          for (int T = 0; T < TW; ++T) {
            if (kIL) {  // k = 2p, 2p + 1 of words 2h and 2h + 1
              b0[T] = P[T][p];
              b1[T] = P[T][8 + p];
            } else {
              b0[T] = __byte_perm(P[T][p >> 1], P[T][(p >> 1) + 4], sel);
              b1[T] = __byte_perm(P[T][8 + (p >> 1)], P[T][12 + (p >> 1)], sel);
            }
          }
#pragma unroll
          for (int rt = 0; rt < kDRT; ++rt) {
            if (pp > 0) {
#pragma unroll
              for (int j = 0; j < 4; ++j) sw[rt][j] *= L.four;
            }
            const uint32_t a0 = ~sw[rt][0] & 0xC000C000u, a1 = ~sw[rt][1] & 0xC000C000u;
            const uint32_t a2 = ~sw[rt][2] & 0xC000C000u, a3 = ~sw[rt][3] & 0xC000C000u;
#pragma unroll
            for (int T = 0; T < TW; ++T) mma_16816(acc[rt][T], a0, a1, a2, a3, b0[T], b1[T]);
          }
        }
      }
    } else {
      // the group scales of this lane's rows, requested before the MMAs that they follow
      const int64_t gi = gi_base + sub;
      float sg[kDRT][2];
      uint32_t zz[kDRT][2];  // zero-point of each row's group (8 for the symmetric format)
#pragma unroll
      for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int64_t n = row0 + rw + 16 * rt + 8 * hr;
          // groups past K (a zero-filled half stage) contribute nothing
          const bool in = n < Nm && gi < G;
          sg[rt][hr] = in ? __half2float(scm[n * G + gi]) : 0.0f;
          zz[rt][hr] = (zpm && in) ? static_cast<uint32_t>(zpm[n * G + gi]) : 8u;
        }
      // the 32 codes of the chunk are k = 32*chunk + 0..31: half (chunk & 1) of activation
      // block chunk / 2, its 16-byte chunks 4*(chunk & 1) + 0..3
      uint32_t P[TW][16];
#pragma unroll
      for (int T = 0; T < TW; ++T)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const uint4 v = ld_x_chunk(xs, xrow[T] + (chunk >> 1), 4 * (chunk & 1) + jj);
          P[T][4 * jj] = v.x;
          P[T][4 * jj + 1] = v.y;
          P[T][4 * jj + 2] = v.z;
          P[T][4 * jj + 3] = v.w;
        }
      float cg[2][kDRT][TW][4];  // two chains: nibble fields at bits 0-3 (unit 2^-24) and 4-7 (2^-20)
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
            make_frag(P[T][8 * h + s2], P[T][8 * h + 2 + s2], P[T][8 * h + 4 + s2], P[T][8 * h + 6 + s2], be0[T],
                      be1[T], bo0[T], bo1[T]);
#pragma unroll
          for (int rt = 0; rt < kDRT; ++rt) {
            const uint32_t x0 = w[rt][0][2 * h] >> (8 * s2), x1 = w[rt][1][2 * h] >> (8 * s2);
            const uint32_t x2 = w[rt][0][2 * h + 1] >> (8 * s2), x3 = w[rt][1][2 * h + 1] >> (8 * s2);
#pragma unroll
            for (int cls = 0; cls < 2; ++cls) {
              // u at bits 0-3 (value u 2^-24) or 4-7 (u 2^-20); minus z units: (u - z) exactly
              const uint32_t mk = cls ? 0x00F000F0u : 0x000F000Fu;
              const uint32_t unit = cls ? 0x00100010u : 0x00010001u;
              const uint32_t zg = zz[rt][0] * unit, zh = zz[rt][1] * unit;  // rows g and g + 8
              const uint32_t d0 = dec_field(x0, mk, zg), d1 = dec_field(x1, mk, zh);
              const uint32_t d2 = dec_field(x2, mk, zg), d3 = dec_field(x3, mk, zh);
#pragma unroll
              for (int T = 0; T < TW; ++T)
                mma_16816(cg[cls][rt][T], d0, d1, d2, d3, cls ? bo0[T] : be0[T], cls ? bo1[T] : be1[T]);
            }
          }
        }
#pragma unroll
      for (int rt = 0; rt < kDRT; ++rt) {
        // the group's sum of (u - z) x in units of 2^-24: the second field's chain (units of
        // 2^-20) times 1/16 (exact powers of two)
        const float s0u = sg[rt][0] * 16777216.0f, s1u = sg[rt][1] * 16777216.0f;
#pragma unroll
        for (int T = 0; T < TW; ++T) {
          float c4[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) c4[c] = fmaf(cg[1][rt][T][c], 0.0625f, cg[0][rt][T][c]);
          acc[rt][T][0] = fmaf(s0u, c4[0], acc[rt][T][0]);
          acc[rt][T][1] = fmaf(s0u, c4[1], acc[rt][T][1]);
          acc[rt][T][2] = fmaf(s1u, c4[2], acc[rt][T][2]);
          acc[rt][T][3] = fmaf(s1u, c4[3], acc[rt][T][3]);
        }
      }
    }
  }
}

// Final fp32 values of a warp's tiles: ternary accumulates 2 (c - 1) x (the decoded weights are
// -2, -0, +2), halved here exactly; W4A16 has the group scales applied already.  Rows
// rw + 16 rt + 8 (ci >> 1), tokens 8 (Tb + T) + 2t + (ci & 1).
template <bool kInt4, int TW>
__device__ __forceinline__ void dec_values(const float (&acc)[kDRT][TW][4], float (&v)[kDRT][TW][4]) {
#pragma unroll
  for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
    for (int T = 0; T < TW; ++T)
#pragma unroll
      for (int ci = 0; ci < 4; ++ci) v[rt][T][ci] = kInt4 ? acc[rt][T][ci] : 0.5f * acc[rt][T][ci];
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
  float* red = reinterpret_cast<float*>(stg + a.ring * a.stage);        // [S][16][own_cap]
  float* part = red + kDRedRows * 16;                                   // [128 rows][8 tokens]
  uint64_t* full = reinterpret_cast<uint64_t*>(part + kDTile * 8);
  uint64_t* empty = full + kDMaxRing;

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
  const uint8_t* zpm = a.zp[grp];
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
    const bool skipx = skip_x_loads();  // failure-path test hook: never set in normal use
    auto load_x = [&](int i) {
      if (skipx) return;
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
    if (lane == 0)
      for (int j = a.ring; j < nst; ++j) {
        const int slot = j % a.ring;
        if (!mbar_wait(&empty[slot], static_cast<uint32_t>((j / a.ring) - 1) & 1u)) break;
        mbar_arrive_expect_tx(&full[slot], tx);
        load_w(j);
        load_x(j);
      }
  } else {
    // ================================================================== consumer warps
    const int rs = warp & (kDRowSets - 1), hi = warp / kDRowSets;  // hi: K half or token group
    const int sub_lo = NT == 1 ? hi : 0, sub_hi = NT == 1 ? hi + 1 : 2;
    const int Tb = TW < NT ? hi : 0;  // first token group of this warp
    int xrow[TW];  // activation row of this lane's token 8(Tb+T) + g (B column g of group Tb+T)
#pragma unroll
    for (int T = 0; T < TW; ++T) xrow[T] = 4 * min(8 * (Tb + T) + g, static_cast<int>(Mi) - 1);
    float acc[kDRT][TW][4];
#pragma unroll
    for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
      for (int T = 0; T < TW; ++T)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[rt][T][c] = 0.0f;
    // MMA tile row g is stored row gp of its group of eight, gp = (g >> 1) | (g & 1) << 2: the
    // eight lanes of a quarter warp then read rows of different swizzle phases (conflict free)
    const int gp = (g >> 1) | ((g & 1) << 2);
    const int rw = rs * 16 * kDRT + gp;  // row of tile 0, lower half; tile rt adds 16 rt, upper +8
    const int64_t G = a.K >> 7;
    const DecLane L{g, t, gp, rw, sub_lo, sub_hi, Tb, a.four};
    pdl_wait_prior_grids();  // block (not poll) until the previous kernel is done
    for (int i = 0; i < nst; ++i) {
      const int slot = i % a.ring;
      const uint32_t ph = static_cast<uint32_t>(i / a.ring) & 1u;
      if (!mbar_wait_warp(&full[slot], ph)) break;  // warp-uniform exit
      const uint8_t* st = stg + slot * a.stage;
      dec_stage<kInt4, NT, TW>(acc, st, a.xhalf, L, xrow, static_cast<int64_t>(st_begin + i) * 2, row0, Nm, scm, zpm,
                               G);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    float v[kDRT][TW][4];
    dec_values<kInt4, TW>(acc, v);
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
      // [q*R/S, (q+1)*R/S) of the R rows)
      const uint32_t red_local = smem_u32(red);
#pragma unroll
      for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int r = rw + 16 * rt + 8 * hr;
          const int q = ((r + 1) * a.S - 1) / F::kRows;
          const int slot = r - (q * F::kRows) / a.S;
#pragma unroll
          for (int T = 0; T < TW; ++T)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const float val = v[rt][T][2 * hr + c];
              const int tok = 8 * (Tb + T) + 2 * t + c;
              st_shared_cluster_f32(
                  mapa_shared(red_local + ((rank * 16 + tok) * own_cap + slot) * 4, static_cast<uint32_t>(q)), val);
            }
        }
    }
  consumers_done:;
  }

  // ==================================================================== cluster reduction
  cluster_sync_all();  // every partial has landed in its owner's shared memory
  pdl_wait_prior_grids();
  if (ep_on) {
    const int Mv = Mi < 8 * NT ? Mi : 8 * NT;
    for (int mm = 0; mm < Mv; ++mm) {
      float v = 0.0f;
      for (int q = 0; q < a.S; ++q)  // fixed order: deterministic
        v += red[(q * 16 + mm) * own_cap + ep_row];  // consecutive rows: conflict free
      if (!kInt4) v *= ep_s;
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
                                       cudaStream_t s, const uint8_t* const* zp = nullptr) {
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
    a.zp[g] = zp ? zp[g] : nullptr;
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
  a.four = 4u;
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
  return plan_decode(int4, (N + rows - 1) / rows, M > 16 ? 16 : M, K, current_device_info().num_sms, &p,
                     (M + 15) / 16);
}

cudaError_t launch_tq_gemm_decode(const __half* x, const uint8_t* packed, const __half* scale,
                                  const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                  cudaStream_t s) {
  const void* w = packed;
  return launch_decode_group<false>(x, 1, &w, &scale, &bias, &y, &N, M, K, s);
}

cudaError_t launch_w4g_gemm_decode(const __half* x, const int32_t* qweight, const __half* scales,
                                   const uint8_t* zeros, const __half* bias, __half* y, int64_t M, int64_t N,
                                   int64_t K, cudaStream_t s) {
  const void* w = qweight;
  return launch_decode_group<true>(x, 1, &w, &scales, &bias, &y, &N, M, K, s, &zeros);
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
