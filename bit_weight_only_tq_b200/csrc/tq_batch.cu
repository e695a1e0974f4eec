// tq_batch.cu -- persistent decode GEMM over a work list of independent linears (M <= 16).
//
// [TQ] §1: a decode step is bound by the HBM stream of packed weights, and a serving engine's
// step runs many small linears; every launch boundary leaves SMs idle for microseconds (the
// previous grid drains, the next one starts, the first activations arrive).  This kernel takes up
// to kBMaxItems linears that share M -- the linears of one decoder layer, say -- and streams all
// their packed weights in ONE launch, with a fixed set of CTAs (two per SM):
//
//   * The work is the sequence of stages (item, block of 128 rows, 128 bytes of every row of the
//     block), item-major, then row-block-major, then along K; T stages in total.  CTA c takes the
//     contiguous range [c T / G, (c + 1) T / G): every CTA streams the same number of bytes, so
//     the launch ends when the bytes are through, whatever the shapes.
//   * A row block whose stages all fall to one CTA is finished there (scale, bias, fp16 y).  A row
//     block split between CTAs (only at the ends of a CTA's range) is summed through a
//     caller-provided workspace: each contributor stores its fp32 partial in its own slot and
//     counts itself in on the row block's counter; the last to arrive adds the slots in K order
//     (deterministic: the same sum whichever CTA arrives last), writes y and resets the counter,
//     so the workspace is ready for the next call.  Nobody waits for anybody.
//   * The producer warp streams the next row blocks' weights into the ring while the consumer
//     warps finish a row block; the weights of the first stages are requested before
//     griddepcontrol.wait (model constants), so they arrive while the previous grid drains.
//
// The per-stage math is the decode kernel's (tq_decode.cu): mma.sync m16n8k16 with the weights
// as the A operand, decoded exactly into fp16 in registers; fp32 accumulation.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kBMaxItems = kBatchMaxItems;
constexpr int kBRows = 128;       // rows of a row block (one packed TMA tile)
constexpr int kBResPitch = 132;   // fp32 row pitch of the result buffer [token][row]
constexpr int kBCtasPerSm = 2;
constexpr bool kBatchM8FourWarps = false;  // M <= 8: four consumer warps over whole stages (measured slower)
constexpr int kBatchPreW = 8;              // stages whose weights are loaded before the PDL wait

struct BatchItem {
  const __half* sc;    // ternary: scale[N]; W4A16: scales[N, K/128]
  const uint8_t* zp;   // W4A16 zero-points [N, K/128], or null (symmetric)
  const __half* bias;  // may be null
  __half* y;           // [M, N]
  int64_t N, K;
  int64_t begin;       // first stage of this item in the launch's sequence
  int C;               // stages per row block (along K)
  int RB;              // row blocks
};

// The next call's linears (an L2 prefetch of the stages its CTAs load first).
struct BatchNextItem {
  int64_t begin;  // first stage of this item in the next call's sequence
  int C, RB;      // stages per row block, row blocks
};

struct BatchParams {
  CUtensorMap w[kBMaxItems];  // packed weights: [N rows][row bytes], box 128 B x 128 rows, 128-B swizzle
  CUtensorMap x[kBMaxItems];  // activations viewed as [M][K/64][64], box 64 x 4 x M, 128-B swizzle
  BatchItem it[kBMaxItems];
  int count;
  int M;
  int G;                      // CTAs
  int ring, stage, xhalf;
  uint32_t four;              // 4 (decode multiplier, see DecLane)
  int pre_w;                  // stages whose weights are requested before the wait on the previous kernel
  int64_t T;                  // stages in total
  int* counters;              // [G] arrivals per split row block, indexed by its first contributor
  float* slots;               // [2 G][16][128] fp32 partials: slot 2c = CTA c's first row block,
                              // 2c + 1 = its last
  // the next call on this stream, when the caller names it: its packed weights, its stage
  // sequence, its CTAs and ring depth (0 items: none)
  CUtensorMap wn[kBMaxItems];
  BatchNextItem nit[kBMaxItems];
  int ncount, Gn, nring;
  int64_t Tn;
};

template <bool kInt4>
struct BatchLayout {
  static constexpr int kRes = 16 * kBResPitch * 4;
  static constexpr int kItems = kBMaxItems * static_cast<int>(sizeof(BatchItem));
  __host__ __device__ static constexpr int fixed() { return 1024 + kRes + 2 * kDMaxRing * 8 + 2 * 8 + 16 + kItems; }
  __host__ __device__ static constexpr int bytes(int ring, int stage) { return fixed() + ring * stage; }
};

// Workspace layout: counters first (256-byte padded), then the partial slots.
__host__ __device__ inline int64_t batch_counter_bytes(int G) { return ((static_cast<int64_t>(G) * 4 + 255) / 256) * 256; }
__host__ __device__ inline int64_t batch_workspace_bytes_for(int G) {
  return batch_counter_bytes(G) + 2 * static_cast<int64_t>(G) * 16 * kBRows * 4;
}

// First stage of CTA c's range, and the CTA whose range holds stage s.
// (The host keeps T * G below 2^32, so both are exact in 32-bit arithmetic.)
__device__ __forceinline__ int64_t range_begin(int c, int64_t T, int G) {
  return static_cast<int64_t>(static_cast<uint32_t>(c) * static_cast<uint32_t>(T) / static_cast<uint32_t>(G));
}
__device__ __forceinline__ int range_owner(int64_t s, int64_t T, int G) {
  return static_cast<int>((static_cast<uint32_t>(s + 1) * static_cast<uint32_t>(G) - 1u) / static_cast<uint32_t>(T));
}

// NT token groups of eight, TW of them per consumer warp, CW consumer warps.  With eight
// consumer warps and one token group the two K halves of a stage go to two warp sets (kSplitK);
// otherwise every consumer warp takes its rows over the whole stage.
template <bool kInt4, int NT, int TW, int CW, bool kIL = false>
__device__ __forceinline__ void batch_body(const BatchParams& P) {
  using F = DecFmt<kInt4>;
  constexpr int kCons = CW;
  constexpr bool kSplitK = NT == 1 && CW == 8;
  constexpr int kEp = kCons * 32;  // consumer threads (epilogue)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stg = base;                                                 // ring x [weights | x]
  float* res = reinterpret_cast<float*>(stg + P.ring * P.stage);       // [16 tokens][kBResPitch]
  uint64_t* full = reinterpret_cast<uint64_t*>(res + 16 * kBResPitch);
  uint64_t* empty = full + kDMaxRing;
  uint64_t* resfull = empty + kDMaxRing;   // a row block's sum is in `res` (consumers)      count 1
  uint64_t* resempty = resfull + 1;        // `res` read by the epilogue warp                 count 1
  volatile int* flags = reinterpret_cast<volatile int*>(resempty + 1);  // [0] abort
  // the items, copied from the launch parameters once: indexed reads of a parameter block go
  // through the generic load path, shared memory is a short-latency read
  BatchItem* its = reinterpret_cast<BatchItem*>(resempty + 3);

  pdl_allow_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = static_cast<int>(blockIdx.x);
  const int64_t s0 = range_begin(c, P.T, P.G), s1 = range_begin(c + 1, P.T, P.G);
  const int nst = static_cast<int>(s1 - s0);
  static_assert(sizeof(BatchItem) % 4 == 0, "items are copied as words");
  if (threadIdx.x < P.count * static_cast<int>(sizeof(BatchItem) / 4))
    reinterpret_cast<uint32_t*>(its)[threadIdx.x] = reinterpret_cast<const uint32_t*>(P.it)[threadIdx.x];
  if (threadIdx.x == 0) {
    for (int i = 0; i < P.ring; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kCons);
    }
    mbar_init(resfull, 1);
    mbar_init(resempty, 1);
    flags[0] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (nst <= 0) return;

  // position of the range's first stage: item, row block, stage within the row block
  int it0 = 0;
  while (it0 + 1 < P.count && its[it0 + 1].begin <= s0) ++it0;
  const uint32_t off0 = static_cast<uint32_t>(s0 - its[it0].begin);
  const int rb0 = static_cast<int>(off0 / static_cast<uint32_t>(its[it0].C));
  const int k0 = static_cast<int>(off0 % static_cast<uint32_t>(its[it0].C));

  if (warp == kCons) {
    // ==================================================================== producer warp
    if (lane == 0) {
      const uint32_t tx = static_cast<uint32_t>(kDWBytes + F::kKB * P.M * 128);  // whole boxes
      for (int q = 0; q < P.count; ++q) {
        tma_prefetch_desc(&P.w[q]);
        tma_prefetch_desc(&P.x[q]);
      }
      const int ring = P.ring;
      int it = it0, rb = rb0, kst = k0, C = its[it0].C;
      auto advance = [&]() {
        if (++kst == C) {
          kst = 0;
          if (++rb == its[it].RB) {
            rb = 0;
            ++it;
            if (it < P.count) C = its[it].C;
          }
        }
      };
      auto load_w = [&](int slot) {
        tma_load_2d(stg + slot * P.stage, &P.w[it], &full[slot], kst * 128, rb * kBRows);
      };
      const bool skipx = skip_x_loads();  // failure-path test hook: never set in normal use
      auto load_x = [&](int slot) {
        if (skipx) return;
        uint8_t* dst = stg + slot * P.stage + kDWBytes;
#pragma unroll
        for (int hb = 0; hb < F::kKB / 4; ++hb)
          tma_load_3d(dst + hb * P.xhalf, &P.x[it], &full[slot], 0, kst * F::kKB + 4 * hb, 0);
      };
      const int pre = nst < ring ? nst : ring;
      // weights are model constants: the first `pw` stages' weights are requested before the
      // wait for the previous kernel (their latency overlaps its tail), the rest after it (a
      // full ring of requests at once would queue the previous kernel's last L2 round trips)
      const int pw = pre < P.pre_w ? pre : P.pre_w;
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], tx);
        if (i < pw) load_w(i);
        advance();
      }
      pdl_wait_prior_grids();  // the activations may come from the previous kernel
      it = it0, rb = rb0, kst = k0, C = its[it0].C;
      for (int i = 0; i < pre; ++i) {
        if (i >= pw) load_w(i);
        load_x(i);
        advance();
      }
      int slot = 0;
      uint32_t ph = 0;  // parity of the slot's last completed `empty` phase
      bool fine = true;
      for (int i = pre; i < nst; ++i) {
        if (!mbar_wait(&empty[slot], ph)) {
          flags[0] = 1;
          fine = false;
          break;
        }
        mbar_arrive_expect_tx(&full[slot], tx);
        load_w(slot);
        load_x(slot);
        advance();
        if (++slot == ring) {
          slot = 0;
          ph ^= 1u;
        }
      }
      // All of this CTA's loads are issued.  The stages that the next call's CTA of this index
      // loads first (its ring fill) are requested into L2 now, while this launch computes: that
      // launch then starts on L2 hits instead of the HBM burst of every CTA's fill at once.
      if (fine && P.ncount > 0 && c < P.Gn) {
        const int64_t b0 = range_begin(c, P.Tn, P.Gn), b1 = range_begin(c + 1, P.Tn, P.Gn);
        const int nn = static_cast<int>(b1 - b0 < P.nring ? b1 - b0 : P.nring);
        int q = 0;
        while (q + 1 < P.ncount && P.nit[q + 1].begin <= b0) ++q;
        const uint32_t o = static_cast<uint32_t>(b0 - P.nit[q].begin);
        int qC = P.nit[q].C, qrb = static_cast<int>(o / static_cast<uint32_t>(qC)),
            qk = static_cast<int>(o % static_cast<uint32_t>(qC));
        for (int i = 0; i < nn && q < P.ncount; ++i) {
          tma_prefetch_l2_2d(&P.wn[q], qk * 128, qrb * kBRows);
          if (++qk == qC) {
            qk = 0;
            if (++qrb == P.nit[q].RB) {
              qrb = 0;
              if (++q < P.ncount) qC = P.nit[q].C;
            }
          }
        }
      }
    }
    return;
  }

  if (warp == kCons + 1) {
    // ==================================================================== epilogue warp
    // Walks the row blocks of the range in order.  Lane l owns rows 4l .. 4l + 3 of a block for
    // every token: one float4 of each token's row of `res` or of a workspace slot.  Per block:
    // the scale and bias of its rows are requested, then it waits until the consumers have put
    // the block's sum in `res`, writes y (a block finished in this CTA) or, for a block split
    // between CTAs, stores this CTA's partial in its workspace slot, frees `res` and counts
    // itself in; the last contributor adds the slots in K order and writes y.  Every load of
    // one slot is issued before the first add (one round trip per contributor: under the
    // weight stream an L2 round trip takes microseconds).  The consumers meanwhile go on with
    // the next stages: they only wait for `res` at their next block end.
    constexpr int kTok = 8 * NT;  // tokens a launch of this shape holds at most
    constexpr int kQ = kBRows / 4;  // float4 per token row of a slot
    constexpr int kCh = kSplitK ? 4 : 8;  // the eight-consumer kernel has 96 registers a thread
    pdl_wait_prior_grids();  // y and the workspace belong to the previous kernel until now
    int it = it0, rb = rb0, kst = k0, u = 0;
    bool ok = true;
    for (int i = 0; i < nst; ++i) {
      const BatchItem& I = its[it];
      if (kst == I.C - 1 || i == nst - 1) {
        const int64_t n0 = static_cast<int64_t>(rb) * kBRows + 4 * lane;
        float es[4], eb[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int64_t n = n0 + j;
          es[j] = 1.0f;
          eb[j] = 0.0f;
          if (n < I.N) {
            if (!kInt4) es[j] = __half2float(I.sc[n]);
            if (I.bias) eb[j] = __half2float(I.bias[n]);
          }
        }
        // y rows n0 .. n0 + 3 of one token from its four fp32 sums
        const bool vec = (I.N & 3) == 0 && (reinterpret_cast<uintptr_t>(I.y) & 7) == 0;
        auto put = [&](int tok, const float4& a) {
          const float r[4] = {a.x, a.y, a.z, a.w};
          __half h[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) h[j] = __float2half_rn(kInt4 ? r[j] + eb[j] : fmaf(r[j], es[j], eb[j]));
          __half* yp = I.y + static_cast<int64_t>(tok) * I.N + n0;
          if (vec && n0 + 3 < I.N) {
            uint2 pk;
            pk.x = static_cast<uint32_t>(__half_as_ushort(h[0])) | (static_cast<uint32_t>(__half_as_ushort(h[1])) << 16);
            pk.y = static_cast<uint32_t>(__half_as_ushort(h[2])) | (static_cast<uint32_t>(__half_as_ushort(h[3])) << 16);
            *reinterpret_cast<uint2*>(yp) = pk;
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (n0 + j < I.N) yp[j] = h[j];
          }
        };
        auto res4 = [&](int tok) { return *reinterpret_cast<const float4*>(res + tok * kBResPitch + 4 * lane); };
        if (ok) ok = mbar_wait_warp(resfull, static_cast<uint32_t>(u & 1));
        const bool abort = !ok || flags[0] != 0;
        const int64_t gB0 = I.begin + static_cast<int64_t>(rb) * I.C, gB1 = gB0 + I.C;  // the block's stages
        if (!abort && gB0 >= s0 && gB1 <= s1) {
#pragma unroll
          for (int q = 0; q < kTok; ++q)
            if (q < P.M) put(q, res4(q));
          __syncwarp();
          if (lane == 0) mbar_arrive(resempty);  // `res` is free again
        } else if (abort) {
          __syncwarp();
          if (lane == 0) mbar_arrive(resempty);
        } else {
          const int cf = range_owner(gB0, P.T, P.G), cl = range_owner(gB1 - 1, P.T, P.G);
          // Adds the contributors' partials in K order (CTA cf first) and writes y: kCh tokens at
          // a time (what the registers allow), all loads of a slot for them in flight together.
          // This CTA's own partial comes from `res` when `own` is set, else from its slot.
          auto sum_and_write = [&](bool own) {
#pragma unroll
            for (int q0 = 0; q0 < kTok; q0 += kCh) {
              if (q0 >= P.M) break;
              float4 v[kCh];
#pragma unroll
              for (int q = 0; q < kCh; ++q) v[q] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              for (int cc = cf; cc <= cl; ++cc) {  // K order: deterministic
                float4 t[kCh];
                if (own && cc == c) {
#pragma unroll
                  for (int q = 0; q < kCh; ++q)
                    if (q0 + q < P.M) t[q] = res4(q0 + q);
                } else {
                  const int64_t sl = 2 * static_cast<int64_t>(cc) + (gB0 <= range_begin(cc, P.T, P.G) ? 0 : 1);
                  const float4* src = reinterpret_cast<const float4*>(P.slots + sl * 16 * kBRows) + lane;
#pragma unroll
                  for (int q = 0; q < kCh; ++q)
                    if (q0 + q < P.M) t[q] = __ldcg(src + (q0 + q) * kQ);
                }
#pragma unroll
                for (int q = 0; q < kCh; ++q)
                  if (q0 + q < P.M) {
                    v[q].x += t[q].x;
                    v[q].y += t[q].y;
                    v[q].z += t[q].z;
                    v[q].w += t[q].w;
                  }
              }
#pragma unroll
              for (int q = 0; q < kCh; ++q)
                if (q0 + q < P.M) put(q0 + q, v[q]);
            }
          };
          // every other contributor already counted in (the usual case for the block that ends
          // a range: the CTA after this one finished its part at its start): this CTA is last
          // and needs neither its slot nor the atomic
          int all = 0;
          if (lane == 0) all = ld_acquire_gpu(&P.counters[cf]) == cl - cf;
          all = __shfl_sync(0xFFFFFFFFu, all, 0);
          if (all) {
            sum_and_write(true);
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(resempty);
              P.counters[cf] = 0;  // ready for the next call
            }
          } else {
            float4* mine = reinterpret_cast<float4*>(P.slots + (2 * static_cast<int64_t>(c) + (gB0 <= s0 ? 0 : 1)) * 16 * kBRows);
#pragma unroll
            for (int q = 0; q < kTok; ++q)
              if (q < P.M) mine[q * kQ + lane] = res4(q);
            __syncwarp();
            if (lane == 0) mbar_arrive(resempty);
            // the warp barrier orders every lane's partial before lane 0's release; the count's
            // acquire orders the other contributors' partials before the warp reads them
            int last = 0;
            if (lane == 0) last = atom_add_acq_rel_gpu(&P.counters[cf], 1) == cl - cf;
            last = __shfl_sync(0xFFFFFFFFu, last, 0);
            if (last) {
              __syncwarp();
              sum_and_write(false);
              if (lane == 0) P.counters[cf] = 0;  // ready for the next call
            }
          }
        }
        ++u;
      }
      if (++kst == I.C) {
        kst = 0;
        if (++rb == I.RB) {
          rb = 0;
          ++it;
        }
      }
    }
    return;
  }

  // ====================================================================== consumer warps
  const int g = lane >> 2, t = lane & 3;
  const int rs = warp & (kDRowSets - 1), hi = warp / kDRowSets;  // hi: K half (M <= 8) or token group
  const int sub_lo = kSplitK ? hi : 0, sub_hi = kSplitK ? hi + 1 : 2;
  const int Tb = TW < NT ? hi : 0;
  // activation row of this lane's token 8 (Tb + T) + g (B column g of token group Tb + T); a
  // lane past the last token reads the last token's row instead (its column is never stored),
  // so the loads need neither a predicate nor zero fill
  int xrow[TW];
#pragma unroll
  for (int T = 0; T < TW; ++T) xrow[T] = 4 * min(8 * (Tb + T) + g, P.M - 1);
  const int gp = (g >> 1) | ((g & 1) << 2);
  const int rw = rs * 16 * kDRT + gp;
  const DecLane L{g, t, gp, rw, sub_lo, sub_hi, Tb, P.four};

  float acc[kDRT][TW][4];
  auto zero_acc = [&]() {
#pragma unroll
    for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
      for (int T = 0; T < TW; ++T)
#pragma unroll
        for (int ci = 0; ci < 4; ++ci) acc[rt][T][ci] = 0.0f;
  };
  zero_acc();

  // The range is walked unit by unit (the stages of one row block that fall in this range); the
  // per-stage loop only waits, decodes, releases and moves the ring slot.
  int it = it0, rb = rb0, kst = k0, u = 0, left = nst;
  int slot = 0;
  uint32_t ph = 0;  // parity of the slot's next `full` phase
  bool ok = true;
  pdl_wait_prior_grids();          // x belongs to the previous kernel until now
  while (left > 0) {
    const BatchItem& I = its[it];
    const int C = I.C;
    const int n = C - kst < left ? C - kst : left;
    const int64_t row0 = static_cast<int64_t>(rb) * kBRows;
    const int64_t Nm = I.N, G = I.K >> 7;
    const __half* scm = I.sc;
    const uint8_t* zpm = I.zp;
    for (int j = 0; j < n; ++j) {
      if (ok) ok = mbar_wait_warp(&full[slot], ph);
      if (ok) {
        dec_stage<kInt4, NT, TW, kIL>(acc, stg + slot * P.stage, P.xhalf, L, xrow, static_cast<int64_t>(kst + j) * 2, row0,
                                 Nm, scm, zpm, G);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      } else {
        flags[0] = 1;  // a wait ran out (recorded in the device status word): results are void
      }
      if (++slot == P.ring) {
        slot = 0;
        ph ^= 1u;
      }
    }
    left -= n;

    // ------------------------------------------------------------------ finish the unit
    float v[kDRT][TW][4];
    dec_values<kInt4, TW>(acc, v);
    zero_acc();
    // this CTA's sum over its stages of the block, [token][row] in `res`, once the epilogue
    // warp has taken the previous block's; for M <= 8 the two K halves (warps 4-7, then 0-3)
    // are added in a fixed order
    if (u > 0 && ok) ok = mbar_wait_warp(resempty, static_cast<uint32_t>((u - 1) & 1));
    if (kSplitK && hi == 0) named_barrier_sync(1, kEp);
#pragma unroll
    for (int rt = 0; rt < kDRT; ++rt)
#pragma unroll
      for (int T = 0; T < TW; ++T)
#pragma unroll
        for (int ci = 0; ci < 4; ++ci) {
          float* dst = res + (8 * (Tb + T) + 2 * t + (ci & 1)) * kBResPitch + rw + 16 * rt + 8 * (ci >> 1);
          if (kSplitK && hi == 0)
            *dst += v[rt][T][ci];
          else
            *dst = v[rt][T][ci];
        }
    if (kSplitK && hi == 1) named_barrier_sync(1, kEp);
    named_barrier_sync(1, kEp);
    if (!ok) flags[0] = 1;
    if (threadIdx.x == 0) mbar_arrive(resfull);  // hand the block to the epilogue warp
    ++u;
    kst += n;
    if (kst == C) {
      kst = 0;
      if (++rb == I.RB) {
        rb = 0;
        ++it;
      }
    }
  }
}

// Threads: the consumer warps, the producer warp, the epilogue warp.
template <int CW>
constexpr int batch_threads() { return (CW + 2) * 32; }

// M <= 8, eight consumer warps (K halves split): two CTAs of ten warps per SM; five warps share
// one SM sub-partition's 16K registers, so a thread may use at most 102 (96 it is).
template <bool kInt4, bool kIL>
__global__ void __maxnreg__(96) batch_decode_kernel_m8(const __grid_constant__ BatchParams P) {
  batch_body<kInt4, 1, 1, 8, kIL>(P);
}

// M <= 8, four consumer warps, each over the whole stage (twice the MMAs per stage and warp).
template <bool kInt4, bool kIL>
__global__ void __launch_bounds__(batch_threads<4>(), 2) batch_decode_kernel_m8w4(const __grid_constant__ BatchParams P) {
  batch_body<kInt4, 1, 1, 4, kIL>(P);
}

template <bool kInt4, bool kIL>
__global__ void __launch_bounds__(batch_threads<4>(), 2) batch_decode_kernel_m16(const __grid_constant__ BatchParams P) {
  batch_body<kInt4, 2, 2, 4, kIL>(P);
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
int64_t tc_batch_workspace_bytes_for(int G);
int64_t batch_workspace_bytes() {
  const int sms = current_device_info().num_sms;
  const int64_t a = batch_workspace_bytes_for(kBCtasPerSm * sms), b = tc_batch_workspace_bytes_for(sms);
  return a > b ? a : b;
}

template <bool kInt4, bool kIL>
static cudaError_t launch_batch_t(const BatchLinear* items, int count, int64_t M, void* ws, int64_t ws_bytes,
                                  cudaStream_t s, const BatchNext& next) {
  using F = DecFmt<kInt4>;
  using L = BatchLayout<kInt4>;
  if (count < 1 || count > kBMaxItems || M < 1 || M > 16) return cudaErrorInvalidValue;
  const DeviceInfo di = current_device_info();
  BatchParams P;
  P.count = count;
  P.M = static_cast<int>(M);
  int64_t T = 0;
  for (int q = 0; q < count; ++q) {
    const BatchLinear& b = items[q];
    BatchItem& I = P.it[q];
    I.sc = b.sc;
    I.zp = b.zp;
    I.bias = b.bias;
    I.y = b.y;
    I.N = b.N;
    I.K = b.K;
    I.C = static_cast<int>((b.K + F::kStageK - 1) / F::kStageK);
    I.RB = static_cast<int>((b.N + kBRows - 1) / kBRows);
    I.begin = T;
    T += static_cast<int64_t>(I.C) * I.RB;
    const int64_t kbytes = kInt4 ? b.K / 2 : b.K / 4;
    if (!make_tmap_2d(&P.w[q], CU_TENSOR_MAP_DATA_TYPE_UINT8, b.w, static_cast<uint64_t>(kbytes),
                      static_cast<uint64_t>(b.N), static_cast<uint64_t>(kbytes), 128, kBRows,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const uint64_t dims[3] = {64, static_cast<uint64_t>(b.K / 64), static_cast<uint64_t>(M)};
    const uint64_t strides[2] = {128, static_cast<uint64_t>(b.K) * 2};
    const uint32_t box[3] = {64, 4, static_cast<uint32_t>(M)};
    if (!make_tmap_3d(&P.x[q], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, b.x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  for (int q = count; q < kBMaxItems; ++q) {
    P.w[q] = P.w[0];
    P.x[q] = P.x[0];
    P.it[q] = P.it[0];
    P.it[q].begin = T;  // never reached
  }
  const int Gmax = kBCtasPerSm * di.num_sms;
  if (ws_bytes < batch_workspace_bytes_for(Gmax)) return cudaErrorInvalidValue;
  P.T = T;
  P.G = static_cast<int>(T < Gmax ? T : Gmax);
  if (T * P.G >= (static_cast<int64_t>(1) << 32)) return cudaErrorInvalidValue;  // 32-bit range arithmetic
  P.xhalf = ((static_cast<int>(M) * 4 * 128 + 1023) / 1024) * 1024;
  P.four = 4u;
  P.pre_w = kBatchPreW;
  P.stage = kDWBytes + (F::kKB / 4) * P.xhalf;
  int ring = kDMaxRing;
  while (ring > 2 && L::bytes(ring, P.stage) > kDSmemBudget) --ring;
  P.ring = ring;
  const int smem = L::bytes(ring, P.stage);
  if (smem > kDSmemBudget) return cudaErrorInvalidValue;
  P.counters = reinterpret_cast<int*>(ws);
  P.slots = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + batch_counter_bytes(Gmax));
  // the next call's stage sequence, CTAs and ring depth, as its own launch will compute them
  P.ncount = 0;
  if (next.count > 0 && next.count <= kBMaxItems && next.M >= 1 && next.M <= 16) {
    int64_t Tn = 0;
    for (int q = 0; q < next.count; ++q) {
      const BatchLinear& b = next.items[q];
      const int64_t kbytes = kInt4 ? b.K / 2 : b.K / 4;
      if (!make_tmap_2d(&P.wn[q], CU_TENSOR_MAP_DATA_TYPE_UINT8, b.w, static_cast<uint64_t>(kbytes),
                        static_cast<uint64_t>(b.N), static_cast<uint64_t>(kbytes), 128, kBRows,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
      P.nit[q].begin = Tn;
      P.nit[q].C = static_cast<int>((b.K + F::kStageK - 1) / F::kStageK);
      P.nit[q].RB = static_cast<int>((b.N + kBRows - 1) / kBRows);
      Tn += static_cast<int64_t>(P.nit[q].C) * P.nit[q].RB;
    }
    if (Tn * (Tn < Gmax ? Tn : Gmax) < (static_cast<int64_t>(1) << 32)) {
      P.Tn = Tn;
      P.Gn = static_cast<int>(Tn < Gmax ? Tn : Gmax);
      const int xh = ((static_cast<int>(next.M) * 4 * 128 + 1023) / 1024) * 1024;
      const int st = kDWBytes + (F::kKB / 4) * xh;
      int rn = kDMaxRing;
      while (rn > 2 && L::bytes(rn, st) > kDSmemBudget) --rn;
      P.nring = rn;
      P.ncount = next.count;
    }
  }

  const bool m16 = M > 8;
  const bool w4 = !m16 && kBatchM8FourWarps;
  auto* kern = m16 ? batch_decode_kernel_m16<kInt4, kIL>
                   : w4 ? batch_decode_kernel_m8w4<kInt4, kIL> : batch_decode_kernel_m8<kInt4, kIL>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kDSmemBudget);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(P.G), 1, 1);
  cfg.blockDim = dim3(m16 || w4 ? batch_threads<4>() : batch_threads<8>(), 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

cudaError_t launch_tq_gemm_batch(const BatchLinear* items, int count, int64_t M, void* ws, int64_t ws_bytes,
                                 cudaStream_t s, bool interleaved, const BatchNext& next) {
  return interleaved ? launch_batch_t<false, true>(items, count, M, ws, ws_bytes, s, next)
                     : launch_batch_t<false, false>(items, count, M, ws, ws_bytes, s, next);
}

cudaError_t launch_w4g_gemm_batch(const BatchLinear* items, int count, int64_t M, void* ws, int64_t ws_bytes,
                                  cudaStream_t s, const BatchNext& next) {
  return launch_batch_t<true, false>(items, count, M, ws, ws_bytes, s, next);
}

}  // namespace tq

namespace tq {

// =============================================================================================
// Allocation-free batch entry point (tq_gemm_batch_noalloc)
// =============================================================================================
// Some callers cannot hand the batch call a workspace and must not allocate one: a custom
// operator behind an interface that passes only its inputs and outputs, or a process whose
// device memory is all reserved by its framework's caching allocator (a raw cudaMalloc there
// fails, or synchronises the device in the middle of a step).  For them the workspace lives in
// this file-scope device array, which every GPU that loads the library holds until the process
// exits.  Its size covers GPUs with up to kNoAllocMaxSms SMs (5.0 MiB).
constexpr int kNoAllocMaxSms = 160;
constexpr int64_t kNoAllocCounterBytes = ((static_cast<int64_t>(kBCtasPerSm) * kNoAllocMaxSms * 4 + 255) / 256) * 256;
constexpr int64_t kNoAllocScratchBytes =
    kNoAllocCounterBytes + 2 * static_cast<int64_t>(kBCtasPerSm) * kNoAllocMaxSms * 16 * kBRows * 4;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// The device address of the array on the current device.  In host code `g_noalloc_scratch` is
// only a host-side stand-in for the symbol (a kernel given it would fault, or silently use host
// memory): the address is looked up once per device with that device current, and cached.
static void* noalloc_scratch_on_current_device() {
  static std::atomic<void*> addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  void* p = addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
  addr[dev].store(p, std::memory_order_release);
  return p;
}

}  // namespace tq

extern "C" TQ_API int tq_gemm_batch_noalloc(const tq_linear* items, int count, int64_t M, void* stream) {
  // the argument checks of tq_gemm_batch, before any device work
  if (count < 1 || count > tq::kBatchMaxItems || M < 0 || M > tq::kBatchMaxM) return TQ_ERR_SHAPE;
  if (!items) return TQ_ERR_NULL;
  if (M == 0) return TQ_OK;
  // the workspace this device needs must fit in the static array
  if (tq::batch_workspace_bytes() > tq::kNoAllocScratchBytes) return TQ_ERR_SHAPE;
  void* ws = tq::noalloc_scratch_on_current_device();
  if (!ws) return TQ_ERR_CUDA;
  // every call shares the array: the arrival counters must start at zero (a completed call
  // leaves them zero, a failed one may not), so they are cleared on the caller's stream
  if (cudaMemsetAsync(ws, 0, static_cast<size_t>(tq::kNoAllocCounterBytes), reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return TQ_ERR_CUDA;
  return gemm_batch_impl<false>(items, count, M, ws, static_cast<size_t>(tq::kNoAllocScratchBytes), TQ_BATCH_AUTO,
                                stream);
}
