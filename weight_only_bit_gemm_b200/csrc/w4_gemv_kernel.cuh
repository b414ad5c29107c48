// w4_gemv_kernel.cuh -- decode path (M <= 32 tokens).
//
// Every warp is an independent streaming worker.  The work units are
// (32-row pair of row groups, 128-channel stage) pairs, numbered row-pair
// major; warp w owns the contiguous range of q + (w < r) units that starts at
// w q + min(w, r) (U = q W + r units, W warps).  Each lane copies its share
// of a unit's packed codes (four 16-byte vectors: 1 KB per row group per warp)
// and a few lanes the row groups' scale and zero bytes into the warp's own
// shared-memory ring with cp.async, three units ahead; the warp then reads the
// unit back into registers, dequantizes into the A fragments of warp-level
// m16n8k16 bf16 MMAs (one activation fragment serves both row groups) and
// accumulates in fp32 registers.  No producer warp and no barriers between
// warps: the only synchronisation is the deterministic reduction over the
// warps that share a row pair, in two levels.  Warps of one CTA combine in
// shared memory (a CTA-scope arrival counter; the last local arrival sums
// the warps' partials in warp order); a row pair that several CTAs share is
// then combined once per CTA through global memory (a partial slot per CTA
// and a device-scope arrival counter; the last CTA sums them in CTA order).
// Measured on B200: the number of partials the last arrival reads from
// global memory, not the arithmetic, sets the tail of each call.
//
// Why not tcgen05 here: a tcgen05.mma of kind::f16 occupies the SM's tensor
// core for ~200 cycles whatever its N (measured on B200 for N = 16..256), so a
// 16-token tile consumes only 128 x 16 weights per 200 cycles per SM (about
// 1.4 TB/s of 4-bit weights on 148 SMs).
//
// Instruction economy matters more than anything else here: the SM issues
// one warp instruction per cycle per sub-partition, and most of the integer
// and bf16x2 instructions this loop needs run at half rate on B200.  So all
// per-launch divisions are by multiplication with host-made constants, loop
// counters are 32-bit, two row groups share each activation load, and
// activations are loaded without predicates (rows past M are clamped to row
// M - 1; the MMA columns they feed are never stored).
//
// The first units' weights are requested before the launch dependency on
// the previous kernel resolves (weights are constant model state; X, Y and
// the workspace are touched only after it), so a chain of these kernels keeps
// HBM busy across kernel boundaries.
//
// Channel order: inside each 16-channel block, lane (g, u) holds channels
// 4u..4u+3 (see w4_prepack.cuh) in the MMA's k slots {2u, 2u+1, 2u+8, 2u+9};
// the B fragment is loaded with the same permutation (X[token][4u..4u+3] as
// one 64-bit load), so the product over the block is unchanged.
#pragma once

#include "w4_gemm.cuh"

namespace w4 {

struct GemvArgs {
  const uint8_t* Wp;        // prepacked weights
  const uint16_t* X;        // bf16 [M, K] (act-order: already gathered)
  const float* s2;          // NF4 second-level scales
  const float* mean;        // NF4 mean-offset double quantization: run means
  uint16_t* Y;              // bf16 [M, N]
  float* partial;           // [row group][slot][32 lanes][4 NB] fp32
  unsigned int* counter;    // [row group] arrivals
  int M, N, K;
  int KS;                   // stages (128 channels) per tile row
  int max_slots;            // partial slots per row group
  uint32_t q, r;            // units per warp: q + (w < r)
  FastDiv32 by_ks, by_q, by_q1;
  FastDivIdx by_dq;          // NF4: 64-block index -> s2 index
  int dq_group;             // NF4: 64-blocks per second-level scale
  int table;                // NF4 layout: level table (kTableNf4 / kTableFp4)
  // buffer extents, read only by the bounds-checked build
  unsigned long long wp_bytes, partial_floats, s2_count;
};

// Row groups (16 rows each) per decode work unit: two share each activation
// fragment.  Accumulator sets per (row group, token block): with one token
// block two alternate between consecutive words so that MMAs do not wait on
// each other; with two or four token blocks the blocks themselves give that
// independence, and one set keeps the registers within budget.
__host__ __device__ constexpr int gemv_row_groups(int) { return 2; }

// CTA shape of the decode kernel: warps per CTA and resident CTAs per SM (one
// wave of CTAs covers the GPU; the planner sizes the grid from these).  One
// CTA of 16 warps per SM (128 registers a thread): measured on B200, the
// same warps as two CTAs of 8 per SM but half as many CTA partials per row
// pair in the global level of the reduction, 0.6 us less per call.
constexpr int kGemvWarps = 16;
constexpr int kGemvCtasPerSm = 1;
__host__ __device__ constexpr int gemv_acc_split(int NB) { return NB >= 2 ? 1 : 2; }

template <int NB_, int FMT_, int G_, bool MEAN_ = false>
struct GemvCfg {
  static constexpr int NB = NB_;   // token blocks of 8
  static constexpr int MT = 8 * NB;
  static constexpr int FMT = FMT_;
  static constexpr int G = G_;
  static constexpr bool MEAN = MEAN_;  // NF4 layout: mean-offset absmax constants
  static constexpr int kStageBytes = FMT == kFmtInt4 ? int4_stage_bytes(G) : nf4_stage_bytes();
  static constexpr int kWarps = kGemvWarps;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kMinBlocks = kGemvCtasPerSm;
  // groups per 128-channel stage (INT4); NF4 keeps its absmax pairs in sp[0] / zp[0]
  static constexpr int kNq = FMT == kFmtInt4 ? 128 / G : 1;
  static constexpr int kDepth = 4;  // per-warp ring slots (3 units in flight)
  static constexpr int kScaleBytes = FMT == kFmtInt4 ? 32 * kNq : 32;  // NF4: absmax pairs
  static constexpr int kZeroBytes = FMT == kFmtInt4 ? 8 * kNq : 0;
  static constexpr int kRG = gemv_row_groups(NB);  // row groups per work unit
  static constexpr int kAS = gemv_acc_split(NB);  // accumulators per (row group, token block)
  static constexpr int kSlot = kRG * 1024 + (kRG * (kScaleBytes + kZeroBytes) + 15) / 16 * 16;
  static constexpr int kRingBytes = kWarps * kDepth * kSlot;
  // CTA-level reduction (up to two token blocks; the slots of four would not
  // fit beside the ring): two partial slots per warp (the warp's first and
  // last row-pair segments), [slot][V/4][32 lanes] float4, and one arrival
  // counter per warp (the row pair that ends the warp's range).
  static constexpr bool kCtaReduce = NB <= 2;
  static constexpr int kV = kRG * NB * 4;  // partial floats per lane
  static constexpr int kRedBytes = kCtaReduce ? kWarps * 2 * 32 * kV * 4 : 0;
  static constexpr int kSmemBytes = kRingBytes + kRedBytes + kWarps * 4;
  static_assert(kSmemBytes + 64 <= 227 * 1024, "shared memory of one CTA");
};

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&d)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One 128-channel stage of a lane's R row groups in registers.
template <class C>
struct StageRegs {
  uint4 c[C::kRG][2];           // code words of channel blocks 0..3 and 4..7
  uint32_t sp[C::kRG][C::kNq];  // INT4: scale pairs per group; NF4: absmax pair, block 0
  uint32_t zp[C::kRG][C::kNq];  // INT4: zero pairs; NF4: absmax pair, block 1
};

template <class C>
__device__ __forceinline__ void issue_stage(const uint8_t* __restrict__ blk, uint32_t slot, int rpl,
                                            int lane, const GemvArgs& args) {
  constexpr int R = C::kRG;
  const int rgl0 = rpl * R;
  if (kChecked && !in_bounds(static_cast<unsigned long long>(blk - args.Wp) + C::kStageBytes - 1,
                             args.wp_bytes))
    return;
  const uint8_t* cb = blk + rgl0 * 1024 + lane * 16;
#pragma unroll
  for (int i = 0; i < 2 * R; ++i) cp_async16(slot + i * 512 + lane * 16, cb + i * 512);
  constexpr int sbytes = R * C::kScaleBytes;
  constexpr int sl = sbytes / 16;
  if constexpr (C::FMT == kFmtInt4) {
    constexpr int gps = C::kNq;
    const uint8_t* sc = blk + kCodeBytes + rgl0 * C::kScaleBytes;
    const uint8_t* zc = blk + kCodeBytes + kTileRows * gps * 2 + rgl0 * C::kZeroBytes;
    if (lane < sl) cp_async16(slot + R * 1024 + lane * 16, sc + lane * 16);
    constexpr int zbytes = R * C::kZeroBytes;
    if constexpr (zbytes == 8) {
      if (lane == sl) cp_async8(slot + R * 1024 + sbytes, zc);
    } else {
      const int zl = lane - sl;
      if (zl >= 0 && zl < zbytes / 16) cp_async16(slot + R * 1024 + sbytes + zl * 16, zc + zl * 16);
    }
  } else {
    if (lane < sl) cp_async16(slot + R * 1024 + lane * 16, blk + kCodeBytes + rgl0 * 32 + lane * 16);
  }
}

template <class C>
__device__ __forceinline__ void read_stage(const uint8_t* slot, StageRegs<C>& r, int lane) {
  constexpr int R = C::kRG;
  const int g = lane >> 2;
#pragma unroll
  for (int rr = 0; rr < R; ++rr) {
    r.c[rr][0] = *reinterpret_cast<const uint4*>(slot + rr * 1024 + lane * 16);
    r.c[rr][1] = *reinterpret_cast<const uint4*>(slot + rr * 1024 + 512 + lane * 16);
    if constexpr (C::FMT == kFmtInt4) {
#pragma unroll
      for (int q = 0; q < C::kNq; ++q) {
        r.sp[rr][q] = *reinterpret_cast<const uint32_t*>(slot + R * 1024 + rr * C::kScaleBytes + (q * 8 + g) * 4);
        r.zp[rr][q] = slot[R * 1024 + R * C::kScaleBytes + rr * C::kZeroBytes + q * 8 + g];
      }
    } else {
      r.sp[rr][0] = *reinterpret_cast<const uint16_t*>(slot + R * 1024 + rr * 32 + g * 2);
      r.zp[rr][0] = *reinterpret_cast<const uint16_t*>(slot + R * 1024 + rr * 32 + (8 + g) * 2);
    }
  }
}

// Words [W0, W0 + NW) of one 64-channel half for the R row groups: one
// activation fragment per word index serves every row group.
// Activation fragments of one 64-channel half: either loaded word by word
// as the MMAs need them (XHalf::ptr) or held in registers, loaded ahead
// (XHalf::reg).  Lane: 8 bytes per word and token block.
template <class C>
struct XHalf {
  const uint16_t* ptr[C::NB];
  uint2 reg[4][C::NB];
};

// Whether a decode configuration holds the next stage's activation fragments
// in registers (loaded while the current stage computes).  Measured on B200:
// faster with one token block, not with two; four would spill.
template <class C>
__host__ __device__ constexpr bool gemv_x_ahead() { return C::NB == 1; }

template <class C, int W0, int NW>
__device__ __forceinline__ void mma_words(const uint32_t (&words)[C::kRG][4],
                                          const Int4Dq (&p0)[C::kRG], const Int4Dq (&p1)[C::kRG],
                                          const float (&a0)[C::kRG], const float (&a1)[C::kRG],
                                          uint32_t tb, const XHalf<C>& xs,
                                          float (&acc)[C::kRG][C::kAS][C::NB][4]) {
#pragma unroll
  for (int w = W0; w < W0 + NW; ++w) {
    uint2 b[C::NB];
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
      b[nb] = gemv_x_ahead<C>() ? xs.reg[w][nb]
                                : __ldg(reinterpret_cast<const uint2*>(xs.ptr[nb] + w * 16));
#pragma unroll
    for (int rr = 0; rr < C::kRG; ++rr) {
      uint32_t pr[4];
      if constexpr (C::FMT == kFmtInt4) {
        int4_dq_word(words[rr][w], p0[rr], p1[rr], pr);
      } else {
        nf4_dq_word(words[rr][w], a0[rr], a1[rr], tb, pr);
      }
      const uint32_t afrag[4] = {pr[0], pr[2], pr[1], pr[3]};
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb) mma_m16n8k16_bf16(acc[rr][w % C::kAS][nb], afrag, b[nb].x, b[nb].y);
    }
  }
}

// Warp owning unit u.
__device__ __forceinline__ uint32_t owner_of(uint32_t u, const GemvArgs& a) {
  const uint32_t big = a.r * (a.q + 1);  // units of the first r warps
  return u < big ? fast_div(u, a.by_q1) : a.r + fast_div(u - big, a.by_q);
}

// First unit after the range of warp w.
__device__ __forceinline__ uint32_t range_end(uint32_t w, const GemvArgs& a) {
  return w * a.q + (w < a.r ? w : a.r) + a.q + (w < a.r ? 1u : 0u);
}

// Shared-memory state of the CTA-level reduction.
struct CtaRed {
  float4* part;            // [warp][kind][V/4][32 lanes]
  unsigned int* count;     // [warp]: arrivals for the row pair that ends its range
};

// Global level: this lane's partial `tot` in slot `slot` of row pair rpg,
// `contrib` slots in all; returns true (with tot the full sum, added in slot
// order) for the last of them to arrive, false for the others.
template <class C>
__device__ __forceinline__ bool global_combine(const GemvArgs& args,
                                               float (&tot)[C::kRG][C::NB][4], int rpg,
                                               uint32_t slot, uint32_t contrib, int lane) {
  constexpr int R = C::kRG;
  constexpr int V = C::kV;
  float* dst = args.partial + ((static_cast<size_t>(rpg) * args.max_slots + slot) * 32 + lane) * V;
  if (kChecked &&
      !(in_bounds(((static_cast<unsigned long long>(rpg) * args.max_slots + contrib - 1) * 32 + lane) * V + V - 1,
                  args.partial_floats) &&
        in_bounds(slot, contrib) && in_bounds(static_cast<unsigned long long>(rpg) * 4 + 3, 65536ull * 4)))
    return false;
#pragma unroll
  for (int rr = 0; rr < R; ++rr)
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
      *reinterpret_cast<float4*>(dst + (rr * C::NB + nb) * 4) =
          make_float4(tot[rr][nb][0], tot[rr][nb][1], tot[rr][nb][2], tot[rr][nb][3]);
  // The warp barrier orders every lane's partial before lane 0's release
  // (the arrival) and, on the last arrival, lane 0's acquire before every
  // lane's reads of the other partials (the shuffle carries the count only
  // as a value).
  __syncwarp();
  unsigned prev = 0;
  if (lane == 0) prev = atom_add_acq_rel_gpu(args.counter + rpg, 1u);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  __syncwarp();
  if (prev != contrib - 1) return false;
#pragma unroll
  for (int rr = 0; rr < R; ++rr)
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
      for (int j = 0; j < 4; ++j) tot[rr][nb][j] = 0.0f;
  const float* base = args.partial + (static_cast<size_t>(rpg) * args.max_slots * 32 + lane) * V;
  for (uint32_t sp = 0; sp < contrib; ++sp) {
#pragma unroll
    for (int rr = 0; rr < R; ++rr)
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(
            base + static_cast<size_t>(sp) * 32 * V + (rr * C::NB + nb) * 4));
        tot[rr][nb][0] += v.x;
        tot[rr][nb][1] += v.y;
        tot[rr][nb][2] += v.z;
        tot[rr][nb][3] += v.w;
      }
  }
  if (lane == 0) args.counter[rpg] = 0u;
  return true;
}

// The warp's sums over units [seg0, seg1) of row pair rpg (its range ends at
// unit wend) go to Y, directly when the warp covered the whole row pair,
// otherwise through the two-level reduction.
template <class C>
__device__ __forceinline__ void flush_row_group(const GemvArgs& args,
                                                float (&acc)[C::kRG][C::kAS][C::NB][4], int rpg,
                                                uint32_t seg0, uint32_t seg1, uint32_t wid,
                                                uint32_t wend, int lane, const CtaRed& cr) {
  constexpr int R = C::kRG;
  const int g = lane >> 2, u = lane & 3;
  float tot[R][C::NB][4];
#pragma unroll
  for (int rr = 0; rr < R; ++rr)
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        tot[rr][nb][j] = C::kAS == 2 ? acc[rr][0][nb][j] + acc[rr][C::kAS - 1][nb][j] : acc[rr][0][nb][j];
        acc[rr][0][nb][j] = 0.0f;
        acc[rr][C::kAS - 1][nb][j] = 0.0f;
      }
  const uint32_t rs = static_cast<uint32_t>(rpg) * static_cast<uint32_t>(args.KS);
  const uint32_t re = rs + static_cast<uint32_t>(args.KS);
  bool write_y = true;
  if (seg0 != rs || seg1 != re) {
    const uint32_t first = owner_of(rs, args);     // warps that touch the row pair
    const uint32_t last = owner_of(re - 1, args);
    const uint32_t cta_w0 = blockIdx.x * C::kWarps;
    const uint32_t cta_w1 = cta_w0 + C::kWarps - 1;
    bool done = false;  // the row pair lies within this CTA and has been summed here
    if constexpr (C::kCtaReduce) {
      const uint32_t lw0 = first > cta_w0 ? first : cta_w0;
      const uint32_t lw1 = last < cta_w1 ? last : cta_w1;
      if (lw1 > lw0) {
        // level 1: deposit in this warp's slot; the last local arrival sums.
        // Slot kind 1 holds a warp's last segment (the one ending its range),
        // kind 0 its first segment when that ends earlier.
        const uint32_t kind = seg1 == wend ? 1u : 0u;
        float4* mine = cr.part + ((wid - cta_w0) * 2 + kind) * (C::kV / 4) * 32 + lane;
#pragma unroll
        for (int rr = 0; rr < R; ++rr)
#pragma unroll
          for (int nb = 0; nb < C::NB; ++nb)
            mine[(rr * C::NB + nb) * 32] =
                make_float4(tot[rr][nb][0], tot[rr][nb][1], tot[rr][nb][2], tot[rr][nb][3]);
        __syncwarp();
        unsigned prev = 0;
        if (lane == 0) {
          asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                       : "=r"(prev)
                       : "r"(smem_u32(cr.count + (lw0 - cta_w0)))
                       : "memory");
        }
        prev = __shfl_sync(0xffffffffu, prev, 0);
        __syncwarp();
        if (prev != lw1 - lw0) return;
        // the first local contributor's range ends inside the row pair and so
        // do the middle ones' (kind 1); the last one's segment is its last
        // one only if its range ends inside the row pair too
        const uint32_t kind_last = range_end(lw1, args) <= re ? 1u : 0u;
#pragma unroll
        for (int rr = 0; rr < R; ++rr)
#pragma unroll
          for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
            for (int j = 0; j < 4; ++j) tot[rr][nb][j] = 0.0f;
        for (uint32_t w = lw0; w <= lw1; ++w) {
          const uint32_t k = w < lw1 ? 1u : kind_last;
          const float4* src = cr.part + ((w - cta_w0) * 2 + k) * (C::kV / 4) * 32 + lane;
#pragma unroll
          for (int rr = 0; rr < R; ++rr)
#pragma unroll
            for (int nb = 0; nb < C::NB; ++nb) {
              const float4 v = src[(rr * C::NB + nb) * 32];
              tot[rr][nb][0] += v.x;
              tot[rr][nb][1] += v.y;
              tot[rr][nb][2] += v.z;
              tot[rr][nb][3] += v.w;
            }
        }
        done = first >= cta_w0 && last <= cta_w1;
      }
    }
    if (!done) {
      // level 2, through global memory: one partial per CTA (per warp
      // without the CTA level)
      const uint32_t per = C::kCtaReduce ? C::kWarps : 1u;
      const uint32_t unit0 = first / per, unit1 = last / per;
      const uint32_t me = C::kCtaReduce ? blockIdx.x : wid;
      write_y = global_combine<C>(args, tot, rpg, me - unit0, unit1 - unit0 + 1, lane);
    }
  }
  if (write_y) {
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      const int r0 = (rpg * R + rr) * 16 + g;
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int m = nb * 8 + 2 * u + (j & 1);
          const int nn = r0 + (j >> 1) * 8;
          if (m < args.M && nn < args.N)
            args.Y[static_cast<size_t>(m) * args.N + nn] =
                __bfloat16_as_ushort(__float2bfloat16_rn(tot[rr][nb][j]));
        }
    }
  }
}

// NF4: per row of the lane, the second-level scale it last looked up and the
// run of 64-blocks (relative to the row's first block) that scale covers.
// Consecutive stages of a row stay in one run for up to dq_group blocks, so a
// scale is loaded once per run instead of once per stage, off the critical
// path of every other stage.
template <class C>
struct S2Cache {
  int rpg = -1;
  int lo[C::kRG][2], hi[C::kRG][2];
  float v[C::kRG][2];
  float mu[C::kRG][2];  // the run's mean (mean-offset constants only)
};

// Registers of half h of stage st <- its activation fragments.
template <class C>
__device__ __forceinline__ void load_x_half(const uint16_t* const (&xrow)[C::NB], int st, int h,
                                            XHalf<C>& xh) {
#pragma unroll
  for (int w = 0; w < 4; ++w)
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
      xh.reg[w][nb] = __ldg(reinterpret_cast<const uint2*>(xrow[nb] + st * kStageK + h * 64 + w * 16));
}

// One stage of a lane's row groups.  With gemv_x_ahead, xf holds this
// stage's activation fragments on entry and, as each half is done with, that
// half of the next stage `nst` (if has_next) is loaded in its place.
template <class C>
__device__ __forceinline__ void stage_compute(const GemvArgs& args, const StageRegs<C>& cur,
                                              int rpg, int st, int g,
                                              const uint16_t* const (&xrow)[C::NB], int nst,
                                              bool has_next, XHalf<C> (&xf)[2], uint32_t tb,
                                              S2Cache<C>& sc,
                                              float (&acc)[C::kRG][C::kAS][C::NB][4]) {
  constexpr int R = C::kRG;
  const int k0 = st * kStageK;
  if constexpr (!gemv_x_ahead<C>()) {
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb) {
      xf[0].ptr[nb] = xrow[nb] + k0;
      xf[1].ptr[nb] = xrow[nb] + k0 + 64;
    }
  }
  const bool nsecond = has_next && nst * kStageK + 64 < args.K;
  auto reload = [&](int h) {
    if constexpr (gemv_x_ahead<C>()) {
      if (h == 0 ? has_next : nsecond) load_x_half<C>(xrow, nst, h, xf[h]);
    }
  };
  const XHalf<C>& xa = xf[0];
  const XHalf<C>& xb = xf[1];
  uint32_t w0[R][4], w1[R][4];
#pragma unroll
  for (int rr = 0; rr < R; ++rr) {
    w0[rr][0] = cur.c[rr][0].x; w0[rr][1] = cur.c[rr][0].y; w0[rr][2] = cur.c[rr][0].z; w0[rr][3] = cur.c[rr][0].w;
    w1[rr][0] = cur.c[rr][1].x; w1[rr][1] = cur.c[rr][1].y; w1[rr][2] = cur.c[rr][1].z; w1[rr][3] = cur.c[rr][1].w;
  }
  const bool second = k0 + 64 < args.K;
  const float fz[R] = {};
  if constexpr (C::FMT == kFmtInt4) {
#pragma unroll
    for (int q = 0; q < C::kNq; ++q) {
      if (q >= C::kNq / 2 && C::kNq > 1 && !second) break;
      Int4Dq e0[R], e1[R];
#pragma unroll
      for (int rr = 0; rr < R; ++rr) int4_dq_params2(cur.sp[rr][q], cur.zp[rr][q], e0[rr], e1[rr]);
      if constexpr (C::G == 128) {
        mma_words<C, 0, 4>(w0, e0, e1, fz, fz, tb, xa, acc);
        reload(0);
        if (second) mma_words<C, 0, 4>(w1, e0, e1, fz, fz, tb, xb, acc);
      } else if constexpr (C::G == 64) {
        if (q == 0) {
          mma_words<C, 0, 4>(w0, e0, e1, fz, fz, tb, xa, acc);
          reload(0);
        } else {
          mma_words<C, 0, 4>(w1, e0, e1, fz, fz, tb, xb, acc);
        }
      } else {
        if (q == 0) {
          mma_words<C, 0, 2>(w0, e0, e1, fz, fz, tb, xa, acc);
        } else if (q == 1) {
          mma_words<C, 2, 2>(w0, e0, e1, fz, fz, tb, xa, acc);
          reload(0);
        } else if (q == 2) {
          mma_words<C, 0, 2>(w1, e0, e1, fz, fz, tb, xb, acc);
        } else {
          mma_words<C, 2, 2>(w1, e0, e1, fz, fz, tb, xb, acc);
        }
      }
    }
    reload(1);
  } else {
    const int kb64 = args.K / 64;
    if (sc.rpg != rpg) {  // a new row group unit: forget the runs
      sc.rpg = rpg;
#pragma unroll
      for (int rr = 0; rr < R; ++rr)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          sc.lo[rr][hf] = 0;
          sc.hi[rr][hf] = 0;
          sc.v[rr][hf] = 0.0f;
          sc.mu[rr][hf] = 0.0f;
        }
    }
    float a0[2][R], a1[2][R];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int blk = st * 2 + h;
#pragma unroll
      for (int rr = 0; rr < R; ++rr) {
        const uint32_t pair = h == 0 ? cur.sp[rr][0] : cur.zp[rr][0];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int r = (rpg * R + rr) * 16 + g + 8 * hf;
          float a = 0.0f;
          if (blk < kb64 && r < args.N) {
            if (blk < sc.lo[rr][hf] || blk >= sc.hi[rr][hf]) {
              const unsigned long long rowb = static_cast<unsigned long long>(r) * kb64;
              unsigned long long idx = fast_div(rowb + static_cast<unsigned long long>(blk), args.by_dq);
              if (!in_bounds(idx, args.s2_count)) idx = 0;
              sc.v[rr][hf] = __ldg(args.s2 + idx);
              if constexpr (C::MEAN) sc.mu[rr][hf] = __ldg(args.mean + idx);
              const long long lo = static_cast<long long>(idx * static_cast<unsigned long long>(args.dq_group)) -
                                   static_cast<long long>(rowb);
              sc.lo[rr][hf] = static_cast<int>(lo);
              sc.hi[rr][hf] = static_cast<int>(lo + args.dq_group);
            }
            a = absmax_from_code<C::MEAN>(hf == 0 ? pair : (pair >> 8), sc.v[rr][hf],
                                          sc.mu[rr][hf]);
          }
          if (hf == 0) a0[h][rr] = a; else a1[h][rr] = a;
        }
      }
    }
    Int4Dq none[R] = {};
    mma_words<C, 0, 4>(w0, none, none, a0[0], a1[0], tb, xa, acc);
    reload(0);
    if (second) mma_words<C, 0, 4>(w1, none, none, a0[1], a1[1], tb, xb, acc);
    reload(1);
  }
}

// One warp's whole share of the launch (returns when the warp is done).
template <class C>
__device__ __forceinline__ void decode_warp(const GemvArgs& args, const CtaRed& cr,
                                            uint8_t* w4_gemv_smem, const float* Ts) {
  constexpr int R = C::kRG;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, u = lane & 3;
  const uint32_t wid = blockIdx.x * C::kWarps + (threadIdx.x >> 5);
  const uint32_t ua = wid * args.q + (wid < args.r ? wid : args.r);
  const int left = static_cast<int>(args.q) + (wid < args.r ? 1 : 0);
  if (left == 0) return;
  const int KS = args.KS;
  constexpr int kPairsPerTile = 8 / R;

  const uint16_t* xrow[C::NB];
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb) {
    const int row = min(nb * 8 + g, args.M - 1);
    xrow[nb] = args.X + static_cast<size_t>(row) * args.K + 4 * u;
    // the last fragment of the row: channels (K/16 - 1) * 16 + 4u .. + 3
    if (kChecked && !in_bounds(static_cast<unsigned long long>(row) * args.K + (args.K - 16) + 4 * u + 3,
                               static_cast<unsigned long long>(args.M) * args.K))
      return;
  }

  const int rpg0 = static_cast<int>(fast_div(ua, args.by_ks));
  const int st0 = static_cast<int>(ua) - rpg0 * KS;
  int pf_rpg = rpg0, pf_st = st0;
  const uint8_t* pf_ptr =
      args.Wp + (static_cast<size_t>(pf_rpg / kPairsPerTile) * KS + pf_st) * C::kStageBytes;
  auto advance = [&]() {
    if (++pf_st == KS) {
      pf_st = 0;
      ++pf_rpg;
      pf_ptr = args.Wp + static_cast<size_t>(pf_rpg / kPairsPerTile) * KS * C::kStageBytes;
    } else {
      pf_ptr += C::kStageBytes;
    }
  };

  uint8_t* ring = w4_gemv_smem + (threadIdx.x >> 5) * (C::kDepth * C::kSlot);
  const uint32_t ring_s = static_cast<uint32_t>(__cvta_generic_to_shared(ring));
#pragma unroll
  for (int i = 0; i < C::kDepth - 1; ++i) {
    if (i < left) {
      issue_stage<C>(pf_ptr, ring_s + i * C::kSlot, pf_rpg % kPairsPerTile, lane, args);
      advance();
    }
    cp_async_commit();
  }
  grid_dep_wait();  // X, Y and the workspace may belong to the previous kernel

  float acc[R][C::kAS][C::NB][4];
#pragma unroll
  for (int rr = 0; rr < R; ++rr)
#pragma unroll
    for (int e = 0; e < C::kAS; ++e)
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[rr][e][nb][j] = 0.0f;

  // activation fragments of the first stage (X is read only after the wait)
  XHalf<C> xf[2];
  if constexpr (gemv_x_ahead<C>()) {
    load_x_half<C>(xrow, st0, 0, xf[0]);
    if (st0 * kStageK + 64 < args.K) load_x_half<C>(xrow, st0, 1, xf[1]);
  }

  S2Cache<C> s2c;  // NF4 only (unused, and removed, for INT4)
  int rpg = rpg0, st = st0;
  uint32_t seg0 = ua;
  int cs = 0;
  for (int n = 0; n < left; ++n) {
    cp_async_wait<C::kDepth - 2>();
    __syncwarp();
    StageRegs<C> cur;
    read_stage<C>(ring + cs * C::kSlot, cur, lane);
    if (n + C::kDepth - 1 < left) {
      const int is = cs == 0 ? C::kDepth - 1 : cs - 1;
      issue_stage<C>(pf_ptr, ring_s + is * C::kSlot, pf_rpg % kPairsPerTile, lane, args);
      advance();
    }
    cp_async_commit();
    cs = cs + 1 == C::kDepth ? 0 : cs + 1;
    const int nst = st == KS - 1 ? 0 : st + 1;
    stage_compute<C>(args, cur, rpg, st, g, xrow, nst, n + 1 < left, xf, smem_u32(Ts), s2c,
                     acc);
    if (st == KS - 1 || n + 1 == left) {
      const uint32_t seg1 = ua + static_cast<uint32_t>(n) + 1;
      flush_row_group<C>(args, acc, rpg, seg0, seg1, wid, ua + static_cast<uint32_t>(left), lane,
                         cr);
      ++rpg;
      st = 0;
      seg0 = seg1;
    } else {
      ++st;
    }
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, C::kMinBlocks) w4_gemv_kernel(const GemvArgs args) {
  __shared__ __align__(256) float Ts[16];  // NF4 / FP4 levels (see nf4_dq_word)
  extern __shared__ __align__(16) uint8_t w4_gemv_smem[];
  CtaRed cr;
  cr.part = reinterpret_cast<float4*>(w4_gemv_smem + C::kRingBytes);
  cr.count = reinterpret_cast<unsigned int*>(w4_gemv_smem + C::kRingBytes + C::kRedBytes);
  if (C::FMT == kFmtNf4 && threadIdx.x < 16) Ts[threadIdx.x] = level_value(args.table, threadIdx.x);
  // the level addresses need a 256-byte-aligned table (bounds-checked build: verified)
  if (C::FMT == kFmtNf4 && kChecked && threadIdx.x == 0) in_bounds(smem_u32(Ts) & 0xFFu, 1u);
  if (threadIdx.x < C::kWarps) cr.count[threadIdx.x] = 0u;
  __syncthreads();
  grid_dep_launch();
  decode_warp<C>(args, cr, w4_gemv_smem, Ts);
}

}  // namespace w4
