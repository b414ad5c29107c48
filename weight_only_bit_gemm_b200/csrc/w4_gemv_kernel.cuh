// w4_gemv_kernel.cuh -- decode path (M <= 32 tokens).
//
// Every warp is an independent streaming worker.  The work units are
// (16-row group, 128-channel stage) pairs, numbered row-group major; warp w
// owns the contiguous range of q + (w < r) units that starts at
// w q + min(w, r) (U = q W + r units, W warps).  A lane loads each unit's
// packed codes (two 16-byte vectors, 512 contiguous bytes per warp each) and
// its row pair's constants straight into registers two units ahead,
// dequantizes into the A fragments of warp-level m16n8k16 bf16 MMAs and
// accumulates in fp32 registers.  No shared memory ring, no producer, no
// barriers between warps: the only synchronisation is the deterministic
// reduction over the warps that share a row group (partials in a fixed slot
// per warp; the last one to arrive sums them in slot order).
//
// Why not tcgen05 here: a tcgen05.mma of kind::f16 occupies the SM's tensor
// core for ~200 cycles whatever its N (measured on B200 for N = 16..256), so a
// 16-token tile consumes only 128 x 16 weights per 200 cycles per SM (about
// 1.4 TB/s of 4-bit weights on 148 SMs).  Plain 16-byte loads from many
// independent warps reach the HBM rate without a copy pipeline.
//
// Instruction economy matters more than anything else here: the SM issues
// one warp instruction per cycle per sub-partition, and most of the integer
// and bf16x2 instructions this loop needs run at half rate on B200.  So all
// per-launch divisions are by multiplication with host-made constants, the
// loop counters are 32-bit, the register ring rotates without copies, and
// activations are loaded without predicates (rows past M are clamped to row
// M - 1; the MMA columns they feed are never stored).
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
  uint16_t* Y;              // bf16 [M, N]
  float* partial;           // [row group][slot][32 lanes][4 NB] fp32
  unsigned int* counter;    // [row group] arrivals
  int M, N, K;
  int KS;                   // stages (128 channels) per tile row
  int max_slots;            // partial slots per row group
  uint32_t q, r;            // units per warp: q + (w < r)
  FastDiv32 by_ks, by_q, by_q1;
  FastDiv64 by_dq;          // NF4: 64-block index -> s2 index
};

template <int NB_, int FMT_, int G_>
struct GemvCfg {
  static constexpr int NB = NB_;   // token blocks of 8
  static constexpr int MT = 8 * NB;
  static constexpr int FMT = FMT_;
  static constexpr int G = G_;
  static constexpr int kStageBytes = FMT == kFmtInt4 ? int4_stage_bytes(G) : nf4_stage_bytes();
  static constexpr int kWarps = 8;
  static constexpr int kThreads = 32 * kWarps;
  // resident CTAs per SM (80 or 128 registers a thread): 3 where the
  // register ring fits in 80 without spilling
  static constexpr int kMinBlocks = NB == 1 && FMT_ == kFmtInt4 && G_ >= 64 ? 3 : 2;
  // groups per 128-channel stage (INT4); NF4 keeps its absmax pairs in sp[0] / zp[0]
  static constexpr int kNq = FMT == kFmtInt4 ? 128 / G : 1;
};

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&d)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Streaming 16-byte load: read once, no L1 allocation.
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// One 128-channel stage of a lane's row group: 8 code words (two 16-byte
// loads, 512 contiguous bytes per warp each) and the constants of its two rows.
template <class C>
struct StageRegs {
  uint4 c0, c1;            // code words of channel blocks 0..3 and 4..7
  uint32_t sp[C::kNq];     // INT4: scale pairs, one per group in the stage; NF4: absmax pair, block 0
  uint32_t zp[C::kNq];     // INT4: zero pairs; NF4: absmax pair, block 1
};

template <class C>
__device__ __forceinline__ void load_stage(const uint8_t* __restrict__ blk, StageRegs<C>& r,
                                           int rgl, int lane) {
  const int g = lane >> 2;
  r.c0 = ldg_stream(blk + code_word_offset(rgl, 0, lane));
  r.c1 = ldg_stream(blk + code_word_offset(rgl, 4, lane));
  if constexpr (C::FMT == kFmtInt4) {
    constexpr int gps = kStageK / C::G;
#pragma unroll
    for (int q = 0; q < C::kNq; ++q) {
      r.sp[q] = __ldg(reinterpret_cast<const uint32_t*>(blk + scale_pair_offset(rgl, q, g, gps)));
      r.zp[q] = __ldg(blk + zero_pair_offset(rgl, q, g, gps));
    }
  } else {
    r.sp[0] = __ldg(reinterpret_cast<const uint16_t*>(blk + absmax_pair_offset(rgl, 0, g)));
    r.zp[0] = __ldg(reinterpret_cast<const uint16_t*>(blk + absmax_pair_offset(rgl, 1, g)));
  }
}

// Dequantize code words [W0, W0 + NW) of one 64-channel half and run their
// MMAs.  xs[nb] points at X[token row of block nb][first channel of the
// half + 4u]; p0 / p1 are the constants of rows r0 / r1 (INT4), a0 / a1 the
// reconstructed absmax (NF4).
template <class C, int W0, int NW>
__device__ __forceinline__ void mma_words(const uint32_t (&words)[4], const Int4Dq& p0,
                                          const Int4Dq& p1, float a0, float a1,
                                          const float* __restrict__ T,
                                          const uint16_t* const (&xs)[C::NB],
                                          float (&acc)[2][C::NB][4]) {
#pragma unroll
  for (int w = W0; w < W0 + NW; ++w) {
    uint32_t pr[4];
    if constexpr (C::FMT == kFmtInt4) {
      int4_dq_word(words[w], p0, p1, pr);
    } else {
      nf4_dq_word(words[w], a0, a1, T, pr);
    }
    const uint32_t afrag[4] = {pr[0], pr[2], pr[1], pr[3]};
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb) {
      const uint2 b = __ldg(reinterpret_cast<const uint2*>(xs[nb] + w * 16));
      mma_m16n8k16_bf16(acc[w & 1][nb], afrag, b.x, b.y);
    }
  }
}

// Warp owning unit u.
__device__ __forceinline__ uint32_t owner_of(uint32_t u, const GemvArgs& a) {
  const uint32_t big = a.r * (a.q + 1);  // units of the first r warps
  return u < big ? fast_div(u, a.by_q1) : a.r + fast_div(u - big, a.by_q);
}

// Hand a row group's accumulated sums on: write Y if this warp covered the
// whole channel range (units [seg0, seg1) == the row group's), else store
// them in the warp's slot; the last contributor of the row group sums the
// slots in order and writes Y.
template <class C>
__device__ __forceinline__ void flush_row_group(const GemvArgs& args, float (&acc)[2][C::NB][4],
                                                int rgg, uint32_t seg0, uint32_t seg1,
                                                uint32_t wid, int lane) {
  const int g = lane >> 2, u = lane & 3;
  const int r0 = rgg * 16 + g;
  float tot[C::NB][4];
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      tot[nb][j] = acc[0][nb][j] + acc[1][nb][j];
      acc[0][nb][j] = 0.0f;
      acc[1][nb][j] = 0.0f;
    }
  const uint32_t rs = static_cast<uint32_t>(rgg) * static_cast<uint32_t>(args.KS);
  const uint32_t re = rs + static_cast<uint32_t>(args.KS);
  bool write_y = true;
  if (seg0 != rs || seg1 != re) {
    const uint32_t first = owner_of(rs, args);
    const uint32_t contributors = owner_of(re - 1, args) - first + 1;
    float* slot = args.partial +
                  ((static_cast<size_t>(rgg) * args.max_slots + (wid - first)) * 32 + lane) * 4 * C::NB;
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
      *reinterpret_cast<float4*>(slot + nb * 4) =
          make_float4(tot[nb][0], tot[nb][1], tot[nb][2], tot[nb][3]);
    // publish the slot with an acquire-release counter update (no full fence,
    // which would also wait for this warp's prefetched loads)
    __syncwarp();
    unsigned prev = 0;
    if (lane == 0) prev = atom_add_acq_rel_gpu(args.counter + rgg, 1u);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    write_y = prev == contributors - 1;
    if (write_y) {
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) tot[nb][j] = 0.0f;
      const float* base =
          args.partial + (static_cast<size_t>(rgg) * args.max_slots * 32 + lane) * 4 * C::NB;
      for (uint32_t sp = 0; sp < contributors; ++sp) {
#pragma unroll
        for (int nb = 0; nb < C::NB; ++nb) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(
              base + static_cast<size_t>(sp) * 32 * 4 * C::NB + nb * 4));
          tot[nb][0] += v.x;
          tot[nb][1] += v.y;
          tot[nb][2] += v.z;
          tot[nb][3] += v.w;
        }
      }
      if (lane == 0) args.counter[rgg] = 0u;  // leave the workspace zeroed
    }
  }
  if (write_y) {
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int m = nb * 8 + 2 * u + (j & 1);
        const int nn = r0 + (j >> 1) * 8;
        if (m < args.M && nn < args.N)
          args.Y[static_cast<size_t>(m) * args.N + nn] =
              __bfloat16_as_ushort(__float2bfloat16_rn(tot[nb][j]));
      }
  }
}

// Dequantize and multiply one 128-channel stage of row group rgg.
template <class C>
__device__ __forceinline__ void stage_compute(const GemvArgs& args, const StageRegs<C>& cur,
                                              int rgg, int st, int g,
                                              const uint16_t* const (&xrow)[C::NB],
                                              const float* __restrict__ Ts,
                                              float (&acc)[2][C::NB][4]) {
  const int k0 = st * kStageK;
  const uint16_t* xa[C::NB];
  const uint16_t* xb[C::NB];
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb) {
    xa[nb] = xrow[nb] + k0;
    xb[nb] = xa[nb] + 64;
  }
  const uint32_t w0[4] = {cur.c0.x, cur.c0.y, cur.c0.z, cur.c0.w};
  const uint32_t w1[4] = {cur.c1.x, cur.c1.y, cur.c1.z, cur.c1.w};
  const bool second = k0 + 64 < args.K;  // K % 64 == 0: the second half exists or not
  if constexpr (C::FMT == kFmtInt4) {
    if constexpr (C::G == 128) {
      const Int4Dq e0 = int4_dq_params(cur.sp[0] & 0xFFFFu, cur.zp[0] & 0xFu);
      const Int4Dq e1 = int4_dq_params(cur.sp[0] >> 16, (cur.zp[0] >> 4) & 0xFu);
      mma_words<C, 0, 4>(w0, e0, e1, 0.f, 0.f, Ts, xa, acc);
      if (second) mma_words<C, 0, 4>(w1, e0, e1, 0.f, 0.f, Ts, xb, acc);
    } else if constexpr (C::G == 64) {
      {
        const Int4Dq e0 = int4_dq_params(cur.sp[0] & 0xFFFFu, cur.zp[0] & 0xFu);
        const Int4Dq e1 = int4_dq_params(cur.sp[0] >> 16, (cur.zp[0] >> 4) & 0xFu);
        mma_words<C, 0, 4>(w0, e0, e1, 0.f, 0.f, Ts, xa, acc);
      }
      if (second) {
        const Int4Dq e0 = int4_dq_params(cur.sp[1] & 0xFFFFu, cur.zp[1] & 0xFu);
        const Int4Dq e1 = int4_dq_params(cur.sp[1] >> 16, (cur.zp[1] >> 4) & 0xFu);
        mma_words<C, 0, 4>(w1, e0, e1, 0.f, 0.f, Ts, xb, acc);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q >= 2 && !second) break;
        const Int4Dq e0 = int4_dq_params(cur.sp[q] & 0xFFFFu, cur.zp[q] & 0xFu);
        const Int4Dq e1 = int4_dq_params(cur.sp[q] >> 16, (cur.zp[q] >> 4) & 0xFu);
        if (q == 0)
          mma_words<C, 0, 2>(w0, e0, e1, 0.f, 0.f, Ts, xa, acc);
        else if (q == 1)
          mma_words<C, 2, 2>(w0, e0, e1, 0.f, 0.f, Ts, xa, acc);
        else if (q == 2)
          mma_words<C, 0, 2>(w1, e0, e1, 0.f, 0.f, Ts, xb, acc);
        else
          mma_words<C, 2, 2>(w1, e0, e1, 0.f, 0.f, Ts, xb, acc);
      }
    }
  } else {
    // NF4: a' = code * s2[block index / dq_group] per (row, 64-block)
    const unsigned long long kb64 = static_cast<unsigned long long>(args.K / 64);
    const int r0 = rgg * 16 + g;
    float a0[2] = {0.0f, 0.0f}, a1[2] = {0.0f, 0.0f};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const unsigned long long blk = static_cast<unsigned long long>(st) * 2 + h;
      if (blk < kb64) {
        const uint32_t pair = h == 0 ? cur.sp[0] : cur.zp[0];
        if (r0 < args.N)
          a0[h] = __fmul_rn(static_cast<float>(pair & 0xFFu),
                            __ldg(args.s2 + fast_div(static_cast<unsigned long long>(r0) * kb64 + blk,
                                                     args.by_dq)));
        if (r0 + 8 < args.N)
          a1[h] = __fmul_rn(static_cast<float>(pair >> 8),
                            __ldg(args.s2 + fast_div(static_cast<unsigned long long>(r0 + 8) * kb64 + blk,
                                                     args.by_dq)));
      }
    }
    const Int4Dq none{};
    mma_words<C, 0, 4>(w0, none, none, a0[0], a1[0], Ts, xa, acc);
    if (second) mma_words<C, 0, 4>(w1, none, none, a0[1], a1[1], Ts, xb, acc);
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, C::kMinBlocks) w4_gemv_kernel(const GemvArgs args) {
  __shared__ float Ts[16];
  if (C::FMT == kFmtNf4) {
    if (threadIdx.x < 16) Ts[threadIdx.x] = __uint_as_float(kNf4LevelBits[threadIdx.x]);
    __syncthreads();
  }
  grid_dep_launch();
  grid_dep_wait();  // X, Y and the workspace may belong to the previous kernel

  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, u = lane & 3;
  const uint32_t wid = blockIdx.x * C::kWarps + (threadIdx.x >> 5);
  // this warp's contiguous range of (row group, stage) units, row-group major
  const uint32_t ua = wid * args.q + (wid < args.r ? wid : args.r);
  const int left = static_cast<int>(args.q) + (wid < args.r ? 1 : 0);
  if (left == 0) return;
  const int KS = args.KS;

  // activation rows of this lane's token columns; rows past M read row M - 1
  // (those accumulator columns are never stored)
  const uint16_t* xrow[C::NB];
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb) {
    const int row = min(nb * 8 + g, args.M - 1);
    xrow[nb] = args.X + static_cast<size_t>(row) * args.K + 4 * u;
  }

  // prefetch cursor: (row group, stage) of the next stage to load and the
  // address of its stage block
  const int rgg0 = static_cast<int>(fast_div(ua, args.by_ks));
  const int st0 = static_cast<int>(ua) - rgg0 * KS;
  int pf_rgg = rgg0, pf_st = st0;
  const uint8_t* pf_ptr =
      args.Wp + (static_cast<size_t>(pf_rgg >> 3) * KS + pf_st) * C::kStageBytes;
  auto advance = [&]() {
    if (++pf_st == KS) {
      pf_st = 0;
      ++pf_rgg;
      pf_ptr = args.Wp + static_cast<size_t>(pf_rgg >> 3) * KS * C::kStageBytes;
    } else {
      pf_ptr += C::kStageBytes;
    }
  };

  // three register sets, two stages in flight: set (i + 2) % 3 is refilled
  // while set i is consumed, so the ring rotates without copies
  StageRegs<C> ring[3];
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (i < left) {
      load_stage<C>(pf_ptr, ring[i], pf_rgg & 7, lane);
      advance();
    }

  float acc[2][C::NB][4];
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[e][nb][j] = 0.0f;

  int rgg = rgg0, st = st0;
  uint32_t seg0 = ua;  // first unit of this warp's part of row group rgg
  int n = 0;
  for (;;) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      if (n == left) return;
      if (n + 2 < left) {
        load_stage<C>(pf_ptr, ring[(i + 2) % 3], pf_rgg & 7, lane);
        advance();
      }
      stage_compute<C>(args, ring[i], rgg, st, g, xrow, Ts, acc);
      if (st == KS - 1 || n + 1 == left) {
        const uint32_t seg1 = ua + static_cast<uint32_t>(n) + 1;
        flush_row_group<C>(args, acc, rgg, seg0, seg1, wid, lane);
        ++rgg;
        st = 0;
        seg0 = seg1;
      } else {
        ++st;
      }
      ++n;
    }
  }
}

}  // namespace w4
