// w4_gemv_kernel.cuh -- decode path (M <= 32 tokens).
//
// Every warp is an independent streaming worker.  Work items are (16-row
// group, channel segment) pairs; a warp walks its items' 64-channel units,
// loading each unit's packed codes (16 bytes per lane, 512 contiguous bytes
// per warp), its per-group constants and the matching activations straight
// into registers several units ahead, dequantizes into the A fragments of
// warp-level m16n8k16 bf16 MMAs and accumulates in fp32 registers.  No shared
// memory ring, no producer, no barriers between warps: the only
// synchronisation is the deterministic reduction over a row group's segments
// (partials in a fixed slot per segment; the last segment to arrive sums them
// in segment order).
//
// Why not tcgen05 here: a tcgen05.mma of kind::f16 occupies the SM's tensor
// core for ~200 cycles whatever its N (measured on B200 for N = 16..256), so a
// 16-token tile consumes only 128 x 16 weights per 200 cycles per SM (about
// 1.4 TB/s of 4-bit weights on 148 SMs).  And a bulk-copy pipeline per CTA
// pays a prologue, queueing behind its own copies and a split epilogue on
// every call; plain 16-byte loads from many independent warps reach the full
// HBM rate on B200 without them.
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
  int row_groups;           // ceil(N / 16)
  int max_slots;            // partial slots per row group
  long long total;          // (row group, stage) work units = row_groups * KS
  int dq_group;             // NF4 double-quant run length
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
  static constexpr int kMinBlocks = NB == 1 ? 3 : 2;  // 85 / 128 registers
  static constexpr int kDepth = 2;  // stages of codes in flight per lane (per-warp: 2 KB)
  // groups per 128-channel stage (INT4); NF4 keeps its absmax pairs in sp[0]
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

// Dequantize code words [w0, w0 + nw) of one 64-channel half and run their
// MMAs.  `xrow` points at X[token g][first channel of the half + 4u] (token
// block 0); tokens_left = M - g; p0 / p1 are the constants of rows r0 / r1 (INT4),
// a0 / a1 the reconstructed absmax (NF4).
template <class C, int W0, int NW>
__device__ __forceinline__ void mma_words(const uint32_t (&words)[4], const Int4Dq& p0,
                                          const Int4Dq& p1, float a0, float a1,
                                          const float* __restrict__ T,
                                          const uint16_t* __restrict__ xrow, size_t xnb_stride,
                                          int tokens_left, float (&acc)[2][C::NB][4]) {
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
      uint2 b = make_uint2(0u, 0u);
      if (nb * 8 < tokens_left)  // token 8 nb + g exists
        b = __ldg(reinterpret_cast<const uint2*>(xrow + nb * xnb_stride + w * 16));
      mma_m16n8k16_bf16(acc[w & 1][nb], afrag, b.x, b.y);
    }
  }
}

// Warp index owning work unit u when warp w owns [floor(w U / W), floor((w+1) U / W)).
__device__ __forceinline__ int owner_of(long long u, long long U, long long W) {
  return static_cast<int>(((u + 1) * W + U - 1) / U) - 1;
}

// Hand a row group's accumulated sums on: write Y if this warp covered the
// whole channel range, else store them in the warp's slot; the last
// contributor of the row group sums the slots in order and writes Y.
template <class C>
__device__ __forceinline__ void flush_row_group(const GemvArgs& args, float (&acc)[2][C::NB][4],
                                                int rgg, long long seg_start, long long seg_end,
                                                long long U, long long W, int lane) {
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
  const long long rs = static_cast<long long>(rgg) * args.KS, re = rs + args.KS;
  bool write_y = true;
  if (seg_start != rs || seg_end != re) {
    const int first = owner_of(rs, U, W);
    const int last = owner_of(re - 1, U, W);
    const int mine = owner_of(seg_start, U, W);
    const int contributors = last - first + 1;
    float* slot = args.partial +
                  ((static_cast<size_t>(rgg) * args.max_slots + (mine - first)) * 32 + lane) * 4 * C::NB;
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
    write_y = prev == static_cast<unsigned>(contributors - 1);
    if (write_y) {
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) tot[nb][j] = 0.0f;
      const float* base =
          args.partial + (static_cast<size_t>(rgg) * args.max_slots * 32 + lane) * 4 * C::NB;
      for (int sp = 0; sp < contributors; ++sp) {
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
  const long long W = static_cast<long long>(gridDim.x) * C::kWarps;
  const long long wid = static_cast<long long>(blockIdx.x) * C::kWarps + (threadIdx.x >> 5);
  const long long U = args.total;
  // this warp's contiguous range of (row group, stage) units, row-group major
  const long long ua = wid * U / W, ub = (wid + 1) * U / W;
  if (ua >= ub) return;
  const int KS = args.KS;
  const size_t xnb_stride = static_cast<size_t>(8) * args.K;
  const int tokens_left = args.M - g;
  const uint16_t* xbase = args.X + static_cast<size_t>(g) * args.K + 4 * u;

  // prefetch cursor: (row group, stage) of the next stage to load and the
  // address of its stage block, advanced without divisions
  int pf_rgg = static_cast<int>(ua / KS);
  int pf_st = static_cast<int>(ua - static_cast<long long>(pf_rgg) * KS);
  const uint8_t* pf_ptr = args.Wp + (static_cast<size_t>(pf_rgg >> 3) * KS + pf_st) * C::kStageBytes;
  auto advance = [&]() {
    if (++pf_st == KS) {
      pf_st = 0;
      ++pf_rgg;
      pf_ptr = args.Wp + static_cast<size_t>(pf_rgg >> 3) * KS * C::kStageBytes;
    } else {
      pf_ptr += C::kStageBytes;
    }
  };

  StageRegs<C> ring[C::kDepth];
#pragma unroll
  for (int i = 0; i < C::kDepth; ++i)
    if (ua + i < ub) {
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

  int rgg = static_cast<int>(ua / KS);
  int st = static_cast<int>(ua - static_cast<long long>(rgg) * KS);
  long long seg_start = ua;
  for (long long base = ua; base < ub; base += C::kDepth) {
#pragma unroll
    for (int i = 0; i < C::kDepth; ++i) {
      const long long un = base + i;
      if (un < ub) {
        const StageRegs<C> cur = ring[i];
        if (un + C::kDepth < ub) {
          load_stage<C>(pf_ptr, ring[i], pf_rgg & 7, lane);
          advance();
        }
        const int r0 = rgg * 16 + g;
        const int k0 = st * kStageK;
        const uint32_t w0[4] = {cur.c0.x, cur.c0.y, cur.c0.z, cur.c0.w};
        const uint32_t w1[4] = {cur.c1.x, cur.c1.y, cur.c1.z, cur.c1.w};
        const bool second = k0 + 64 < args.K;
        if constexpr (C::FMT == kFmtInt4) {
          if constexpr (C::G == 128) {
            const Int4Dq e0 = int4_dq_params(cur.sp[0] & 0xFFFFu, cur.zp[0] & 0xFu);
            const Int4Dq e1 = int4_dq_params(cur.sp[0] >> 16, (cur.zp[0] >> 4) & 0xFu);
            mma_words<C, 0, 4>(w0, e0, e1, 0.f, 0.f, Ts, xbase + k0, xnb_stride, tokens_left, acc);
            if (second)
              mma_words<C, 0, 4>(w1, e0, e1, 0.f, 0.f, Ts, xbase + k0 + 64, xnb_stride,
                                 tokens_left, acc);
          } else if constexpr (C::G == 64) {
            {
              const Int4Dq e0 = int4_dq_params(cur.sp[0] & 0xFFFFu, cur.zp[0] & 0xFu);
              const Int4Dq e1 = int4_dq_params(cur.sp[0] >> 16, (cur.zp[0] >> 4) & 0xFu);
              mma_words<C, 0, 4>(w0, e0, e1, 0.f, 0.f, Ts, xbase + k0, xnb_stride, tokens_left, acc);
            }
            if (second) {
              const Int4Dq e0 = int4_dq_params(cur.sp[1] & 0xFFFFu, cur.zp[1] & 0xFu);
              const Int4Dq e1 = int4_dq_params(cur.sp[1] >> 16, (cur.zp[1] >> 4) & 0xFu);
              mma_words<C, 0, 4>(w1, e0, e1, 0.f, 0.f, Ts, xbase + k0 + 64, xnb_stride,
                                 tokens_left, acc);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (q >= 2 && !second) break;
              const Int4Dq e0 = int4_dq_params(cur.sp[q] & 0xFFFFu, cur.zp[q] & 0xFu);
              const Int4Dq e1 = int4_dq_params(cur.sp[q] >> 16, (cur.zp[q] >> 4) & 0xFu);
              if (q == 0)
                mma_words<C, 0, 2>(w0, e0, e1, 0.f, 0.f, Ts, xbase + k0, xnb_stride, tokens_left, acc);
              else if (q == 1)
                mma_words<C, 2, 2>(w0, e0, e1, 0.f, 0.f, Ts, xbase + k0, xnb_stride, tokens_left, acc);
              else if (q == 2)
                mma_words<C, 0, 2>(w1, e0, e1, 0.f, 0.f, Ts, xbase + k0 + 64, xnb_stride,
                                   tokens_left, acc);
              else
                mma_words<C, 2, 2>(w1, e0, e1, 0.f, 0.f, Ts, xbase + k0 + 64, xnb_stride,
                                   tokens_left, acc);
            }
          }
        } else {
          const long long kb64 = args.K / 64;
          float a0[2] = {0.0f, 0.0f}, a1[2] = {0.0f, 0.0f};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int blk = st * 2 + h;
            if (blk < kb64) {
              const uint32_t pair = h == 0 ? cur.sp[0] : cur.zp[0];
              if (r0 < args.N)
                a0[h] = __fmul_rn(static_cast<float>(pair & 0xFFu),
                                  __ldg(args.s2 + (static_cast<long long>(r0) * kb64 + blk) / args.dq_group));
              if (r0 + 8 < args.N)
                a1[h] = __fmul_rn(static_cast<float>(pair >> 8),
                                  __ldg(args.s2 + (static_cast<long long>(r0 + 8) * kb64 + blk) / args.dq_group));
            }
          }
          const Int4Dq none{};
          mma_words<C, 0, 4>(w0, none, none, a0[0], a1[0], Ts, xbase + k0, xnb_stride,
                             tokens_left, acc);
          if (second)
            mma_words<C, 0, 4>(w1, none, none, a0[1], a1[1], Ts, xbase + k0 + 64, xnb_stride,
                               tokens_left, acc);
        }
        // end of this row group's part of the range: flush
        if (st == KS - 1 || un + 1 == ub) {
          flush_row_group<C>(args, acc, rgg, seg_start, un + 1, U, W, lane);
          ++rgg;
          st = 0;
          seg_start = un + 1;
        } else {
          ++st;
        }
      }
    }
  }
}

}  // namespace w4
