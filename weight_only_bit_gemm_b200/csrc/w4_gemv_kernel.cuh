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
  float* partial;           // [row group][segment][32 lanes][4 NB] fp32
  unsigned int* counter;    // [row group] arrivals
  int M, N, K;
  int KS;                   // stages (128 channels) per tile row
  int units;                // 64-channel units per row = ceil(K / 64)
  int row_groups;           // ceil(N / 16)
  int segs;                 // segments per row group
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
  static constexpr int kDepth = NB <= 2 ? 8 : 4;  // units of codes in flight per lane
  static constexpr int kNq = (FMT == kFmtInt4 && G == 32) ? 2 : 1;  // groups per unit
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

// Per-unit weight data of a lane: 4 code words and the constants of its two
// rows (prefetched kDepth units ahead).
template <class C>
struct CodeRegs {
  uint4 codes;
  uint32_t sp[C::kNq];     // INT4: scale pairs (per group in the unit); NF4: absmax pair
  uint32_t zp[C::kNq];     // INT4: zero pairs
};

// Activation fragments of one unit (fetched one unit ahead).
template <class C>
struct XRegs {
  uint2 b[4][C::NB];
};

template <class C>
__device__ __forceinline__ void load_codes(const GemvArgs& a, CodeRegs<C>& r, int rgg, int unit,
                                           int lane) {
  const int g = lane >> 2;
  const int tile = rgg >> 3, rgl = rgg & 7;
  const int stage = unit >> 1, half = unit & 1;
  const uint8_t* blk = a.Wp + (static_cast<size_t>(tile) * a.KS + stage) * C::kStageBytes;
  r.codes = ldg_stream(blk + code_word_offset(rgl, 4 * half, lane));
  if constexpr (C::FMT == kFmtInt4) {
    constexpr int gps = kStageK / C::G;
#pragma unroll
    for (int q = 0; q < C::kNq; ++q) {
      const int gl = (half * 64 + q * 32) / C::G;
      r.sp[q] = __ldg(reinterpret_cast<const uint32_t*>(blk + scale_pair_offset(rgl, gl, g, gps)));
      r.zp[q] = __ldg(blk + zero_pair_offset(rgl, gl, g, gps));
    }
  } else {
    r.sp[0] = __ldg(reinterpret_cast<const uint16_t*>(blk + absmax_pair_offset(rgl, half, g)));
  }
}

template <class C>
__device__ __forceinline__ void load_x(const GemvArgs& a, XRegs<C>& r, int unit, int lane) {
  const int g = lane >> 2, u = lane & 3;
  const int k0 = unit * 64;
#pragma unroll
  for (int w = 0; w < 4; ++w)
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb) {
      const int n = nb * 8 + g;
      const int k = k0 + w * 16 + 4 * u;
      r.b[w][nb] = (n < a.M && k < a.K)
                       ? __ldg(reinterpret_cast<const uint2*>(a.X + static_cast<size_t>(n) * a.K + k))
                       : make_uint2(0u, 0u);
    }
}

template <class C>
__device__ __forceinline__ void compute_unit(const GemvArgs& a, const CodeRegs<C>& r,
                                             const XRegs<C>& x, int rgg, int unit, int lane,
                                             const float* __restrict__ T,
                                             float (&acc)[2][C::NB][4]) {
  const int g = lane >> 2;
  const uint32_t words[4] = {r.codes.x, r.codes.y, r.codes.z, r.codes.w};
  Int4Dq p0[C::kNq], p1[C::kNq];
  float a0 = 0.0f, a1 = 0.0f;
  if constexpr (C::FMT == kFmtInt4) {
#pragma unroll
    for (int q = 0; q < C::kNq; ++q) {
      p0[q] = int4_dq_params(r.sp[q] & 0xFFFFu, r.zp[q] & 0xFu);
      p1[q] = int4_dq_params(r.sp[q] >> 16, (r.zp[q] >> 4) & 0xFu);
    }
  } else {
    const int r0 = rgg * 16 + g;
    if (unit * 64 < a.K) {
      const long long kb64 = a.K / 64;
      if (r0 < a.N)
        a0 = __fmul_rn(static_cast<float>(r.sp[0] & 0xFFu),
                       __ldg(a.s2 + (static_cast<long long>(r0) * kb64 + unit) / a.dq_group));
      if (r0 + 8 < a.N)
        a1 = __fmul_rn(static_cast<float>((r.sp[0] >> 8) & 0xFFu),
                       __ldg(a.s2 + (static_cast<long long>(r0 + 8) * kb64 + unit) / a.dq_group));
    }
  }
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t pr[4];
    if constexpr (C::FMT == kFmtInt4) {
      const int q = (C::kNq == 2) ? (w >> 1) : 0;
      int4_dq_word(words[w], p0[q], p1[q], pr);
    } else {
      nf4_dq_word(words[w], a0, a1, T, pr);
    }
    const uint32_t afrag[4] = {pr[0], pr[2], pr[1], pr[3]};
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
      mma_m16n8k16_bf16(acc[w & 1][nb], afrag, x.b[w][nb].x, x.b[w][nb].y);
  }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads) w4_gemv_kernel(const GemvArgs args) {
  __shared__ float Ts[16];
  if (C::FMT == kFmtNf4) {
    if (threadIdx.x < 16) Ts[threadIdx.x] = __uint_as_float(kNf4LevelBits[threadIdx.x]);
    __syncthreads();
  }
  grid_dep_launch();
  grid_dep_wait();  // X, Y and the workspace may belong to the previous kernel

  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, u = lane & 3;
  const int warp_global = blockIdx.x * C::kWarps + (threadIdx.x >> 5);
  const int warps_total = gridDim.x * C::kWarps;
  const int items = args.row_groups * args.segs;

  for (int item = warp_global; item < items; item += warps_total) {
    const int rgg = item / args.segs;
    const int seg = item - rgg * args.segs;
    const int u0 = static_cast<int>(static_cast<long long>(seg) * args.units / args.segs);
    const int u1 = static_cast<int>(static_cast<long long>(seg + 1) * args.units / args.segs);
    float acc[2][C::NB][4];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[e][nb][j] = 0.0f;

    // ring of kDepth units of codes in flight; activations one unit ahead
    CodeRegs<C> cr[C::kDepth];
#pragma unroll
    for (int i = 0; i < C::kDepth; ++i)
      if (u0 + i < u1) load_codes<C>(args, cr[i], rgg, u0 + i, lane);
    XRegs<C> xa;
    load_x<C>(args, xa, u0, lane);
    for (int ub = u0; ub < u1; ub += C::kDepth) {
#pragma unroll
      for (int i = 0; i < C::kDepth; ++i) {
        const int un = ub + i;
        if (un < u1) {
          XRegs<C> xn;
          if (un + 1 < u1) load_x<C>(args, xn, un + 1, lane);
          compute_unit<C>(args, cr[i], xa, rgg, un, lane, Ts, acc);
          if (un + C::kDepth < u1) load_codes<C>(args, cr[i], rgg, un + C::kDepth, lane);
          xa = xn;
        }
      }
    }

    // tot[nb] = D[rows r0, r0 + 8][tokens 8 nb + 2u, 8 nb + 2u + 1]
    float tot[C::NB][4];
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
      for (int j = 0; j < 4; ++j) tot[nb][j] = acc[0][nb][j] + acc[1][nb][j];
    const int r0 = rgg * 16 + g;
    bool write_y = true;
    if (args.segs > 1) {
      float* slot = args.partial +
                    ((static_cast<size_t>(rgg) * args.segs + seg) * 32 + lane) * 4 * C::NB;
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb)
        *reinterpret_cast<float4*>(slot + nb * 4) =
            make_float4(tot[nb][0], tot[nb][1], tot[nb][2], tot[nb][3]);
      __threadfence();
      __syncwarp();
      unsigned prev = 0;
      if (lane == 0) prev = atomicAdd(args.counter + rgg, 1u);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      write_y = prev == static_cast<unsigned>(args.segs - 1);
      if (write_y) {
        // last segment of this row group: sum all slots in segment order
        __threadfence();
#pragma unroll
        for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
          for (int j = 0; j < 4; ++j) tot[nb][j] = 0.0f;
        const float* base =
            args.partial + (static_cast<size_t>(rgg) * args.segs * 32 + lane) * 4 * C::NB;
        for (int sp = 0; sp < args.segs; ++sp) {
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
}

}  // namespace w4
