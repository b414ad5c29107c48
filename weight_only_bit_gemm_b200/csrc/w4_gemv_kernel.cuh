// w4_gemv_kernel.cuh -- decode path (M <= 32 tokens): weights stream from HBM
// through a shared-memory ring (one bulk copy per 128x128 stage), each warp
// dequantizes its 16-row group straight into the A fragments of warp-level
// m16n8k16 bf16 MMAs (fp32 accumulate in registers), with X read as B
// fragments from a TMA tile.
//
// Why not tcgen05 here: a tcgen05.mma of kind::f16 occupies the SM's tensor
// core for ~200 cycles whatever its N (measured on B200 for N = 16..256), so a
// 16-token tile consumes only 128 x 16 weights per 200 cycles per SM (about
// 1.4 TB/s of 4-bit weights on 148 SMs).  The warp-level MMA has no such
// floor, and the dequantized weights never leave registers.
//
// Channel order: inside each 16-channel block, lane (g, u) holds channels
// 4u..4u+3 (see w4_prepack.cuh) in the MMA's k slots {2u, 2u+1, 2u+8, 2u+9};
// the B fragment is read with the same permutation (X[token][4u..4u+3] as one
// 64-bit load), so the product over the block is unchanged.
#pragma once

#include "w4_gemm.cuh"

namespace w4 {

template <int NB_, int STAGES_, int FMT_, int G_>
struct GemvCfg {
  static constexpr int NB = NB_;          // token blocks of 8 (tokens per tile = 8 NB)
  static constexpr int MT = 8 * NB;
  static constexpr int STAGES = STAGES_;
  static constexpr int FMT = FMT_;
  static constexpr int G = G_;
  static constexpr int kXBoxBytes = MT * 128;          // [MT][64] bf16, 128-byte rows
  static constexpr int kXStageBytes = 2 * kXBoxBytes;  // 128 channels
  static constexpr int kWStageBytes = FMT == kFmtInt4 ? int4_stage_bytes(G) : nf4_stage_bytes();
  static constexpr int kWSlot = (kWStageBytes + 127) / 128 * 128;
  // two warps per 16-row group, one per 64-channel half of each stage
  static constexpr int kConsumers = 16;
  static constexpr int kThreads = 32 * (1 + kConsumers);
  static constexpr int kNumBars = 2 * STAGES + 3;
  static constexpr int kXRegion = (STAGES * kXStageBytes + 1023) / 1024 * 1024;
  static constexpr int kRedBytes = 8 * 32 * 4 * NB * 4;  // half-sum exchange
  static constexpr int kSmemBytes =
      1024 + kXRegion + STAGES * kWSlot + kRedBytes + kNumBars * 8 + 16 + 64;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&d)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <class C>
__global__ void __launch_bounds__(C::kThreads)
    w4_gemv_kernel(const __grid_constant__ CUtensorMap xmap, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* xs = smem;                                 // STAGES x kXStageBytes (1024-aligned)
  uint8_t* wsl = xs + C::kXRegion;                    // STAGES x kWSlot
  float* red = reinterpret_cast<float*>(wsl + C::STAGES * C::kWSlot);  // [8][32][4 NB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + C::kRedBytes);
  uint64_t* full = bars;                              // X + W landed     (tx)
  uint64_t* empty = full + C::STAGES;                 // 16 warps consumed
  uint64_t* redb = empty + C::STAGES;                 // upper halves stored (8 warps)
  uint64_t* epi1 = redb + 1;                          // partials stored  (8 warps)
  uint64_t* epi2 = epi1 + 1;                          // last-arrival known
  int* last_flag = reinterpret_cast<int*>(epi2 + 1);
  float* Ts = reinterpret_cast<float*>(epi2 + 1) + 4;  // NF4 levels [16]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nt = blockIdx.x / args.splits;
  const int split = blockIdx.x % args.splits;
  const int mtile = blockIdx.y;
  const int s0 = static_cast<int>(static_cast<long long>(split) * args.KS / args.splits);
  const int s1 = static_cast<int>(static_cast<long long>(split + 1) * args.KS / args.splits);
  const int nst = s1 - s0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::kConsumers);
    }
    mbar_init(redb, C::kConsumers / 2);
    mbar_init(epi1, C::kConsumers / 2);
    mbar_init(epi2, 1);
    fence_barrier_init();
    grid_dep_launch();
  }
  if (C::FMT == kFmtNf4 && threadIdx.x < 16)
    Ts[threadIdx.x] = __uint_as_float(kNf4LevelBits[threadIdx.x]);
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&xmap);
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const uint8_t* wsrc =
          args.Wp + (static_cast<size_t>(nt) * args.KS + s0) * C::kWStageBytes;
      const int first = nst < C::STAGES ? nst : C::STAGES;
      for (int it = 0; it < first; ++it) {
        mbar_arrive_expect_tx(&full[it], C::kXStageBytes + C::kWStageBytes);
        bulk_g2s(wsl + it * C::kWSlot, wsrc + static_cast<size_t>(it) * C::kWStageBytes,
                 C::kWStageBytes, &full[it], pol_w);
      }
      grid_dep_wait();
      int issued = 0;
      for (int it = 0; it < nst; ++it) {
        const int s = it % C::STAGES;
        if (it >= C::STAGES) {
          if (!mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1)) break;
          mbar_arrive_expect_tx(&full[s], C::kXStageBytes + C::kWStageBytes);
          bulk_g2s(wsl + s * C::kWSlot, wsrc + static_cast<size_t>(it) * C::kWStageBytes,
                   C::kWStageBytes, &full[s], pol_w);
        }
        // both 64-channel boxes of the stage in one copy (X viewed as
        // [K/64][M][64])
        tma_load_3d(xs + s * C::kXStageBytes, &xmap, 0, mtile * C::MT, (s0 + it) * 2, &full[s],
                    pol_x);
        ++issued;
      }
      for (int it = issued - 1; it >= 0 && it >= issued - C::STAGES; --it)
        mbar_wait(&full[it % C::STAGES], (it / C::STAGES) & 1);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int cw = warp - 1;            // 0..15
    const int rg = cw & 7;              // 16-row group of the tile
    const int kq = cw >> 3;             // channel half of every stage
    const int g = lane >> 2, u = lane & 3;
    const int r0 = nt * kTileRows + rg * 16 + g;
    // two accumulator sets (even / odd channel blocks) to shorten the MMA
    // dependency chain
    float acc[2][C::NB][4];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[e][nb][j] = 0.0f;
    bool ok = true;
    for (int it = 0; it < nst; ++it) {
      const int s = it % C::STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (it / C::STAGES) & 1))) {
        ok = false;
        break;
      }
      const uint8_t* wb = wsl + s * C::kWSlot;
      // X box of this half: token n = 8 nb + g, channels 16 w + 4u .. +3; with
      // the 128-byte swizzle the 16-byte chunk c of row n sits at c ^ (n % 8)
      const uint8_t* xbox = xs + s * C::kXStageBytes + kq * C::kXBoxBytes;
      const uint4 cwd = *reinterpret_cast<const uint4*>(wb + code_word_offset(rg, 4 * kq, lane));
      const uint32_t words[4] = {cwd.x, cwd.y, cwd.z, cwd.w};
      Int4Dq p0[2], p1[2];
      float a0 = 0.0f, a1 = 0.0f;
      if constexpr (C::FMT == kFmtInt4) {
        constexpr int gps = kStageK / C::G;
#pragma unroll
        for (int q = 0; q < (C::G == 32 ? 2 : 1); ++q) {
          const int gl = (kq * 64 + q * 32) / C::G;
          const uint32_t sp = *reinterpret_cast<const uint32_t*>(wb + scale_pair_offset(rg, gl, g, gps));
          const uint32_t zp = wb[zero_pair_offset(rg, gl, g, gps)];
          p0[q] = int4_dq_params(sp & 0xFFFFu, zp & 0xFu);
          p1[q] = int4_dq_params(sp >> 16, zp >> 4);
        }
      } else {
        const int blk_in_row = (s0 + it) * 2 + kq;
        const uint32_t cp = *reinterpret_cast<const uint16_t*>(wb + absmax_pair_offset(rg, kq, g));
        if (blk_in_row * 64 < args.K) {
          const long long kb64 = args.K / 64;
          if (r0 < args.N)
            a0 = __fmul_rn(static_cast<float>(cp & 0xFFu),
                           __ldg(args.s2 + (static_cast<long long>(r0) * kb64 + blk_in_row) / args.dq_group));
          if (r0 + 8 < args.N)
            a1 = __fmul_rn(static_cast<float>(cp >> 8),
                           __ldg(args.s2 + (static_cast<long long>(r0 + 8) * kb64 + blk_in_row) / args.dq_group));
        }
      }
      uint2 bfr[4][C::NB];
#pragma unroll
      for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int nb = 0; nb < C::NB; ++nb) {
          const int n = nb * 8 + g;
          const int chunk = w * 2 + (u >> 1);
          bfr[w][nb] = *reinterpret_cast<const uint2*>(xbox + n * 128 + ((chunk ^ (n & 7)) << 4) +
                                                       (u & 1) * 8);
        }
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t pr[4];
        if constexpr (C::FMT == kFmtInt4) {
          const int q = (C::G == 32) ? (w >> 1) : 0;
          int4_dq_word(words[w], p0[q], p1[q], pr);
        } else {
          nf4_dq_word(words[w], a0, a1, Ts, pr);
        }
        const uint32_t afrag[4] = {pr[0], pr[2], pr[1], pr[3]};
#pragma unroll
        for (int nb = 0; nb < C::NB; ++nb)
          mma_m16n8k16_bf16(acc[w & 1][nb], afrag, bfr[w][nb].x, bfr[w][nb].y);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ------------------------------------------------------------ epilogue
    // the upper-half warp hands its sums to the lower-half warp of the same
    // row group through shared memory
    float tot[C::NB][4];
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
      for (int j = 0; j < 4; ++j) tot[nb][j] = acc[0][nb][j] + acc[1][nb][j];
    float* rslot = red + (rg * 32 + lane) * 4 * C::NB;
    if (kq == 1) {
      if (ok) {
#pragma unroll
        for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
          for (int j = 0; j < 4; ++j) rslot[nb * 4 + j] = tot[nb][j];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(redb);
    } else if (ok && __all_sync(0xffffffffu, mbar_wait(redb, 0))) {
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) tot[nb][j] += rslot[nb * 4 + j];
      // tot[nb] = D[rows r0, r0+8][tokens 8nb + 2u, 8nb + 2u + 1]
      grid_dep_wait();
      const int tile_id = mtile * args.tiles_n + nt;
      const int row_l = rg * 16 + g;  // tile row of tot[.][0..1]; +8 for [2..3]
      if (args.splits == 1) {
#pragma unroll
        for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int m = mtile * C::MT + nb * 8 + 2 * u + (j & 1);
            const int nn = r0 + (j >> 1) * 8;
            if (m < args.M && nn < args.N)
              args.Y[static_cast<size_t>(m) * args.N + nn] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(tot[nb][j]));
          }
      } else {
        float* part = args.partial +
                      (static_cast<size_t>(tile_id) * args.splits + split) * C::MT * kTileRows;
#pragma unroll
        for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            part[(nb * 8 + 2 * u + (j & 1)) * kTileRows + row_l + (j >> 1) * 8] = tot[nb][j];
        // the last CTA of this tile to arrive sums the partials in split order
        // (mbarriers with bounded waits, not bar.sync, so that a warp that gave
        // up earlier cannot leave the others blocked)
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(epi1);
        if (cw == 0 && lane == 0) {
          if (mbar_wait(epi1, 0)) {
            const unsigned prev = atomicAdd(args.counter + tile_id, 1u);
            *last_flag = (prev == static_cast<unsigned>(args.splits - 1)) ? 1 : 0;
          } else {
            *last_flag = 0;
          }
          mbar_arrive(epi2);
        }
        const bool have = __all_sync(0xffffffffu, mbar_wait(epi2, 0));
        if (have && *last_flag) {
          __threadfence();
          const float* base =
              args.partial + static_cast<size_t>(tile_id) * args.splits * C::MT * kTileRows;
          float sum[C::NB][4];
#pragma unroll
          for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
            for (int j = 0; j < 4; ++j) sum[nb][j] = 0.0f;
          // fixed split order, loads of four splits in flight at a time
          for (int sp0 = 0; sp0 < args.splits; sp0 += 4) {
            float v[4][C::NB][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int sp = sp0 + q;
#pragma unroll
              for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  v[q][nb][j] = sp < args.splits
                                    ? __ldcg(base + (static_cast<size_t>(sp) * C::MT + nb * 8 +
                                                     2 * u + (j & 1)) * kTileRows +
                                             row_l + (j >> 1) * 8)
                                    : 0.0f;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  if (sp0 + q < args.splits) sum[nb][j] += v[q][nb][j];
          }
#pragma unroll
          for (int nb = 0; nb < C::NB; ++nb)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int m = mtile * C::MT + nb * 8 + 2 * u + (j & 1);
              const int nn = r0 + (j >> 1) * 8;
              if (m < args.M && nn < args.N)
                args.Y[static_cast<size_t>(m) * args.N + nn] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(sum[nb][j]));
            }
          if (cw == 0 && lane == 0) args.counter[tile_id] = 0u;
        }
      }
    }
  }
  __syncthreads();
}

}  // namespace w4
