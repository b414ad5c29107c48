// w4_int8_tc.cuh -- the LLM.int8 product for more than 32 tokens on the
// tensor cores: tcgen05.mma of kind::i8 (s8 x s8, s32 accumulate in tensor
// memory).  The INT8 part of the mixed decomposition is an exact integer sum
// ("大模型量化选型：五种主流方案对比与实战" §2.1), so the accumulator is exact
// whatever the order of the K steps and of the split-K partial sums.
//
// Tile: 128 weight rows (the MMA's M) x MT tokens (its N), K in stages of
// 128 channels (four MMAs of K = 32).  Both operands arrive by TMA into
// shared memory in the 128-byte swizzled layout (128 int8 channels = one
// 128-byte row), so the same K-major descriptors as for bf16 apply, K = 32
// bytes per instruction.  Warp roles: warp 0 the producer (the weight tiles
// of the first ring are requested before the launch dependency resolves),
// warp 1 tensor-memory allocation and the single MMA thread, warps 2..5 the
// epilogue (one weight row per thread: y = acc s_x s_w + d, bf16 out; with
// split K the int32 partials go to the workspace and the last CTA of the
// tile sums them).  d, the 16-bit product of the outlier channels
// (§2.2's second matrix multiplication), is itself a small GEMM,
// D2 = W_o X_o^T over the outlier channels: once the INT8 accumulator is
// complete the operand ring is idle, the epilogue warps write
// W_o[row][i] = bf16(q_w s_w) and X_o[token][i] = x into it (128-byte swizzled,
// K-major, 64 channels per chunk, zero beyond the last outlier) and one of
// them issues kind::f16 MMAs into a second accumulator in tensor memory.
// Operands that do not fit the ring (more than about 256 outlier channels)
// are read from global memory by each output instead, one fma per channel.
#pragma once

#include <cuda_bf16.h>

#include "w4_int8.cuh"
#include "w4_ptx.cuh"

namespace w4 {

constexpr int kI8Rows = 128;  // weight rows per tile (the MMA's M)

template <int MT_, int STAGES_>
struct I8Cfg {
  static constexpr int MT = MT_;
  static constexpr int STAGES = STAGES_;
  static constexpr int kWStage = 128 * 128;  // weight tile bytes per stage
  static constexpr int kXStage = MT * 128;   // activation tile bytes per stage
  static constexpr int kThreads = 64 + 4 * 32;
  // the s32 accumulator in columns [0, MT), the outlier product's fp32 one in [MT, 2 MT)
  static constexpr int kTmemCols = MT <= 16 ? 32 : MT <= 32 ? 64 : MT <= 64 ? 128 : MT <= 128 ? 256 : 512;
  static constexpr int kRingBytes = STAGES * (kWStage + kXStage);
  // one 64-channel chunk of the outlier operands: 128 weight rows and MT
  // token rows of 128 bytes (a multiple of 1024: swizzle atoms stay aligned)
  static constexpr int kOChunkBytes = (128 + MT) * 128;
  // + per epilogue warp, its copy of the tile's token scales s_x
  static constexpr int kSmemBytes = 1024 + kRingBytes + (2 * STAGES + 6) * 8 + 16 + 4 * MT * 4;
  static_assert(MT % 16 == 0 && MT >= 16 && MT <= 256, "MMA N for M = 128");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// Instruction descriptor, kind::i8: s32 accumulator (bits 4-5 = 2), A and B
// signed 8-bit (bits 7-9 = 1, bits 10-12 = 1), both K-major, N >> 3 at bits
// 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int m, int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::i8.
__device__ __forceinline__ void mma_s8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// bf16_rne of two floats, packed with the first in the low half.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
}

struct I8TcArgs {
  const float* sx;        // [M]
  const float* sw;        // [N]
  const uint16_t* X;      // bf16 [M, K] (outlier channels)
  const int8_t* qw;       // [N, K] (outlier channels' weights)
  const int32_t* olist;   // ascending outlier channels
  const int32_t* ocount;
  uint16_t* Y;            // bf16 [M, N]
  int* partial;           // split-K int32 partials [tile][split][MT][128]
  unsigned int* counter;  // [tile], cleared by the call's scan kernel
  int M, N, K, KS, tiles_n, tiles_m, splits;
  unsigned long long partial_count;  // extent, for the bounds-checked build
};

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    int8_tc_kernel(const __grid_constant__ CUtensorMap wmap,
                   const __grid_constant__ CUtensorMap xmap, const I8TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ws = smem;                              // STAGES x kWStage
  uint8_t* xs = ws + C::STAGES * C::kWStage;       // STAGES x kXStage
  uint64_t* full = reinterpret_cast<uint64_t*>(xs + C::STAGES * C::kXStage);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;              // accumulator ready (commit)
  uint64_t* epi1 = accf + 1;                       // partials stored (4 warps)
  uint64_t* epi2 = epi1 + 1;                       // last-arrival known (1)
  uint64_t* epi3 = epi2 + 1;                       // outlier operands gathered (4 warps)
  uint64_t* ofull = epi3 + 1;                      // outlier product ready (commit)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ofull + 1);
  int* last_flag = reinterpret_cast<int*>(tmem_holder + 1);
  float* sxs = reinterpret_cast<float*>(tmem_holder + 4);  // [4 warps][MT]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tile order: token tile fastest, so the CTAs that share a weight tile run together
  const int ns = a.tiles_n * a.splits;
  const int mtile = static_cast<int>(blockIdx.x) % a.tiles_m;
  const int nts = static_cast<int>(blockIdx.x) / a.tiles_m;
  const int nt = nts / a.splits, split = nts % a.splits;
  const int s0 = static_cast<int>(static_cast<long long>(split) * a.KS / a.splits);
  const int s1 = static_cast<int>(static_cast<long long>(split + 1) * a.KS / a.splits);
  const int nst = s1 - s0;
  (void)ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accf, 1);
    mbar_init(epi1, 4);
    mbar_init(epi2, 1);
    mbar_init(epi3, 4);
    mbar_init(ofull, 1);
    fence_barrier_init();
    grid_dep_launch();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&wmap);
      prefetch_tensormap(&xmap);
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const int first = nst < C::STAGES ? nst : C::STAGES;
      // weights are constant: request the first ring before the dependency
      for (int it = 0; it < first; ++it) {
        mbar_arrive_expect_tx(&full[it], C::kWStage + C::kXStage);
        tma_load_3d(ws + it * C::kWStage, &wmap, (s0 + it) * 128, nt * 128, 0, &full[it], pol_w);
      }
      grid_dep_wait();  // q_x comes from the previous kernel
      int issued = 0;
      for (int it = 0; it < nst; ++it) {
        const int s = it % C::STAGES;
        if (it >= C::STAGES) {
          if (!mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1)) break;
          mbar_arrive_expect_tx(&full[s], C::kWStage + C::kXStage);
          tma_load_3d(ws + s * C::kWStage, &wmap, (s0 + it) * 128, nt * 128, 0, &full[s], pol_w);
        }
        tma_load_3d(xs + s * C::kXStage, &xmap, (s0 + it) * 128, mtile * C::MT, 0, &full[s], pol_x);
        ++issued;
      }
      if (issued < first)
        for (int it = issued; it < first; ++it) mbar_wait(&full[it], 0);
      for (int it = issued - 1; it >= 0 && it >= issued - C::STAGES; --it)
        mbar_wait(&full[it % C::STAGES], (it / C::STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_s8_s32(128, C::MT);
      for (int it = 0; it < nst; ++it) {
        const int s = it % C::STAGES;
        if (!mbar_wait(&full[s], (it / C::STAGES) & 1)) break;
        tc_fence_after();
        const uint32_t wa = smem_u32(ws + s * C::kWStage);
        const uint32_t xa = smem_u32(xs + s * C::kXStage);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_s8_ss(tmem, smem_desc_sw128(wa + kk * 32), smem_desc_sw128(xa + kk * 32), idesc,
                    (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      mma_commit(accf);
    }
  } else {
    // epilogue: warp (quadrant q) owns TMEM lanes 32q..32q+31 = weight rows
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int n = nt * 128 + row;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int tile_id = mtile * a.tiles_n + nt;
    if (__all_sync(0xffffffffu, mbar_wait(accf, 0))) {
      tc_fence_after();
      grid_dep_wait();  // s_x, the outlier list, Y and the workspace
      const float swn = n < a.N ? a.sw[n] : 0.0f;
      const int no = min(*a.ocount, a.K);
      // the tile's token scales, one copy per warp (all loads in flight at
      // once; the outputs then read them without a global round trip each)
      float* so = sxs + (warp - 2) * C::MT;
#pragma unroll
      for (int j = lane; j < C::MT; j += 32) {
        const int m = mtile * C::MT + j;
        so[j] = m < a.M ? a.sx[m] : 0.0f;
      }
      __syncwarp();
      const int nch = (no + 63) >> 6;  // 64-channel chunks of the outlier operands
      const bool tc_out =
          no > 0 && static_cast<long long>(nch) * C::kOChunkBytes <= C::kRingBytes;
      // byte offset of 16-byte unit u (channels 8u..8u+7) of row r in a
      // 128-byte swizzled K-major operand (8-row atoms of 1024 bytes)
      auto sw_off = [](int r, int u) { return (r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4); };
      // the outlier product D2 into tensor-memory columns [MT, 2 MT)
      bool have_d2 = false;
      auto outlier_mma = [&]() {
        const int e = threadIdx.x - 64;  // epilogue thread 0..127
        for (int c = 0; c < nch; ++c) {
          uint8_t* A = ws + c * C::kOChunkBytes;
          uint8_t* B = A + 128 * 128;
          for (int u = 0; u < 8; ++u) {  // this thread's weight row
            uint32_t pk[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              float v[2];
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                const int i = c * 64 + u * 8 + 2 * h + t;
                v[t] = 0.0f;
                if (i < no && n < a.N) {
                  const int k = a.olist[i];
                  if (in_bounds(static_cast<unsigned int>(k), static_cast<unsigned int>(a.K)))
                    v[t] = __fmul_rn(static_cast<float>(a.qw[static_cast<size_t>(n) * a.K + k]), swn);
                }
              }
              pk[h] = bf16x2_rn(v[0], v[1]);
            }
            *reinterpret_cast<uint4*>(A + sw_off(row, u)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          for (int idx = e; idx < C::MT * 8; idx += 128) {  // token rows
            const int r = idx >> 3, u = idx & 7;
            const int m = mtile * C::MT + r;
            uint32_t pk[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              uint32_t b2[2];
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                const int i = c * 64 + u * 8 + 2 * h + t;
                b2[t] = 0u;
                if (i < no && m < a.M) {
                  const int k = a.olist[i];
                  if (in_bounds(static_cast<unsigned int>(k), static_cast<unsigned int>(a.K)))
                    b2[t] = a.X[static_cast<size_t>(m) * a.K + k];
                }
              }
              pk[h] = b2[0] | (b2[1] << 16);
            }
            *reinterpret_cast<uint4*>(B + sw_off(r, u)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        fence_proxy_async_smem();  // the stores above are read by the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(epi3);
        if (threadIdx.x == 64) {
          if (mbar_wait(epi3, 0)) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16_f32(128, C::MT);
            int step = 0;
            for (int c = 0; c < nch; ++c) {
              const uint32_t Aa = smem_u32(ws + c * C::kOChunkBytes);
              const uint32_t Ba = Aa + 128 * 128;
              const int ksteps = min(4, (no - 64 * c + 15) >> 4);  // K = 16 each
              for (int kk = 0; kk < ksteps; ++kk, ++step)
                mma_bf16_ss(tmem + C::MT, smem_desc_sw128(Aa + kk * 32), smem_desc_sw128(Ba + kk * 32),
                            idesc, step > 0 ? 1u : 0u);
            }
          }
          mma_commit(ofull);  // (with no MMA issued it arrives at once)
        }
        have_d2 = __all_sync(0xffffffffu, mbar_wait(ofull, 0));
        tc_fence_after();
      };
      // y = acc s_x s_w + d; d from D2, or (operands beyond the ring) one fma
      // per outlier channel in ascending order from global memory
      auto finish = [&](int m, int v, float d2) {
        if (m >= a.M || n >= a.N) return;
        float y = __fmul_rn(__fmul_rn(static_cast<float>(v), so[m - mtile * C::MT]), swn);
        if (have_d2) {
          y = __fadd_rn(y, d2);
        } else {
          for (int i = 0; i < no; ++i) {
            const int k = a.olist[i];
            if (!in_bounds(static_cast<unsigned int>(k), static_cast<unsigned int>(a.K))) continue;
            const float w16 = __bfloat162float(__float2bfloat16_rn(
                __fmul_rn(static_cast<float>(a.qw[static_cast<size_t>(n) * a.K + k]), swn)));
            y = fmaf(bf16_bits_f32(a.X[static_cast<size_t>(m) * a.K + k]), w16, y);
          }
        }
        a.Y[static_cast<size_t>(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
      };
      int* part = a.partial + (static_cast<size_t>(tile_id) * a.splits + split) * C::MT * kI8Rows;
      if (a.splits == 1 && tc_out) outlier_mma();
#pragma unroll 1
      for (int cb = 0; cb < C::MT; cb += 8) {
        uint32_t v[8], d[8];
        tmem_ld8(tmem + lane_base + cb, v);
        if (a.splits == 1 && have_d2) tmem_ld8(tmem + lane_base + C::MT + cb, d);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int m = mtile * C::MT + cb + j;
          if (a.splits == 1) {
            finish(m, static_cast<int>(v[j]), have_d2 ? __uint_as_float(d[j]) : 0.0f);
          } else if (in_bounds(static_cast<unsigned long long>(part - a.partial) + (cb + j) * kI8Rows + row,
                               a.partial_count)) {
            part[(cb + j) * kI8Rows + row] = static_cast<int>(v[j]);
          }
        }
      }
      tc_fence_before();
      if (a.splits > 1) {
        // the last CTA of the tile sums the exact partials (any order)
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(epi1);
        if (threadIdx.x == 64) {
          if (mbar_wait(epi1, 0) && in_bounds(tile_id, 65536)) {
            const unsigned prev = atomicAdd(a.counter + tile_id, 1u);
            *last_flag = (prev == static_cast<unsigned>(a.splits - 1)) ? 1 : 0;
          } else {
            *last_flag = 0;
          }
          mbar_arrive(epi2);
        }
        if (__all_sync(0xffffffffu, mbar_wait(epi2, 0)) && *last_flag) {
          __threadfence();
          if (tc_out) outlier_mma();
          const int* base = a.partial + static_cast<size_t>(tile_id) * a.splits * C::MT * kI8Rows;
          // 8 columns of 4 K ranges at a time: 32 loads in flight per L2 round
          // trip (exact integer sums, so the order is free)
          constexpr int kSu = 4;
#pragma unroll 1
          for (int c0 = 0; c0 < C::MT; c0 += 8) {
            int acc[8] = {};
#pragma unroll 1
            for (int sp0 = 0; sp0 < a.splits; sp0 += kSu) {
              int v[kSu][8];
#pragma unroll
              for (int u = 0; u < kSu; ++u) {
                const int* src = base + (static_cast<size_t>(sp0 + u) * C::MT + c0) * kI8Rows + row;
                const bool ok = sp0 + u < a.splits &&
                                in_bounds(static_cast<unsigned long long>(src - a.partial) + 7 * kI8Rows,
                                          a.partial_count);
#pragma unroll
                for (int j = 0; j < 8; ++j) v[u][j] = ok ? __ldcg(src + j * kI8Rows) : 0;
              }
#pragma unroll
              for (int u = 0; u < kSu; ++u)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] += v[u][j];
            }
            float d2[8] = {};
            if (have_d2) {
              uint32_t d[8];
              tmem_ld8(tmem + lane_base + C::MT + c0, d);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 8; ++j) d2[j] = __uint_as_float(d[j]);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) finish(mtile * C::MT + c0 + j, acc[j], d2[j]);
          }
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    mbar_wait(accf, 0);  // every issued MMA has completed
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace w4
