// w4_prepack.cuh -- canonical (row-major nibbles + per-group constants) to the
// tile/stage layout that one bulk copy per pipeline stage brings into shared
// memory, plus the inverse used by the tests.
//
// Tile = 128 output rows = 8 row groups of 16; stage = 128 input channels =
// 8 channel blocks of 16.  For row group rg, channel block kb and lane t of a
// warp (g = t / 4, u = t % 4) one 32-bit word holds the 8 codes
//     rows r0 = 16 rg + g and r1 = r0 + 8,  channels k0 = 16 kb + 4 u .. k0 + 3
// as four pairs, pair j in bits 4j..4j+3 (first code) and 16+4j..19+4j
// (second code):
//     pair 0 = (r0, k0, k0+1)   pair 1 = (r0, k0+2, k0+3)
//     pair 2 = (r1, k0, k0+1)   pair 3 = (r1, k0+2, k0+3)
// so that ((word >> 4j) & 0x000F000F) is a pair of codes in the low nibble of
// each 16-bit half.  Pairs 0..3 are exactly the four registers a thread holds
// in the 16-lane x 256-bit tensor-memory access pattern (lanes g and g+8,
// 32-bit columns 2u and 2u+1) and, with the channel order inside a block
// permuted the same way on the activation side, the A fragment of a 16x16
// warp-level MMA.
//
// Stage block:
//   [0, 8192)  codes: [rg<8][kq<2][lane<32][4 words], word w covering kb = 4kq+w
//   INT4: scales fp16 [rg][group in stage][g<8][2] = (row r0, row r1),
//         then zeros u8 [rg][group][g<8] = z(r0) | z(r1) << 4
//   NF4:  absmax codes u8 [rg][block of 64 in stage (2)][g<8][2]
#pragma once

#include "w4_ptx.cuh"

namespace w4 {

constexpr int kTileRows = 128;
constexpr int kStageK = 128;
constexpr int kCodeBytes = kTileRows * kStageK / 2;  // 8192

__host__ __device__ constexpr int int4_stage_bytes(int G) {
  return kCodeBytes + kTileRows * (kStageK / G) * 2 + kTileRows * (kStageK / G) / 2;
}
__host__ __device__ constexpr int nf4_stage_bytes() { return kCodeBytes + kTileRows * 2; }

// Byte offsets inside a stage block.
__host__ __device__ constexpr int code_word_offset(int rg, int kb, int lane) {
  return (((rg * 2 + (kb >> 2)) * 32 + lane) * 4 + (kb & 3)) * 4;
}
__host__ __device__ constexpr int scale_pair_offset(int rg, int gl, int g, int gps) {
  return kCodeBytes + ((rg * gps + gl) * 8 + g) * 4;
}
__host__ __device__ constexpr int zero_pair_offset(int rg, int gl, int g, int gps) {
  return kCodeBytes + kTileRows * gps * 2 + (rg * gps + gl) * 8 + g;
}
__host__ __device__ constexpr int absmax_pair_offset(int rg, int blk, int g) {
  return kCodeBytes + ((rg * 2 + blk) * 8 + g) * 2;
}

__device__ __forceinline__ uint32_t nibble_at(const uint8_t* __restrict__ row_codes, int k) {
  return (row_codes[k >> 1] >> ((k & 1) * 4)) & 0xFu;
}

// The 8 code words of one (row group, lane) for one stage: kb = 0..7.
__device__ __forceinline__ void pack_stage_words(const uint8_t* __restrict__ Wq, int N, int K,
                                                 int n0, int kbase,
                                                 const int32_t* __restrict__ perm,
                                                 uint8_t* __restrict__ blk, int rg, int lane) {
  const int g = lane >> 2, u = lane & 3;
  const int r0 = n0 + rg * 16 + g, r1 = r0 + 8;
  const uint8_t* row0 = Wq + static_cast<size_t>(r0) * (K / 2);
  const uint8_t* row1 = Wq + static_cast<size_t>(r1) * (K / 2);
  uint32_t words[8];
#pragma unroll
  for (int kb = 0; kb < 8; ++kb) {
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = (j < 2) ? r0 : r1;
      const uint8_t* row = (j < 2) ? row0 : row1;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = kbase + kb * 16 + 4 * u + 2 * (j & 1) + e;  // prepacked channel
        uint32_t code = 0;
        if (r < N && k < K) {
          const int kk = perm ? perm[k] : k;
          if (in_bounds(static_cast<unsigned int>(kk), static_cast<unsigned int>(K)))
            code = nibble_at(row, kk);
        }
        w |= code << (e ? 16 + 4 * j : 4 * j);
      }
    }
    words[kb] = w;
  }
  uint4* dst = reinterpret_cast<uint4*>(blk + code_word_offset(rg, 0, lane));
  dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
  uint4* dst1 = reinterpret_cast<uint4*>(blk + code_word_offset(rg, 4, lane));
  dst1[0] = make_uint4(words[4], words[5], words[6], words[7]);
}

// grid (stages, tiles), block 256 = 8 row groups x 32 lanes.
__global__ void int4_prepack_kernel(const uint8_t* __restrict__ Wq,
                                    const uint16_t* __restrict__ scales,
                                    const uint8_t* __restrict__ zeros,
                                    const int32_t* __restrict__ perm, int N, int K, int G,
                                    uint8_t* __restrict__ Wp) {
  const int s = blockIdx.x, nt = blockIdx.y;
  const int rg = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = gridDim.x;
  const int gps = kStageK / G, ng = K / G;
  uint8_t* blk = Wp + (static_cast<size_t>(nt) * KS + s) * int4_stage_bytes(G);
  const int n0 = nt * kTileRows;
  pack_stage_words(Wq, N, K, n0, s * kStageK, perm, blk, rg, lane);
  if (lane < 8) {
    const int g = lane;
    const int r0 = n0 + rg * 16 + g, r1 = r0 + 8;
    for (int gl = 0; gl < gps; ++gl) {
      const int gg = s * gps + gl;
      uint32_t s0 = 0, s1 = 0, z0 = 0, z1 = 0;
      if (gg < ng) {
        if (r0 < N) {
          s0 = scales[static_cast<size_t>(r0) * ng + gg];
          z0 = zeros[static_cast<size_t>(r0) * ng + gg] & 0xFu;
        }
        if (r1 < N) {
          s1 = scales[static_cast<size_t>(r1) * ng + gg];
          z1 = zeros[static_cast<size_t>(r1) * ng + gg] & 0xFu;
        }
      }
      *reinterpret_cast<uint32_t*>(blk + scale_pair_offset(rg, gl, g, gps)) = s0 | (s1 << 16);
      blk[zero_pair_offset(rg, gl, g, gps)] = static_cast<uint8_t>(z0 | (z1 << 4));
    }
  }
  // The GEMM kernels start streaming Wp before their launch dependency on
  // the previous kernel resolves: make every write visible before exiting.
  __threadfence();
}

// grid (stages, tiles), block 256.
__global__ void nf4_prepack_kernel(const uint8_t* __restrict__ Wq,
                                   const uint8_t* __restrict__ absmax_q, int N, int K,
                                   uint8_t* __restrict__ Wp) {
  const int s = blockIdx.x, nt = blockIdx.y;
  const int rg = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = gridDim.x;
  uint8_t* blk = Wp + (static_cast<size_t>(nt) * KS + s) * nf4_stage_bytes();
  const int n0 = nt * kTileRows;
  pack_stage_words(Wq, N, K, n0, s * kStageK, nullptr, blk, rg, lane);
  if (lane < 8) {
    const int g = lane;
    const int bpr = K / 64;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int bi = s * 2 + b;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = n0 + rg * 16 + g + 8 * h;
        uint8_t v = 0;
        if (r < N && bi < bpr) v = absmax_q[static_cast<size_t>(r) * bpr + bi];
        blk[absmax_pair_offset(rg, b, g) + h] = v;
      }
    }
  }
  __threadfence();  // as in int4_prepack_kernel
}

// Act-order channel permutation: a stable sort of k by g_idx[k] when every
// group has exactly G members.  One thread per group scans g_idx in order.
// Out-of-range values or a group of the wrong size set W4_DEV_ERR_INPUT (and
// the permutation is then filled with the identity so that no later gather
// can go out of bounds).
__global__ void act_order_perm_kernel(const int32_t* __restrict__ g_idx, int K, int G,
                                      int32_t* __restrict__ perm) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  const int ng = K / G;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const int g = g_idx[k];
    if (g < 0 || g >= ng) bad = 1;
  }
  __syncthreads();
  for (int g = threadIdx.x; g < ng; g += blockDim.x) {
    int cnt = 0;
    for (int k = 0; k < K; ++k) {
      if (g_idx[k] == g) {
        if (cnt < G) perm[g * G + cnt] = k;
        ++cnt;
      }
    }
    if (cnt != G) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) set_dev_error(W4_DEV_ERR_INPUT);
    for (int k = threadIdx.x; k < K; k += blockDim.x) perm[k] = k;
  }
  __threadfence();  // as in int4_prepack_kernel
}

// Inverse of int4_prepack_kernel in prepacked channel order.  grid (stages,
// tiles), block 256 = 8 row groups x 32 lanes.
__global__ void int4_unprepack_kernel(const uint8_t* __restrict__ Wp, int N, int K, int G,
                                      uint8_t* __restrict__ Wq, uint16_t* __restrict__ scales,
                                      uint8_t* __restrict__ zeros) {
  const int s = blockIdx.x, nt = blockIdx.y;
  const int rg = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = gridDim.x;
  const int gps = kStageK / G, ng = K / G;
  const uint8_t* blk = Wp + (static_cast<size_t>(nt) * KS + s) * int4_stage_bytes(G);
  const int g = lane >> 2, u = lane & 3;
  const int r0 = nt * kTileRows + rg * 16 + g, r1 = r0 + 8;
  for (int kb = 0; kb < 8; ++kb) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(blk + code_word_offset(rg, kb, lane));
    for (int j = 0; j < 4; ++j) {
      const int r = (j < 2) ? r0 : r1;
      const int k = s * kStageK + kb * 16 + 4 * u + 2 * (j & 1);  // even
      if (r >= N || k >= K) continue;
      const uint32_t lo = (w >> (4 * j)) & 0xFu;
      const uint32_t hi = (w >> (16 + 4 * j)) & 0xFu;
      Wq[static_cast<size_t>(r) * (K / 2) + k / 2] = static_cast<uint8_t>(lo | (hi << 4));
    }
  }
  if (lane < 8) {
    for (int gl = 0; gl < gps; ++gl) {
      const int gg = s * gps + gl;
      if (gg >= ng) continue;
      const uint32_t sp = *reinterpret_cast<const uint32_t*>(blk + scale_pair_offset(rg, gl, lane, gps));
      const uint32_t zp = blk[zero_pair_offset(rg, gl, lane, gps)];
      const int a = nt * kTileRows + rg * 16 + lane, b = a + 8;
      if (a < N) {
        scales[static_cast<size_t>(a) * ng + gg] = static_cast<uint16_t>(sp & 0xFFFFu);
        zeros[static_cast<size_t>(a) * ng + gg] = zp & 0xFu;
      }
      if (b < N) {
        scales[static_cast<size_t>(b) * ng + gg] = static_cast<uint16_t>(sp >> 16);
        zeros[static_cast<size_t>(b) * ng + gg] = zp >> 4;
      }
    }
  }
}

}  // namespace w4
