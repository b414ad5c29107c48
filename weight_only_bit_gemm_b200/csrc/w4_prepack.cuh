// w4_prepack.cuh -- canonical (row-major nibbles + per-group constants) to the
// tile/stage layout that one bulk copy per pipeline stage brings into shared
// memory, plus the inverse used by the tests.
//
// Tile = 128 output rows, stage = 128 input channels.  Stage block:
//   [0, 8192)           codes: [chunk c<4][row r<128][16 B]; in each 32-bit
//                       word of channels k0..k0+7, bits 4j.. hold k0+2j and
//                       bits 16+4j.. hold k0+2j+1, so that
//                       ((word >> 4j) & 0x000F000F) is a pair of codes in the
//                       low nibble of each 16-bit half.
//   INT4: scales fp16 [row][gps], then zeros 4-bit [row][gps] (gps = 128/G)
//   NF4:  absmax codes [row][2]
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

__device__ __forceinline__ uint32_t nibble_at(const uint8_t* __restrict__ row_codes, int k) {
  return (row_codes[k >> 1] >> ((k & 1) * 4)) & 0xFu;
}

// Codes of one stage for one row (thread): gathers through `perm` when given.
__device__ __forceinline__ void pack_stage_codes(const uint8_t* __restrict__ Wq, int n, int N,
                                                 int K, int kbase,
                                                 const int32_t* __restrict__ perm,
                                                 uint8_t* __restrict__ dst_block, int r) {
  const uint8_t* row = Wq + static_cast<size_t>(n) * (K / 2);
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t words[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t w = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j = kbase + 32 * c + 8 * i + e;  // channel in prepacked order
        uint32_t code = 0;
        if (n < N && j < K) code = nibble_at(row, perm ? perm[j] : j);
        const int pair = e >> 1;
        w |= code << ((e & 1) ? (16 + 4 * pair) : (4 * pair));
      }
      words[i] = w;
    }
    *reinterpret_cast<uint4*>(dst_block + c * 2048 + r * 16) =
        make_uint4(words[0], words[1], words[2], words[3]);
  }
}

// grid (stages, tiles), block 128.
__global__ void int4_prepack_kernel(const uint8_t* __restrict__ Wq,
                                    const uint16_t* __restrict__ scales,
                                    const uint8_t* __restrict__ zeros,
                                    const int32_t* __restrict__ perm, int N, int K, int G,
                                    uint8_t* __restrict__ Wp) {
  const int s = blockIdx.x, nt = blockIdx.y, r = threadIdx.x;
  const int KS = gridDim.x;
  const int gps = kStageK / G, ng = K / G;
  const int sb = int4_stage_bytes(G);
  uint8_t* blk = Wp + (static_cast<size_t>(nt) * KS + s) * sb;
  const int n = nt * kTileRows + r;
  pack_stage_codes(Wq, n, N, K, s * kStageK, perm, blk, r);
  uint16_t* sc = reinterpret_cast<uint16_t*>(blk + kCodeBytes);
  uint8_t* zb = blk + kCodeBytes + kTileRows * gps * 2;
  uint32_t znib = 0;  // this row's zero nibbles, group gl at bits 4*gl
  for (int gl = 0; gl < gps; ++gl) {
    const int g = s * gps + gl;
    uint16_t sv = 0;
    uint32_t zv = 0;
    if (n < N && g < ng) {
      sv = scales[static_cast<size_t>(n) * ng + g];
      zv = zeros[static_cast<size_t>(n) * ng + g] & 0xFu;
    }
    sc[r * gps + gl] = sv;
    znib |= zv << (4 * gl);
  }
  if (gps == 1) {
    // two rows share a byte: the even row writes it
    const uint32_t other = __shfl_down_sync(0xffffffffu, znib, 1);
    if ((r & 1) == 0) zb[r >> 1] = static_cast<uint8_t>(znib | (other << 4));
  } else {
    for (int b = 0; b < gps / 2; ++b) zb[r * (gps / 2) + b] = static_cast<uint8_t>(znib >> (8 * b));
  }
}

// grid (stages, tiles), block 128.
__global__ void nf4_prepack_kernel(const uint8_t* __restrict__ Wq,
                                   const uint8_t* __restrict__ absmax_q, int N, int K,
                                   uint8_t* __restrict__ Wp) {
  const int s = blockIdx.x, nt = blockIdx.y, r = threadIdx.x;
  const int KS = gridDim.x;
  uint8_t* blk = Wp + (static_cast<size_t>(nt) * KS + s) * nf4_stage_bytes();
  const int n = nt * kTileRows + r;
  pack_stage_codes(Wq, n, N, K, s * kStageK, nullptr, blk, r);
  const int bpr = K / 64;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int b = s * 2 + h;
    uint8_t v = 0;
    if (n < N && b < bpr) v = absmax_q[static_cast<size_t>(n) * bpr + b];
    blk[kCodeBytes + r * 2 + h] = v;
  }
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
}

// Inverse of int4_prepack_kernel in prepacked channel order.  grid (stages,
// tiles), block 128.
__global__ void int4_unprepack_kernel(const uint8_t* __restrict__ Wp, int N, int K, int G,
                                      uint8_t* __restrict__ Wq, uint16_t* __restrict__ scales,
                                      uint8_t* __restrict__ zeros) {
  const int s = blockIdx.x, nt = blockIdx.y, r = threadIdx.x;
  const int KS = gridDim.x;
  const int gps = kStageK / G, ng = K / G;
  const uint8_t* blk = Wp + (static_cast<size_t>(nt) * KS + s) * int4_stage_bytes(G);
  const int n = nt * kTileRows + r;
  if (n >= N) return;
  for (int c = 0; c < 4; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(blk + c * 2048 + r * 16);
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
    for (int i = 0; i < 4; ++i) {
      for (int p = 0; p < 4; ++p) {
        const int j = s * kStageK + 32 * c + 8 * i + 2 * p;
        if (j >= K) continue;
        const uint32_t lo = (words[i] >> (4 * p)) & 0xFu;
        const uint32_t hi = (words[i] >> (16 + 4 * p)) & 0xFu;
        Wq[static_cast<size_t>(n) * (K / 2) + j / 2] = static_cast<uint8_t>(lo | (hi << 4));
      }
    }
  }
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(blk + kCodeBytes);
  const uint8_t* zb = blk + kCodeBytes + kTileRows * gps * 2;
  for (int gl = 0; gl < gps; ++gl) {
    const int g = s * gps + gl;
    if (g >= ng) continue;
    scales[static_cast<size_t>(n) * ng + g] = sc[r * gps + gl];
    const int idx = r * gps + gl;
    zeros[static_cast<size_t>(n) * ng + g] = (zb[idx >> 1] >> ((idx & 1) * 4)) & 0xFu;
  }
}

}  // namespace w4
