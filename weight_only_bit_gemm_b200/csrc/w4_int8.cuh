// w4_int8.cuh -- LLM.int8 mixed decomposition (W8A8 with 16-bit outliers).
//
// "大模型量化选型：五种主流方案对比与实战" §2.1: vector-wise quantization (one
// scale per output feature of the weights) and mixed-precision decomposition
// (input channels whose activation exceeds the threshold, 6.0, in magnitude
// go through a 16-bit product, the others through INT8, and the two results
// are added); "【推理与部署篇05】模型量化部署深度对比" §6.1: llm_int8_threshold 6.0,
// no 16-bit copy of the weights.  Per call:
//   outliers  one CTA: flag[k] = |x[m,k]| > threshold for some token m, and
//             the ascending list of flagged channels (block prefix sum);
//   quantize  one CTA per token: s_x = max over unflagged |x| / 127,
//             q_x = clamp(rint(x / s_x), +-127), 0 on flagged channels;
//   product   warp-level INT8 MMAs (m16n8k32, s32 accumulate) over
//             (16-row tile, K slice) work items, exact int32 partial sums
//             added atomically (exact, so the order does not matter);
//   epilogue  y = acc s_x s_w + sum over flagged k of x * bf16(q_w s_w).
#pragma once

#include <cuda_bf16.h>

#include "w4_ptx.cuh"

namespace w4 {

constexpr int kInt8Warps = 8;      // warps per product CTA
constexpr int kInt8MaxNB = 4;      // token blocks of 8 per pass over the weights

__device__ __forceinline__ float bf16_bits_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// q_w = clamp(rint(w / s_w), +-127), s_w = max_k |w| / 127 (1 if 0); one CTA per row.
__global__ void __launch_bounds__(256) int8_quantize_weights_kernel(const float* __restrict__ W,
                                                                    int N, int K,
                                                                    int8_t* __restrict__ qw,
                                                                    float* __restrict__ sw) {
  __shared__ float red[256];
  const int n = blockIdx.x;
  const float* row = W + static_cast<size_t>(n) * K;
  float a = 0.0f;
  for (int k = threadIdx.x; k < K; k += 256) a = fmaxf(a, fabsf(row[k]));
  red[threadIdx.x] = a;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  float s = __fdiv_rn(red[0], 127.0f);
  if (s == 0.0f) s = 1.0f;
  if (threadIdx.x == 0) sw[n] = s;
  for (int k = threadIdx.x; k < K; k += 256) {
    const float q = fminf(fmaxf(rintf(__fdiv_rn(row[k], s)), -127.0f), 127.0f);
    qw[static_cast<size_t>(n) * K + k] = static_cast<int8_t>(q);
  }
}

// Outlier channels of the call (one CTA of 1024 threads; thread t owns the
// contiguous channel range [t c, (t + 1) c)), listed in ascending order.
__global__ void __launch_bounds__(1024) int8_outliers_kernel(const uint16_t* __restrict__ X, int M,
                                                             int K, float threshold,
                                                             uint8_t* __restrict__ flag,
                                                             int32_t* __restrict__ list,
                                                             int32_t* __restrict__ count) {
  __shared__ int warp_sum[32];
  const int t = threadIdx.x;
  const int c = (K + 1023) / 1024;
  const int k0 = min(K, t * c), k1 = min(K, k0 + c);
  int mine = 0;
  for (int k = k0; k < k1; ++k) {
    bool o = false;
    for (int m = 0; m < M && !o; ++m)
      o = fabsf(bf16_bits_f32(X[static_cast<size_t>(m) * K + k])) > threshold;
    flag[k] = o ? 1 : 0;
    mine += o ? 1 : 0;
  }
  // exclusive prefix sum of `mine` over the block
  const int lane = t & 31, wid = t >> 5;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sum[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int v = warp_sum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    warp_sum[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  int base = incl - mine + (wid > 0 ? warp_sum[wid - 1] : 0);
  for (int k = k0; k < k1; ++k)
    if (flag[k] && in_bounds(static_cast<unsigned int>(base), static_cast<unsigned int>(K)))
      list[base++] = k;
  if (t == 1023) *count = warp_sum[31];
}

// Per token: s_x = max over unflagged channels |x| / 127 (1 if 0); q_x.
__global__ void __launch_bounds__(256) int8_quantize_x_kernel(const uint16_t* __restrict__ X,
                                                              const uint8_t* __restrict__ flag,
                                                              int K, int8_t* __restrict__ qx,
                                                              float* __restrict__ sx) {
  __shared__ float red[256];
  const int m = blockIdx.x;
  const uint16_t* row = X + static_cast<size_t>(m) * K;
  float a = 0.0f;
  for (int k = threadIdx.x; k < K; k += 256)
    if (!flag[k]) a = fmaxf(a, fabsf(bf16_bits_f32(row[k])));
  red[threadIdx.x] = a;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  float s = __fdiv_rn(red[0], 127.0f);
  if (s == 0.0f) s = 1.0f;
  if (threadIdx.x == 0) sx[m] = s;
  for (int k = threadIdx.x; k < K; k += 256) {
    float q = 0.0f;
    if (!flag[k]) q = fminf(fmaxf(rintf(__fdiv_rn(bf16_bits_f32(row[k]), s)), -127.0f), 127.0f);
    qx[static_cast<size_t>(m) * K + k] = static_cast<int8_t>(q);
  }
}

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// acc[m][n] += sum over the warp's K slice of q_x[m][k] q_w[n][k].
// Work item = (16-row tile, slice of `steps` 64-channel steps); lane (g, u)
// = (lane / 4, lane % 4) loads 16 consecutive bytes of weight rows g and
// g + 8 and of token row g at channel k0 + 16u: bytes 0-3 / 4-7 feed the
// first MMA's k-slots 4u.. / 16 + 4u.., bytes 8-15 the second MMA's.  A and
// B use the same channel-to-slot map, so the exact sum is the plain dot
// product.  Tokens in passes of up to kInt8MaxNB blocks of 8.
__global__ void __launch_bounds__(kInt8Warps * 32) int8_product_kernel(
    const int8_t* __restrict__ qw, const int8_t* __restrict__ qx, int M, int N, int K,
    int row_tiles, int slices, int steps, int* __restrict__ acc) {
  const int lane = threadIdx.x & 31, g = lane >> 2, u = lane & 3;
  const long long item = static_cast<long long>(blockIdx.x) * kInt8Warps + (threadIdx.x >> 5);
  if (item >= static_cast<long long>(row_tiles) * slices) return;
  const int rt = static_cast<int>(item % row_tiles);
  const int sl = static_cast<int>(item / row_tiles);
  const int r0 = rt * 16 + g, r1 = r0 + 8;
  const int kbeg = sl * steps * 64;
  const int kend = min(K, kbeg + steps * 64);
  const int NB = (M + 7) / 8;
  for (int tb0 = 0; tb0 < NB; tb0 += kInt8MaxNB) {
    int d[kInt8MaxNB][4] = {};
    for (int k0 = kbeg; k0 < kend; k0 += 64) {
      const int kk = k0 + 16 * u;
      if (!in_bounds(static_cast<unsigned int>(kk + 15), static_cast<unsigned int>(K))) continue;
      uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = make_uint4(0u, 0u, 0u, 0u);
      if (r0 < N) wa = *reinterpret_cast<const uint4*>(qw + static_cast<size_t>(r0) * K + kk);
      if (r1 < N) wb = *reinterpret_cast<const uint4*>(qw + static_cast<size_t>(r1) * K + kk);
#pragma unroll
      for (int j = 0; j < kInt8MaxNB; ++j) {
        const int tok = (tb0 + j) * 8 + g;
        if (tb0 + j >= NB) break;
        uint4 xv = make_uint4(0u, 0u, 0u, 0u);
        if (tok < M) xv = *reinterpret_cast<const uint4*>(qx + static_cast<size_t>(tok) * K + kk);
        mma_s8_16832(d[j], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
        mma_s8_16832(d[j], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
      }
    }
#pragma unroll
    for (int j = 0; j < kInt8MaxNB; ++j) {
      if (tb0 + j >= NB) break;
      const int t0 = (tb0 + j) * 8 + 2 * u;
      // d0, d1: row r0, tokens t0, t0 + 1; d2, d3: row r1
      if (r0 < N && t0 < M) atomicAdd(&acc[static_cast<size_t>(t0) * N + r0], d[j][0]);
      if (r0 < N && t0 + 1 < M) atomicAdd(&acc[static_cast<size_t>(t0 + 1) * N + r0], d[j][1]);
      if (r1 < N && t0 < M) atomicAdd(&acc[static_cast<size_t>(t0) * N + r1], d[j][2]);
      if (r1 < N && t0 + 1 < M) atomicAdd(&acc[static_cast<size_t>(t0 + 1) * N + r1], d[j][3]);
    }
  }
}

// y[m][n] = acc s_x s_w + sum over listed outlier channels x * bf16(q_w s_w).
__global__ void int8_epilogue_kernel(const int* __restrict__ acc, const float* __restrict__ sx,
                                     const float* __restrict__ sw, const uint16_t* __restrict__ X,
                                     const int8_t* __restrict__ qw,
                                     const int32_t* __restrict__ list,
                                     const int32_t* __restrict__ count, int M, int N, int K,
                                     uint16_t* __restrict__ Y) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<size_t>(M) * N) return;
  const int m = static_cast<int>(idx / N);
  const int n = static_cast<int>(idx - static_cast<size_t>(m) * N);
  const float s = sw[n];
  float y = __fmul_rn(__fmul_rn(static_cast<float>(acc[idx]), sx[m]), s);
  const int no = *count;
  for (int i = 0; i < no; ++i) {
    if (!in_bounds(static_cast<unsigned int>(i), static_cast<unsigned int>(K))) break;
    const int k = list[i];
    if (!in_bounds(static_cast<unsigned int>(k), static_cast<unsigned int>(K))) continue;
    const float w16 = __bfloat162float(__float2bfloat16_rn(
        __fmul_rn(static_cast<float>(qw[static_cast<size_t>(n) * K + k]), s)));
    y = fmaf(bf16_bits_f32(X[static_cast<size_t>(m) * K + k]), w16, y);
  }
  Y[idx] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
}

}  // namespace w4
