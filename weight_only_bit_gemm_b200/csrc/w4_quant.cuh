// w4_quant.cuh -- quantize / dequantize kernels (INT4 asymmetric RTN, NF4 with
// double-quantized absmax).  Every floating-point step uses the explicit
// round-to-nearest intrinsics so that no multiply-add is contracted and the
// results are bit-identical to the CPU definition.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "w4_ptx.cuh"

namespace w4 {

// ---------------------------------------------------------------- INT4 RTN
// "【推理与部署篇05】模型量化部署深度对比" §2.3 (asymmetric min-max, /(2^b-1),
// zero_point = round(-min/scale)), with b = 4; group-wise per §2.2.

struct RtnParam {
  float sf;   // fp16 scale widened to fp32
  float zp;   // zero point 0..15
  float lo;   // lowest code: 0 (asymmetric) or 1 (symmetric, levels -7..7)
  uint16_t s16;
};

// From the group's largest positive part mx = max(w, 0) and largest negative
// magnitude nx = max(-w, 0) (so the range always includes 0).
__device__ __forceinline__ RtnParam rtn_param(float mx, float nx) {
  const float mn = -nx;
  const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
  __half s16 = __float2half_rn(s32);
  if (__half2float(s16) == 0.0f) s16 = __float2half_rn(1.0f);
  RtnParam p;
  p.s16 = __half_as_ushort(s16);
  p.sf = __half2float(s16);
  float z = rintf(__fdiv_rn(nx, p.sf));
  p.zp = fminf(fmaxf(z, 0.0f), 15.0f);
  p.lo = 0.0f;
  return p;
}

// Symmetric (absmax) form of the same section: scale = max|w| / (2^(b-1) - 1)
// = max|w| / 7 for b = 4, levels -7..7 stored with zero point 8.
__device__ __forceinline__ RtnParam sym_param(float mx, float nx) {
  const float s32 = __fdiv_rn(fmaxf(mx, nx), 7.0f);
  __half s16 = __float2half_rn(s32);
  if (__half2float(s16) == 0.0f) s16 = __float2half_rn(1.0f);
  RtnParam p;
  p.s16 = __half_as_ushort(s16);
  p.sf = __half2float(s16);
  p.zp = 8.0f;
  p.lo = 1.0f;
  return p;
}

// rint(w / scale) + zp clamped to [lo, 15]; for the symmetric form that is
// clamp(rint(w / scale), -7, 7) + 8 (all values are small integers in fp32).
__device__ __forceinline__ uint32_t rtn_code(float w, const RtnParam& p) {
  float q = __fadd_rn(rintf(__fdiv_rn(w, p.sf)), p.zp);
  q = fminf(fmaxf(q, p.lo), 15.0f);
  return static_cast<uint32_t>(q);
}

// One CTA per output row.  Shared memory: per-group max(w,0) and max(-w,0)
// as ordered non-negative float bit patterns (so integer max is float max).
// Dynamic shared memory: 2 * ngroups * 4 bytes + 2 * ngroups * 4 bytes.
// SYM selects the symmetric scale and zero point 8.
template <bool SYM>
__global__ void __launch_bounds__(256) rtn_quantize_kernel(
    const float* __restrict__ W, int N, int K, int G, const int32_t* __restrict__ g_idx,
    uint8_t* __restrict__ Wq, uint16_t* __restrict__ scales, uint8_t* __restrict__ zeros) {
  extern __shared__ uint32_t sm_q[];
  const int ng = K / G;
  uint32_t* pos_bits = sm_q;            // [ng]
  uint32_t* neg_bits = sm_q + ng;       // [ng]
  float* sf_s = reinterpret_cast<float*>(sm_q + 2 * ng);
  float* zp_s = sf_s + ng;
  const int n = blockIdx.x;
  const float* row = W + static_cast<size_t>(n) * K;
  const unsigned long long nk = static_cast<unsigned long long>(N) * K;  // extents
  const unsigned long long nrow0 = static_cast<unsigned long long>(n) * K;

  for (int g = threadIdx.x; g < ng; g += blockDim.x) {
    pos_bits[g] = 0u;
    neg_bits[g] = 0u;
  }
  __syncthreads();

  if (g_idx == nullptr) {
    // contiguous groups: one warp reduces one group at a time
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int g = warp; g < ng; g += blockDim.x >> 5) {
      float mx = 0.0f, nx = 0.0f;
      for (int k = lane; k < G; k += 32) {
        if (!in_bounds(nrow0 + g * G + k, nk)) continue;
        const float w = row[g * G + k];
        if (w > mx) mx = w;
        if (-w > nx) nx = -w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        nx = fmaxf(nx, __shfl_xor_sync(0xffffffffu, nx, o));
      }
      if (lane == 0) {
        pos_bits[g] = __float_as_uint(mx);
        neg_bits[g] = __float_as_uint(nx);
      }
    }
  } else {
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
      if (!in_bounds(nrow0 + k, nk)) continue;
      const int g = g_idx[k];
      if (g < 0 || g >= ng) {
        set_dev_error(W4_DEV_ERR_INPUT);
        continue;
      }
      const float w = row[k];
      // bit patterns of max(w, 0) and max(-w, 0); never a negative zero,
      // whose pattern would compare above every positive value
      atomicMax(&pos_bits[g], w > 0.0f ? __float_as_uint(w) : 0u);
      atomicMax(&neg_bits[g], w < 0.0f ? __float_as_uint(-w) : 0u);
    }
  }
  __syncthreads();

  for (int g = threadIdx.x; g < ng; g += blockDim.x) {
    const float mx = __uint_as_float(pos_bits[g]), nx = __uint_as_float(neg_bits[g]);
    const RtnParam p = SYM ? sym_param(mx, nx) : rtn_param(mx, nx);
    sf_s[g] = p.sf;
    zp_s[g] = p.zp;
    if (!in_bounds(static_cast<unsigned long long>(n) * ng + g,
                   static_cast<unsigned long long>(N) * ng))
      continue;
    scales[static_cast<size_t>(n) * ng + g] = p.s16;
    zeros[static_cast<size_t>(n) * ng + g] = static_cast<uint8_t>(p.zp);
  }
  __syncthreads();

  uint8_t* out = Wq + static_cast<size_t>(n) * (K / 2);
  for (int b = threadIdx.x; b < K / 2; b += blockDim.x) {
    uint32_t code[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int k = 2 * b + e;
      int g = g_idx ? g_idx[k] : k / G;
      if (g < 0 || g >= ng || !in_bounds(nrow0 + k, nk)) {
        code[e] = 0;
        continue;
      }
      RtnParam p;
      p.sf = sf_s[g];
      p.zp = zp_s[g];
      p.lo = SYM ? 1.0f : 0.0f;
      code[e] = rtn_code(row[k], p);
    }
    if (in_bounds(nrow0 / 2 + b, nk / 2)) out[b] = static_cast<uint8_t>(code[0] | (code[1] << 4));
  }
}

// rint(RN(w / s)) without a division in the common case.  With r = RN(1/s),
// t = RN(w r) and the exact quotient Q = w / s differ by at most
// |Q| (2^-23 + 2^-48), and so do RN(Q) and Q by |Q| 2^-24: when t lies
// further than |t| 2^-19 from every half-integer, Q, RN(Q) and t all round to
// the same integer (ties included, as RN(Q) cannot sit on a half-integer
// either).  Otherwise the IEEE division decides.
__device__ __forceinline__ float rint_quotient(float w, float s, float r) {
  const float t = __fmul_rn(w, r);
  const float c = rintf(t);
  const float d = fabsf(__fsub_rn(t, c));  // exact: |t - c| <= 1/2
  if (fabsf(__fsub_rn(d, 0.5f)) > __fmaf_rn(fabsf(t), 0x1p-19f, 0x1p-60f)) return c;
  return rintf(__fdiv_rn(w, s));
}

// Contiguous groups (no g_idx): W is N*K/G consecutive groups of G weights in
// row-major order (K % G == 0), so the kernel works on the flat array.  A warp
// takes a chunk of 512 weights (512 / G whole groups); a group belongs to G/16
// lanes, each holding 16 of its weights as four float4 loads (load u of lane j
// of the group is float4 u * G/16 + j, so that every load instruction reads
// whole 32..128-byte runs).  Each lane reduces max(w, 0) and max(-w, 0) over
// its 16 weights, the group's lanes combine them with shuffles, and every lane
// derives the group's scale and zero point itself and writes 2 bytes of codes
// per float4; the group's first lane writes the scale and zero point.
template <bool SYM, int G>
__global__ void __launch_bounds__(256) rtn_quantize_flat_kernel(
    const float* __restrict__ W, long long ngroups, uint8_t* __restrict__ Wq,
    uint16_t* __restrict__ scales, uint8_t* __restrict__ zeros) {
  constexpr int kLpg = G / 16;     // lanes per group
  constexpr int kGpc = 32 / kLpg;  // groups per 512-weight chunk
  const int lane = threadIdx.x & 31;
  const int gi = lane / kLpg, j = lane % kLpg;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long nchunks = (ngroups + kGpc - 1) / kGpc;
  const unsigned long long n4 = static_cast<unsigned long long>(ngroups) * (G / 4);  // float4s
  const float4* src = reinterpret_cast<const float4*>(W);
  for (long long c = warp; c < nchunks; c += nwarps) {
    const long long grp = c * kGpc + gi;
    const bool valid = grp < ngroups;  // whole groups only: the same for a group's lanes
    const long long f0 = grp * (G / 4) + j;  // this lane's first float4
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      v[u] = valid && in_bounds(f0 + u * kLpg, n4) ? __ldcs(src + f0 + u * kLpg)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    // max(w, 0) and max(-w, 0) without ever producing -0
    float mx = 0.0f, nx = 0.0f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (w[e] > mx) mx = w[e];
        if (-w[e] > nx) nx = -w[e];
      }
    }
#pragma unroll
    for (int o = 1; o < kLpg; o <<= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      nx = fmaxf(nx, __shfl_xor_sync(0xffffffffu, nx, o));
    }
    if (!valid) continue;
    const RtnParam p = SYM ? sym_param(mx, nx) : rtn_param(mx, nx);
    const float r = __frcp_rn(p.sf);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t codes = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float q = __fadd_rn(rint_quotient(w[e], p.sf, r), p.zp);
        q = fminf(fmaxf(q, p.lo), 15.0f);
        codes |= static_cast<uint32_t>(q) << (4 * e);
      }
      // float4 f0 + u * kLpg holds weights 4 (f0 + u * kLpg) .. + 3: code bytes 2 (f0 + ...)
      const unsigned long long h = static_cast<unsigned long long>(f0 + u * kLpg);
      if (in_bounds(h, n4)) reinterpret_cast<uint16_t*>(Wq)[h] = static_cast<uint16_t>(codes);
    }
    if (j == 0 && in_bounds(static_cast<unsigned long long>(grp), static_cast<unsigned long long>(ngroups))) {
      scales[grp] = p.s16;
      zeros[grp] = static_cast<uint8_t>(p.zp);
    }
  }
}

// Contiguous groups: 16 consecutive weights per thread (one group, as G is a
// multiple of 16), flat over the row-major array.
template <int G>
__global__ void rtn_dequant_flat_kernel(const uint8_t* __restrict__ Wq,
                                        const uint16_t* __restrict__ scales,
                                        const uint8_t* __restrict__ zeros, long long total16,
                                        uint16_t* __restrict__ out) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= total16) return;
  const long long e0 = i * 16;
  if (!in_bounds(e0 / G, static_cast<unsigned long long>(total16) * 16 / G)) return;
  const uint2 codes = __ldcs(reinterpret_cast<const uint2*>(Wq) + i);
  const float sf = __half2float(__ushort_as_half(scales[e0 / G]));
  const float z = static_cast<float>(zeros[e0 / G]);
  uint32_t res[8];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint32_t word = e < 8 ? codes.x : codes.y;
    const float q = static_cast<float>((word >> (4 * (e & 7))) & 0xFu);
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__fsub_rn(q, z), sf)));
    if (e & 1)
      res[e >> 1] |= b << 16;
    else
      res[e >> 1] = b;
  }
  uint4* dst = reinterpret_cast<uint4*>(out + e0);
  __stcs(dst, make_uint4(res[0], res[1], res[2], res[3]));
  __stcs(dst + 1, make_uint4(res[4], res[5], res[6], res[7]));
}

// w_hat = bf16_rne(float(q - zp) * scale): 8 weights per thread.
__global__ void rtn_dequant_kernel(const uint8_t* __restrict__ Wq,
                                   const uint16_t* __restrict__ scales,
                                   const uint8_t* __restrict__ zeros,
                                   const int32_t* __restrict__ g_idx, int N, int K, int G,
                                   uint16_t* __restrict__ out) {
  const int ng = K / G;
  const size_t per_row = static_cast<size_t>(K) / 8;
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= per_row * N) return;
  const int n = static_cast<int>(idx / per_row);
  const int k0 = static_cast<int>(idx % per_row) * 8;
  const unsigned long long nk = static_cast<unsigned long long>(N) * K;
  if (!in_bounds(static_cast<unsigned long long>(n) * K + k0 + 7, nk)) return;
  const uint32_t codes = *reinterpret_cast<const uint32_t*>(Wq + static_cast<size_t>(n) * (K / 2) + k0 / 2);
  uint32_t res[4];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int k = k0 + e;
    const int g = g_idx ? g_idx[k] : k / G;
    float v = 0.0f;
    if (g >= 0 && g < ng &&
        in_bounds(static_cast<unsigned long long>(n) * ng + g, static_cast<unsigned long long>(N) * ng)) {
      const float sf = __half2float(__ushort_as_half(scales[static_cast<size_t>(n) * ng + g]));
      const float z = static_cast<float>(zeros[static_cast<size_t>(n) * ng + g]);
      const float q = static_cast<float>((codes >> (4 * e)) & 0xFu);
      v = __fmul_rn(__fsub_rn(q, z), sf);
    } else {
      set_dev_error(W4_DEV_ERR_INPUT);
    }
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    if (e & 1)
      res[e >> 1] |= b << 16;
    else
      res[e >> 1] = b;
  }
  *reinterpret_cast<uint4*>(out + static_cast<size_t>(n) * K + k0) =
      make_uint4(res[0], res[1], res[2], res[3]);
}

// ---------------------------------------------------------------- AWQ factor
// "大模型量化选型：五种主流方案对比与实战" §4.1: the weights of input channel k
// are multiplied by s_k before quantization (the activations are divided by
// it at run time).  W_out[n, k] = fp32(W[n, k] * s_k); W_out may be W.
__global__ void awq_scale_weights_kernel(const float* W, const float* __restrict__ s, int N,
                                         int K, float* W_out) {
  const size_t total = static_cast<size_t>(N) * K;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    if (in_bounds(i % static_cast<size_t>(K), static_cast<unsigned long long>(K)))
      W_out[i] = __fmul_rn(W[i], s[i % static_cast<size_t>(K)]);
}

// The same product for K % 4 == 0 and 16-byte aligned W, s, W_out: CTAs walk
// whole rows (no index division), each thread 4 float4 of a row per trip,
// all 4 loads issued before the stores.  W_out may be W (each element is
// read and written by the same thread).
constexpr int kAwqThreads = 256;
__global__ void __launch_bounds__(kAwqThreads) awq_scale_weights_vec_kernel(
    const float4* W, const float4* __restrict__ s, int N, int K4, float4* W_out) {
  const unsigned long long total = static_cast<unsigned long long>(N) * K4;
  for (int n = blockIdx.x; n < N; n += gridDim.x) {
    const size_t row = static_cast<size_t>(n) * K4;
    for (int k0 = threadIdx.x; k0 < K4; k0 += 4 * kAwqThreads) {
      float4 v[4], f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + u * kAwqThreads;
        if (k < K4 && in_bounds(row + k, total)) {
          v[u] = __ldcs(W + row + k);
          f[u] = __ldg(s + k);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + u * kAwqThreads;
        if (k < K4 && in_bounds(row + k, total))
          __stcs(W_out + row + k,
                 make_float4(__fmul_rn(v[u].x, f[u].x), __fmul_rn(v[u].y, f[u].y),
                             __fmul_rn(v[u].z, f[u].z), __fmul_rn(v[u].w, f[u].w)));
      }
    }
  }
}

// ---------------------------------------------------------------- NF4
// "大模型量化选型" §6.1 (normal quantiles), §6.3 (blocks of 64),
// §6.2 (double quantization).  Levels: normal quantiles at equally spaced
// probabilities from 1 - (1/30 + 1/32)/2 toward 1/2 (8 positive, 7 negative,
// plus 0), normalised to [-1, 1]; midpoints are the fp32 average of
// neighbours.  Written as fp32 bit patterns.
__constant__ uint32_t kNf4LevelBits[16] = {
    0xbf800000u, 0xbf3239b1u, 0xbf066b2eu, 0xbeca329eu, 0xbe91a24bu, 0xbe3d353du,
    0xbdba7869u, 0x00000000u, 0x3da2fb01u, 0x3e24cadfu, 0x3e7c04dau, 0x3ead0336u,
    0x3ee1a4b5u, 0x3f1007a9u, 0x3f3913b0u, 0x3f800000u};
__constant__ uint32_t kNf4MidBits[15] = {
    0xbf591cd8u, 0xbf1c5270u, 0xbeeb847du, 0xbeadea74u, 0xbe703ceau, 0xbe0d38b9u,
    0xbd3a7869u, 0x3d22fb01u, 0x3df64860u, 0x3e5067dcu, 0x3e9582d2u, 0x3ec753f6u,
    0x3f006d02u, 0x3f248dacu, 0x3f5c89d8u};

static const uint32_t kNf4LevelBitsHost[16] = {
    0xbf800000u, 0xbf3239b1u, 0xbf066b2eu, 0xbeca329eu, 0xbe91a24bu, 0xbe3d353du,
    0xbdba7869u, 0x00000000u, 0x3da2fb01u, 0x3e24cadfu, 0x3e7c04dau, 0x3ead0336u,
    0x3ee1a4b5u, 0x3f1007a9u, 0x3f3913b0u, 0x3f800000u};

__device__ __forceinline__ uint32_t nf4_code(float v) {
  uint32_t q = 0;
#pragma unroll
  for (int i = 0; i < 15; ++i) q += (v > __uint_as_float(kNf4MidBits[i])) ? 1u : 0u;
  return q;
}

// FP4 in the same block-wise scheme ("大模型量化选型" §6.3 names NF4 and FP4
// as its two 4-bit types; "【推理与部署篇05】模型量化部署深度对比" §7.2 gives
// the 4-bit float layout [S:1][E:2][M:1]).  Code bit 3 = sign, bits 2..1 =
// exponent e, bit 0 = mantissa m; magnitude m/2 (e = 0) or 2^(e-1)(1 + m/2):
// 0, 0.5, 1, 1.5, 2, 3, 4, 6, divided by 6 so that the table spans [-1, 1].
__constant__ float kFp4Levels[16] = {
    0.0f,  0.5f / 6.0f,  1.0f / 6.0f,  1.5f / 6.0f,  2.0f / 6.0f,  3.0f / 6.0f,  4.0f / 6.0f,  1.0f,
    -0.0f, -0.5f / 6.0f, -1.0f / 6.0f, -1.5f / 6.0f, -2.0f / 6.0f, -3.0f / 6.0f, -4.0f / 6.0f, -1.0f};

static const float kFp4LevelsHost[16] = {
    0.0f,  0.5f / 6.0f,  1.0f / 6.0f,  1.5f / 6.0f,  2.0f / 6.0f,  3.0f / 6.0f,  4.0f / 6.0f,  1.0f,
    -0.0f, -0.5f / 6.0f, -1.0f / 6.0f, -1.5f / 6.0f, -2.0f / 6.0f, -3.0f / 6.0f, -4.0f / 6.0f, -1.0f};

// Which 16-entry level table a block-wise (NF4-layout) weight uses.
enum LevelTable : int { kTableNf4 = 0, kTableFp4 = 1 };

__device__ __forceinline__ float level_value(int table, int i) {
  return table == kTableFp4 ? kFp4Levels[i] : __uint_as_float(kNf4LevelBits[i]);
}

// Decision thresholds of a block-wise table in shared memory, padded with
// +inf to a power of two: NF4 the 15 midpoints t_i (code = #{i : v > t_i}),
// FP4 the 7 magnitude midpoints (magnitude code = #{i : |v| > t_i}); the
// count by binary search (the exact-division path of LevelBuckets::code).
template <int TABLE>
struct LevelSearch {
  static constexpr int kSteps = TABLE == kTableFp4 ? 3 : 4;  // 8 or 16 entries
  static constexpr int kEntries = 1 << kSteps;
  static __device__ __forceinline__ float threshold(int i) {
    if (TABLE == kTableFp4)
      return i < 7 ? __fmul_rn(__fadd_rn(kFp4Levels[i], kFp4Levels[i + 1]), 0.5f)
                   : __int_as_float(0x7f800000);
    return i < 15 ? __uint_as_float(kNf4MidBits[i]) : __int_as_float(0x7f800000);
  }
  // #{i : x > t_i}, branch-free over the sorted thresholds
  static __device__ __forceinline__ int count_below(const float* t, float x) {
    int q = 0;
#pragma unroll
    for (int step = kEntries / 2; step > 0; step >>= 1)
      if (t[q + step - 1] < x) q += step;
    return q;
  }
};

// The code of v = w / a (a > 0, r = RN(1/a)): from t = RN(w r) when t is
// further than |t| 2^-20 from the thresholds around it (then t, the exact
// quotient and RN(w / a) lie on the same side of every threshold: they are
// within |w/a| 2^-23 of each other), else from the IEEE division.  The
// decision uses a bucket table rather than a search over the thresholds: the
// range of x (NF4: [-1, 1], FP4: |x| in [0, 1]) cut into buckets 1/64 (NF4)
// or 1/128 (FP4) wide, bucket b = round(x S + O) taken from the low mantissa
// bits of one fused multiply-add with a 1.5 * 2^23 offset.  No bucket holds
// more than one threshold, and every threshold lies at least 7e-4 from a
// bucket edge (checked for both tables, far above the 2^-20 |x| margin), so
// #{i : x > t_i} = (thresholds below the bucket) + (x > the bucket's
// threshold), and the margin test needs only the bucket's threshold: the
// others are further from x than its bucket edges.  Entry b = {the bucket's
// threshold (+inf if none), the count below the bucket}; 256 entries so that
// any mantissa bits index inside.  An infinite or NaN t (a subnormal absmax
// overflows 1/a) fails the margin test and takes the IEEE division.
template <int TABLE>
struct LevelBuckets {
  static constexpr float kScale = TABLE == kTableFp4 ? 128.0f : 64.0f;
  static constexpr float kOffset = TABLE == kTableFp4 ? 0.0f : 64.0f;
  static constexpr int kUsed = 129;  // buckets 0..128 cover the range
  // thr: LevelSearch<TABLE>'s thresholds in shared memory (built first)
  static __device__ void build(float2* bk, const float* thr) {
    using LS = LevelSearch<TABLE>;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
      float tau = __int_as_float(0x7f800000);
      int below = LS::kEntries - 1;  // unused entries: +inf (no decision made here)
      if (b < kUsed) {
        const float lo = (static_cast<float>(b) - 0.5f - kOffset) / kScale;
        const float hi = (static_cast<float>(b) + 0.5f - kOffset) / kScale;
        below = 0;
        for (int i = 0; i < LS::kEntries; ++i) {
          const float t = thr[i];
          if (t < lo) ++below;
          else if (t < hi) tau = t;
        }
      }
      bk[b] = make_float2(tau, __int_as_float(below));
    }
  }
  static __device__ __forceinline__ uint32_t code(const float2* bk, const float* thr, float w,
                                                  float a, float r) {
    using LS = LevelSearch<TABLE>;
    const float x = __fmul_rn(w, r);
    const float ax = TABLE == kTableFp4 ? fabsf(x) : x;
    const float y = __fmaf_rn(ax, kScale, 12582912.0f + kOffset);
    const float2 e = bk[__float_as_uint(y) & 0xFFu];
    int q = __float_as_int(e.y) + (ax > e.x ? 1 : 0);
    const float m = __fmaf_rn(fabsf(x), 0x1p-20f, 0x1p-60f);
    float v = x;
    if (!(fabsf(__fsub_rn(ax, e.x)) > m)) {
      v = __fdiv_rn(w, a);
      q = LS::count_below(thr, TABLE == kTableFp4 ? fabsf(v) : v);
    }
    if (TABLE == kTableFp4) return (v < 0.0f && q != 0) ? (static_cast<uint32_t>(q) | 8u) : q;
    return static_cast<uint32_t>(q);
  }
};

// One CTA (kNf4QThreads threads) per run of dq_group consecutive 64-weight blocks.
// Codes: kNf4QLanes lanes per block, 64 / kNf4QLanes weights each (load u of
// lane j is float4 u kNf4QLanes + j of the block, so that every load
// instruction reads whole runs of 16 kNf4QLanes bytes), all of a lane's loads
// issued at once; the block absmax is a shuffle reduction over the block's
// lanes and the codes come from LevelBuckets.  Then
// the run's constants:
//   MEAN false  s2 = max(a) / 255 (1 if 0), c = clamp(rint(a / s2), 0, 255) (u8);
//   MEAN true   mean-offset: mu = fp32(fp64 sum of the run's a in block order / n),
//               d = a - mu, s2 = max|d| / 127 (1 if 0),
//               c = clamp(rint(d / s2), -127, 127) (int8), mean[run] = mu.
// TABLE selects the NF4 or the FP4 codes.  Shared memory: 2 KB of level
// buckets, then dq_group + 64 floats.
constexpr int kNf4QThreads = 512;  // threads per CTA (a multiple of 128)
constexpr int kNf4QCtasPerSm = 4;  // resident CTAs per SM (caps the registers)
constexpr int kNf4QLanes = 8;       // lanes per 64-weight block (4 or 8)
template <int TABLE, bool MEAN>
__global__ void __launch_bounds__(kNf4QThreads, kNf4QCtasPerSm) nf4_quantize_kernel(const float* __restrict__ W,
                                                            long long nblocks, int dq_group,
                                                            uint8_t* __restrict__ Wq,
                                                            uint8_t* __restrict__ absmax_q,
                                                            float* __restrict__ s2,
                                                            float* __restrict__ mean) {
  using LS = LevelSearch<TABLE>;
  using LB = LevelBuckets<TABLE>;
  extern __shared__ float sm_q4[];
  float2* bk = reinterpret_cast<float2*>(sm_q4);  // [256] level buckets
  float* a_s = sm_q4 + 512;       // [dq_group] block absmax, block order
  float* red = a_s + dq_group;    // [32] warp maxima, [32] the run's max, [33] its mean
  float* thr = red + 48;          // [16] decision thresholds
  const long long run0 = static_cast<long long>(blockIdx.x) * dq_group;
  const long long left = nblocks - run0;
  const int nrun = left < dq_group ? static_cast<int>(left) : dq_group;
  if (threadIdx.x < LS::kEntries) thr[threadIdx.x] = LS::threshold(threadIdx.x);
  __syncthreads();
  LB::build(bk, thr);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kL = kNf4QLanes;  // lanes per block
  constexpr int kF = 16 / kL;     // float4 loads per lane
  const int j = threadIdx.x % kL;
  const float4* src = reinterpret_cast<const float4*>(W);
  const unsigned long long n4 = static_cast<unsigned long long>(nblocks) * 16;
  for (int b0 = 0; b0 < nrun; b0 += kNf4QThreads / kL) {
    const int b = b0 + static_cast<int>(threadIdx.x) / kL;
    const bool valid = b < nrun;  // the same for a block's lanes
    const unsigned long long f0 = static_cast<unsigned long long>(run0 + b) * 16 + j;
    float4 v[kF];
#pragma unroll
    for (int u = 0; u < kF; ++u)
      v[u] = valid && in_bounds(f0 + kL * u, n4) ? __ldcs(src + f0 + kL * u)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    float a = 0.0f;
#pragma unroll
    for (int u = 0; u < kF; ++u)
      a = fmaxf(a, fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w))));
#pragma unroll
    for (int o = 1; o < kL; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (!valid) continue;
    if (j == 0) a_s[b] = a;
    const float r = a > 0.0f ? __frcp_rn(a) : 0.0f;
    const uint32_t zc = static_cast<uint32_t>(LS::count_below(thr, 0.0f));
#pragma unroll
    for (int u = 0; u < kF; ++u) {
      const float w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t codes = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        codes |= (a > 0.0f ? LB::code(bk, thr, w[e], a, r) : zc) << (4 * e);
      // float4 f0 + kL u holds weights 4 (f0 + kL u) .. + 3: code bytes 2 (f0 + kL u) ..
      if (in_bounds(f0 + kL * u, n4))
        reinterpret_cast<uint16_t*>(Wq)[f0 + kL * u] = static_cast<uint16_t>(codes);
    }
  }
  __syncthreads();

  // the run's constants
  float mu = 0.0f;
  if constexpr (MEAN) {
    if (threadIdx.x == 0) {
      double sum = 0.0;
      for (int i = 0; i < nrun; ++i) sum += static_cast<double>(a_s[i]);
      red[33] = static_cast<float>(sum / static_cast<double>(nrun));
    }
    __syncthreads();
    mu = red[33];
  }
  float key = 0.0f;
  for (int b = threadIdx.x; b < nrun; b += kNf4QThreads)
    key = fmaxf(key, MEAN ? fabsf(__fsub_rn(a_s[b], mu)) : a_s[b]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) key = fmaxf(key, __shfl_xor_sync(0xffffffffu, key, o));
  if (lane == 0) red[warp] = key;
  __syncthreads();
  if (warp == 0) {
    key = lane < kNf4QThreads / 32 ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) key = fmaxf(key, __shfl_xor_sync(0xffffffffu, key, o));
    if (lane == 0) red[32] = key;
  }
  __syncthreads();
  float sc = __fdiv_rn(red[32], MEAN ? 127.0f : 255.0f);
  if (sc == 0.0f) sc = 1.0f;
  if (threadIdx.x == 0) {
    s2[blockIdx.x] = sc;
    if constexpr (MEAN) mean[blockIdx.x] = mu;
  }
  for (int b = threadIdx.x; b < nrun; b += kNf4QThreads) {
    const float a = a_s[b];
    uint8_t byte;
    if constexpr (MEAN) {
      const float c = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(a, mu), sc)), -127.0f), 127.0f);
      byte = static_cast<uint8_t>(static_cast<int8_t>(c));
    } else {
      byte = static_cast<uint8_t>(fminf(fmaxf(rintf(__fdiv_rn(a, sc)), 0.0f), 255.0f));
    }
    if (in_bounds(static_cast<unsigned long long>(run0 + b), static_cast<unsigned long long>(nblocks)))
      absmax_q[run0 + b] = byte;
  }
}

// The reconstructed absmax of a block from its 8-bit code byte:
//   plain      a' = fp32(c * s2), c unsigned;
//   mean-offset a' = fp32(fp32(c * s2) + mu), c signed (int8).
template <bool MEAN>
__device__ __forceinline__ float absmax_from_code(uint32_t byte, float s2v, float mu) {
  if constexpr (MEAN)
    return __fadd_rn(__fmul_rn(static_cast<float>(static_cast<int8_t>(byte & 0xFFu)), s2v), mu);
  else
    return __fmul_rn(static_cast<float>(byte & 0xFFu), s2v);
}

// w_hat = bf16_rne(fp32(T[q] * a')), a' from the block's code byte (see
// absmax_from_code): 8 weights per thread.
template <bool MEAN>
__global__ void nf4_dequant_kernel(const uint8_t* __restrict__ Wq,
                                   const uint8_t* __restrict__ absmax_q,
                                   const float* __restrict__ s2, const float* __restrict__ mean,
                                   long long total8, int dq_group, int table,
                                   uint16_t* __restrict__ out) {
  __shared__ float T[16];
  if (threadIdx.x < 16) T[threadIdx.x] = level_value(table, threadIdx.x);
  __syncthreads();
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total8) return;
  const long long e0 = idx * 8;
  const long long b = e0 / 64;
  const long long run = b / dq_group;
  if (!in_bounds(e0 + 7, static_cast<unsigned long long>(total8) * 8)) return;
  const float a = absmax_from_code<MEAN>(absmax_q[b], s2[run], MEAN ? mean[run] : 0.0f);
  const uint32_t codes = *reinterpret_cast<const uint32_t*>(Wq + e0 / 2);
  uint32_t res[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float f0 = __fmul_rn(T[(codes >> (8 * j)) & 0xFu], a);
    const float f1 = __fmul_rn(T[(codes >> (8 * j + 4)) & 0xFu], a);
    const __nv_bfloat162 p = __floats2bfloat162_rn(f0, f1);
    res[j] = *reinterpret_cast<const uint32_t*>(&p);
  }
  *reinterpret_cast<uint4*>(out + e0) = make_uint4(res[0], res[1], res[2], res[3]);
}

}  // namespace w4
