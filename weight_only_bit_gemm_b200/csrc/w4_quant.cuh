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
      if (g < 0 || g >= ng) {
        code[e] = 0;
        continue;
      }
      RtnParam p;
      p.sf = sf_s[g];
      p.zp = zp_s[g];
      p.lo = SYM ? 1.0f : 0.0f;
      code[e] = rtn_code(row[k], p);
    }
    out[b] = static_cast<uint8_t>(code[0] | (code[1] << 4));
  }
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
  const uint32_t codes = *reinterpret_cast<const uint32_t*>(Wq + static_cast<size_t>(n) * (K / 2) + k0 / 2);
  uint32_t res[4];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int k = k0 + e;
    const int g = g_idx ? g_idx[k] : k / G;
    float v = 0.0f;
    if (g >= 0 && g < ng) {
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
    W_out[i] = __fmul_rn(W[i], s[i % static_cast<size_t>(K)]);
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

// Nearest magnitude among levels 0..7 (the lower one on a midpoint; the
// midpoints are the fp32 averages of neighbours), sign bit only when the
// magnitude is not zero.
struct Fp4Mids {
  float t[7];
  __device__ __forceinline__ Fp4Mids() {
#pragma unroll
    for (int i = 0; i < 7; ++i) t[i] = __fmul_rn(__fadd_rn(kFp4Levels[i], kFp4Levels[i + 1]), 0.5f);
  }
  __device__ __forceinline__ uint32_t code(float v) const {
    const float av = fabsf(v);
    uint32_t mag = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) mag += (av > t[i]) ? 1u : 0u;
    return (v < 0.0f && mag != 0u) ? (mag | 8u) : mag;
  }
};

// One thread per 64-block, one CTA per run of dq_group blocks
// (blockDim.x == dq_group).  Writes packed codes, absmax codes and s2.
// TABLE selects the NF4 or the FP4 codes; everything else is shared.
// MEAN selects the double quantization of the absmax constants:
//   false  s2 = max(a) / 255 (1 if 0), c = clamp(rint(a / s2), 0, 255) (u8);
//   true   mean-offset: mu = fp32(fp64 sum of the run's a in block order / n),
//          d = a - mu, s2 = max|d| / 127 (1 if 0),
//          c = clamp(rint(d / s2), -127, 127) (int8), mean[run] = mu.
// Shared memory: dq_group floats (MEAN: 2 dq_group + 1).
template <int TABLE, bool MEAN>
__global__ void nf4_quantize_kernel(const float* __restrict__ W, long long nblocks, int dq_group,
                                    uint8_t* __restrict__ Wq, uint8_t* __restrict__ absmax_q,
                                    float* __restrict__ s2, float* __restrict__ mean) {
  extern __shared__ float sm_a[];
  const long long run0 = static_cast<long long>(blockIdx.x) * dq_group;
  const long long b = run0 + threadIdx.x;
  const bool valid = b < nblocks;
  float w[64];
  float a = 0.0f;
  if (valid) {
    const float4* src = reinterpret_cast<const float4*>(W + b * 64);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float4 v = src[i];
      w[4 * i + 0] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
#pragma unroll
    for (int i = 0; i < 64; ++i) a = fmaxf(a, fabsf(w[i]));
  }
  float key = a;  // what the run's scale is taken from: a, or |a - mu|
  if constexpr (MEAN) {
    float* sm_blk = sm_a + dq_group;  // the run's constants, in block order
    sm_blk[threadIdx.x] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
      const long long left = nblocks - run0;
      const int n = left < dq_group ? static_cast<int>(left) : dq_group;
      double sum = 0.0;
      for (int i = 0; i < n; ++i) sum += static_cast<double>(sm_blk[i]);
      sm_blk[dq_group] = static_cast<float>(sum / static_cast<double>(n));
    }
    __syncthreads();
    key = valid ? fabsf(__fsub_rn(a, sm_blk[dq_group])) : 0.0f;
  }
  sm_a[threadIdx.x] = key;
  __syncthreads();
  for (int s = 1; s < blockDim.x; s <<= 1) {
    float other = 0.0f;
    if ((threadIdx.x % (2 * s)) == 0 && threadIdx.x + s < blockDim.x) other = sm_a[threadIdx.x + s];
    __syncthreads();
    if ((threadIdx.x % (2 * s)) == 0) sm_a[threadIdx.x] = fmaxf(sm_a[threadIdx.x], other);
    __syncthreads();
  }
  float sc = __fdiv_rn(sm_a[0], MEAN ? 127.0f : 255.0f);
  if (sc == 0.0f) sc = 1.0f;
  if (threadIdx.x == 0) {
    s2[blockIdx.x] = sc;
    if constexpr (MEAN) mean[blockIdx.x] = sm_a[2 * dq_group];
  }
  if (!valid) return;
  if constexpr (MEAN) {
    const float d = __fsub_rn(a, sm_a[2 * dq_group]);
    const float c = fminf(fmaxf(rintf(__fdiv_rn(d, sc)), -127.0f), 127.0f);
    absmax_q[b] = static_cast<uint8_t>(static_cast<int8_t>(c));
  } else {
    const float c = fminf(fmaxf(rintf(__fdiv_rn(a, sc)), 0.0f), 255.0f);
    absmax_q[b] = static_cast<uint8_t>(c);
  }
  uint32_t packed[8];
  const Fp4Mids fp4;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float v = (a > 0.0f) ? __fdiv_rn(w[8 * i + e], a) : 0.0f;
      word |= (TABLE == kTableFp4 ? fp4.code(v) : nf4_code(v)) << (4 * e);
    }
    packed[i] = word;
  }
  uint4* dst = reinterpret_cast<uint4*>(Wq + b * 32);
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
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
