// w4_int8.cuh -- LLM.int8 mixed decomposition (W8A8 with 16-bit outliers).
//
// "大模型量化选型：五种主流方案对比与实战" §2.1: vector-wise quantization (one
// scale per output feature of the weights) and mixed-precision decomposition
// (input channels whose activation exceeds the threshold, 6.0, in magnitude
// go through a 16-bit product, the others through INT8, and the two results
// are added); "【推理与部署篇05】模型量化部署深度对比" §6.1: llm_int8_threshold 6.0,
// no 16-bit copy of the weights.  Per call, three launches:
//   scan      one CTA per 32 input channels: flag[k] = |x[m,k]| > threshold
//             for some token m; the CTA's flagged channels in ascending
//             order in its own list region; per token the largest unflagged
//             |x| of the CTA's channels (a partial maximum);
//   quantize  s_x = max of the partial maxima / 127 per token, q_x =
//             clamp(rint(x / s_x), +-127), 0 on flagged channels; the first
//             CTA also concatenates the scan CTAs' lists into one ascending
//             list of outlier channels;
//   product   warp-level INT8 MMAs (m16n8k32, s32 accumulate) over
//             (16-row tile, K slice) work items, exact int32 partial sums
//             added atomically (exact, so the order does not matter); the
//             last work item of a row tile to finish (an arrival counter)
//             runs the epilogue y = acc s_x s_w + sum over flagged k of
//             x * bf16(q_w s_w) for the tile.
// The scan clears the row-tile counters and the quantization clears the
// accumulator, so the workspace's contents before the call do not matter.
#pragma once

#include <cuda_bf16.h>

#include "w4_ptx.cuh"

namespace w4 {

constexpr int kInt8Warps = 8;      // warps per product CTA
constexpr int kInt8MaxNB = 4;      // token blocks of 8 per pass over the weights
constexpr int kInt8ScanCh = 32;    // input channels per outlier-scan CTA
constexpr int kInt8EpiChunk = 8;   // outlier channels per step of the epilogue
constexpr int kInt8EpiDirectM = 4; // up to this many tokens the epilogue reads global memory
constexpr int kInt8StepsAhead = 2; // 64-channel weight steps loaded together per warp
constexpr int kInt8CtasPerSm = 3;  // resident product CTAs per SM (caps the registers)

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

// One CTA of min(M, 32) warps per kInt8ScanCh = 32 input channels: lane =
// channel, warp w of nw = the tokens m = w (mod nw), eight of them loaded at
// once (independent loads), so a long prefill batch is read in M / 256 round
// trips per thread, short K still gives many CTAs, and a short batch does
// not launch idle warps.  Flags: a ballot per warp,
// OR-ed over the warps in shared memory.  The per-token maximum of the
// unflagged |x| over the CTA's channels is one warp's maximum (shuffles), so
// each partial is written by exactly one lane.
__global__ void __launch_bounds__(1024) int8_scan_kernel(const uint16_t* __restrict__ X, int M,
                                                         int K, float threshold,
                                                         uint8_t* __restrict__ flag,
                                                         int32_t* __restrict__ list,
                                                         int32_t* __restrict__ cnt,
                                                         float* __restrict__ part,
                                                         unsigned int* __restrict__ counter,
                                                         int row_tiles) {
  __shared__ unsigned int warp_bits[32];
  grid_dep_launch();
  grid_dep_wait();  // X may come from the previous kernel
  const int c = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int nw = static_cast<int>(blockDim.x) >> 5;
  for (int i = c * blockDim.x + t; i < row_tiles; i += gridDim.x * blockDim.x) counter[i] = 0u;
  const int k = c * kInt8ScanCh + lane;
  const bool in = k < K;
  bool og = false;
  for (int m0 = w; m0 < M; m0 += nw * 8) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int m = m0 + nw * j;
      v[j] = in && m < M ? fabsf(bf16_bits_f32(X[static_cast<size_t>(m) * K + k])) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) og = og || v[j] > threshold;
  }
  const unsigned bits = __ballot_sync(0xffffffffu, og);
  if (lane == 0) warp_bits[w] = bits;
  __syncthreads();
  unsigned flagged = 0u;
  for (int i = 0; i < nw; ++i) flagged |= warp_bits[i];
  const bool o = (flagged >> lane) & 1u;
  // the CTA's flagged channels, ascending, in its list region
  if (w == 0) {
    if (in) flag[k] = o ? 1 : 0;
    if (o) {
      const int pos = __popc(flagged & ((1u << lane) - 1u));
      if (in_bounds(static_cast<unsigned>(c * kInt8ScanCh + pos),
                    static_cast<unsigned>(gridDim.x * kInt8ScanCh)))
        list[c * kInt8ScanCh + pos] = k;
    }
    if (lane == 0) cnt[c] = __popc(flagged);
  }
  // per token, the largest unflagged |x| among the CTA's channels
  for (int m0 = w; m0 < M; m0 += nw * 8) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int m = m0 + nw * j;
      v[j] = in && !o && m < M ? fabsf(bf16_bits_f32(X[static_cast<size_t>(m) * K + k])) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v[j] = fmaxf(v[j], __shfl_xor_sync(0xffffffffu, v[j], off));
    }
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (m0 + nw * j < M) part[static_cast<size_t>(c) * M + m0 + nw * j] = v[j];
    }
  }
}

// grid (M, ceil(K / 2048)), 256 threads x 8 channels: q_x of one token.
// s_x = max over the scan CTAs' partial maxima / 127 (1 if 0).  CTA (0, 0)
// also writes the ascending list of all outlier channels and its length.
__global__ void __launch_bounds__(256) int8_quantize_x_kernel(
    const uint16_t* __restrict__ X, const uint8_t* __restrict__ flag,
    const float* __restrict__ part, const int32_t* __restrict__ list,
    const int32_t* __restrict__ cnt, int nscan, int M, int K, int8_t* __restrict__ qx,
    float* __restrict__ sx, int32_t* __restrict__ olist, int32_t* __restrict__ ocount,
    int* __restrict__ acc, int N) {
  __shared__ float red[256];
  __shared__ int pre[257];
  grid_dep_launch();
  grid_dep_wait();
  const int m = blockIdx.x, t = threadIdx.x;
  // this token's row of the INT8 accumulator starts at zero
  for (int n = blockIdx.y * 256 + t; n < N; n += gridDim.y * 256) acc[static_cast<size_t>(m) * N + n] = 0;
  float a = 0.0f;
  for (int c = t; c < nscan; c += 256) a = fmaxf(a, part[static_cast<size_t>(c) * M + m]);
  red[t] = a;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (t < w) red[t] = fmaxf(red[t], red[t + w]);
    __syncthreads();
  }
  float s = __fdiv_rn(red[0], 127.0f);
  if (s == 0.0f) s = 1.0f;
  if (blockIdx.y == 0 && t == 0) sx[m] = s;
  const int k0 = blockIdx.y * 2048 + t * 8;
  if (k0 < K) {
    const uint4 xv = *reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + k0);
    const uint2 fv = *reinterpret_cast<const uint2*>(flag + k0);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
    uint32_t q[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = bf16_bits_f32(static_cast<uint16_t>(xw[e >> 1] >> (16 * (e & 1))));
      const uint32_t fl = ((e < 4 ? fv.x : fv.y) >> (8 * (e & 3))) & 0xFFu;
      const float qq = fl ? 0.0f : fminf(fmaxf(rintf(__fdiv_rn(x, s)), -127.0f), 127.0f);
      q[e >> 2] |= (static_cast<uint32_t>(static_cast<int32_t>(qq)) & 0xFFu) << (8 * (e & 3));
    }
    *reinterpret_cast<uint2*>(qx + static_cast<size_t>(m) * K + k0) = make_uint2(q[0], q[1]);
  }
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    // concatenate the scan CTAs' ascending lists: thread t takes scan CTAs
    // t per .. t per + per - 1, in order
    const int per = (nscan + 255) / 256;
    int n = 0;
    for (int i = 0; i < per; ++i) {
      const int cc = t * per + i;
      if (cc < nscan) n += cnt[cc];
    }
    pre[t + 1] = n;
    if (t == 0) pre[0] = 0;
    __syncthreads();
    for (int off = 1; off < 256; off <<= 1) {
      const int v = t + 1 - off >= 1 ? pre[t + 1 - off] : 0;
      __syncthreads();
      pre[t + 1] += v;
      __syncthreads();
    }
    int pos = pre[t];
    for (int i = 0; i < per; ++i) {
      const int cc = t * per + i;
      if (cc >= nscan) break;
      const int nc = cnt[cc];
      for (int j = 0; j < nc; ++j, ++pos)
        if (in_bounds(static_cast<unsigned>(pos), static_cast<unsigned>(K)) &&
            in_bounds(static_cast<unsigned>(j), static_cast<unsigned>(kInt8ScanCh)))
          olist[pos] = list[cc * kInt8ScanCh + j];
    }
    if (t == 0) *ocount = pre[256];
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

struct Int8Args {  // (acc and counter are cleared by the call's first two kernels)
  const int8_t* qw;        // [N, K]
  const int8_t* qx;        // [M, K]
  const float* sx;         // [M]
  const float* sw;         // [N]
  const uint16_t* X;       // bf16 [M, K] (outlier channels)
  const int32_t* olist;    // ascending outlier channels
  const int32_t* ocount;
  int* acc;                // [M, N] int32
  unsigned int* counter;   // [row tiles]
  uint16_t* Y;             // bf16 [M, N]
  int M, N, K, row_tiles, slices, steps;
};

// The epilogue of row tile rt, run by the last of its work items' warps.
__device__ __forceinline__ void int8_epilogue(const Int8Args& a, int rt, int lane) {
  // y[m][n] = acc s_x s_w + sum over outlier channels (ascending) of
  // x * bf16(q_w s_w), one fp32 fma per channel in ascending order.  Up to
  // kInt8EpiDirectM tokens (at most two outputs per lane) each output's chain
  // reads its operands from global memory (measured faster there).  Above,
  // lane l owns outputs l + 32 j (token idx / 16, row idx % 16 of the tile);
  // the outlier channels go kInt8EpiChunk at a time: the warp gathers their 16
  // rows' weights bf16(q_w s_w) and the M tokens' activations into its slice
  // of shared memory (independent loads spread over the lanes), then every
  // lane advances its outputs' fma chains over the chunk.  The slice is kept
  // small so that the L1 left beside it still holds the activation codes
  // every warp streams.
  if (a.M <= kInt8EpiDirectM) {
    // a few outputs per lane: each lane's output straight from global memory
    const int no = min(*a.ocount, a.K);
    for (int idx = lane; idx < 16 * a.M; idx += 32) {
      const int m = idx >> 4, n = rt * 16 + (idx & 15);
      if (n >= a.N) continue;
      const size_t o = static_cast<size_t>(m) * a.N + n;
      const float s = a.sw[n];
      float y = __fmul_rn(__fmul_rn(static_cast<float>(__ldcg(a.acc + o)), a.sx[m]), s);
      for (int i = 0; i < no; ++i) {
        const int k = a.olist[i];
        if (!in_bounds(static_cast<unsigned int>(k), static_cast<unsigned int>(a.K))) continue;
        const float w16 = __bfloat162float(__float2bfloat16_rn(
            __fmul_rn(static_cast<float>(a.qw[static_cast<size_t>(n) * a.K + k]), s)));
        y = fmaf(bf16_bits_f32(a.X[static_cast<size_t>(m) * a.K + k]), w16, y);
      }
      a.Y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
    }
    return;
  }
  extern __shared__ float i8_epi[];
  const int per = 16 + a.M;  // rows, then tokens
  float* wsm = i8_epi + (threadIdx.x >> 5) * (per * kInt8EpiChunk + kInt8EpiChunk);
  float* xsm = wsm + 16 * kInt8EpiChunk;
  float* okm = wsm + per * kInt8EpiChunk;  // 1: the channel is inside K
  const int no = min(*a.ocount, a.K);
  const int nout = 16 * a.M;  // at most 512: 16 outputs per lane
  float y[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int idx = lane + 32 * j;
    y[j] = 0.0f;
    if (idx < nout) {
      const int m = idx >> 4, n = rt * 16 + (idx & 15);
      if (n < a.N)
        y[j] = __fmul_rn(__fmul_rn(static_cast<float>(__ldcg(a.acc + static_cast<size_t>(m) * a.N + n)),
                                   a.sx[m]),
                         a.sw[n]);
    }
  }
  static_assert(32 % kInt8EpiChunk == 0, "a lane keeps one channel of the chunk");
  constexpr int kMaxV = (16 + 32) * kInt8EpiChunk / 32;  // values a lane gathers at most
  for (int c0 = 0; c0 < no; c0 += kInt8EpiChunk) {
    // lane l gathers channel l % chunk of the chunk for rows / tokens
    // l / chunk + (32 / chunk) t: the channel index once, then all its loads
    // at once
    const int ch = lane % kInt8EpiChunk;
    int k = 0;
    bool ok = false;
    if (c0 + ch < no) {
      k = a.olist[c0 + ch];
      ok = in_bounds(static_cast<unsigned int>(k), static_cast<unsigned int>(a.K));
    }
    if (lane < kInt8EpiChunk) okm[lane] = ok ? 1.0f : 0.0f;
    float vals[kMaxV];
#pragma unroll
    for (int t = 0; t < kMaxV; ++t) {
      const int v = lane + 32 * t, rr = v / kInt8EpiChunk;
      vals[t] = 0.0f;
      if (ok && rr < per) {
        if (rr < 16) {
          const int n = rt * 16 + rr;
          if (n < a.N)
            vals[t] = __bfloat162float(__float2bfloat16_rn(
                __fmul_rn(static_cast<float>(a.qw[static_cast<size_t>(n) * a.K + k]), a.sw[n])));
        } else {
          vals[t] = bf16_bits_f32(a.X[static_cast<size_t>(rr - 16) * a.K + k]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kMaxV; ++t) {
      const int v = lane + 32 * t;
      if (v < per * kInt8EpiChunk) wsm[v] = vals[t];  // rows, then tokens (xsm)
    }
    __syncwarp();
    const int cn = min(kInt8EpiChunk, no - c0);
    for (int ii = 0; ii < cn; ++ii) {
      if (okm[ii] == 0.0f) continue;  // a channel outside K (bounds-checked build)
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int idx = lane + 32 * j;
        if (idx < nout)
          y[j] = fmaf(xsm[(idx >> 4) * kInt8EpiChunk + ii], wsm[(idx & 15) * kInt8EpiChunk + ii], y[j]);
      }
    }
    __syncwarp();
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int idx = lane + 32 * j;
    if (idx < nout) {
      const int m = idx >> 4, n = rt * 16 + (idx & 15);
      if (n < a.N) a.Y[static_cast<size_t>(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y[j]));
    }
  }
}

// acc[m][n] += sum over the warp's K slice of q_x[m][k] q_w[n][k].
// Work item = (16-row tile, slice of `steps` 64-channel steps); lane (g, u)
// = (lane / 4, lane % 4) loads 16 consecutive bytes of weight rows g and
// g + 8 and of token row g at channel k0 + 16u: bytes 0-3 / 4-7 feed the
// first MMA's k-slots 4u.. / 16 + 4u.., bytes 8-15 the second MMA's.  A and
// B use the same channel-to-slot map, so the exact sum is the plain dot
// product.  Tokens in passes of up to kInt8MaxNB blocks of 8.  The last of a
// row tile's work items to finish (counted after a release fence on the
// tile's counter) applies the epilogue to the tile's outputs.
__global__ void __launch_bounds__(kInt8Warps * 32, kInt8CtasPerSm) int8_product_kernel(const Int8Args a) {
  grid_dep_launch();
  const int lane = threadIdx.x & 31, g = lane >> 2, u = lane & 3;
  const long long item = static_cast<long long>(blockIdx.x) * kInt8Warps + (threadIdx.x >> 5);
  if (item >= static_cast<long long>(a.row_tiles) * a.slices) {
    grid_dep_wait();
    return;
  }
  const int rt = static_cast<int>(item % a.row_tiles);
  const int sl = static_cast<int>(item / a.row_tiles);
  const int r0 = rt * 16 + g, r1 = r0 + 8;
  const int kbeg = sl * a.steps * 64;
  const int kend = min(a.K, kbeg + a.steps * 64);
  const int NB = (a.M + 7) / 8;
  // weights of kInt8StepsAhead 64-channel steps requested together (the
  // first batch before the launch dependency: weights do not depend on the
  // previous kernels), so that enough bytes are in flight to cover the HBM
  // latency with one wave of warps
  constexpr int kU = kInt8StepsAhead;
  uint4 wa[kU], wb[kU];
  auto load_batch = [&](int k0) {
#pragma unroll
    for (int st = 0; st < kU; ++st) {
      const int kk = k0 + 64 * st + 16 * u;
      wa[st] = make_uint4(0u, 0u, 0u, 0u);
      wb[st] = make_uint4(0u, 0u, 0u, 0u);
      if (k0 + 64 * st < kend &&
          in_bounds(static_cast<unsigned int>(kk + 15), static_cast<unsigned int>(a.K))) {
        if (r0 < a.N) wa[st] = *reinterpret_cast<const uint4*>(a.qw + static_cast<size_t>(r0) * a.K + kk);
        if (r1 < a.N) wb[st] = *reinterpret_cast<const uint4*>(a.qw + static_cast<size_t>(r1) * a.K + kk);
      }
    }
  };
  load_batch(kbeg);
  grid_dep_wait();  // q_x, s_x and the outlier list come from the previous kernels
  for (int tb0 = 0; tb0 < NB; tb0 += kInt8MaxNB) {
    int d[kInt8MaxNB][4] = {};
    for (int k0 = kbeg; k0 < kend; k0 += 64 * kU) {
      if (k0 != kbeg || tb0 != 0) load_batch(k0);
#pragma unroll
      for (int st = 0; st < kU; ++st) {
        if (k0 + 64 * st >= kend) break;  // the same for the whole warp
        const int kk = k0 + 64 * st + 16 * u;
#pragma unroll
        for (int j = 0; j < kInt8MaxNB; ++j) {
          const int tok = (tb0 + j) * 8 + g;
          if (tb0 + j >= NB) break;
          uint4 xv = make_uint4(0u, 0u, 0u, 0u);
          if (tok < a.M && in_bounds(static_cast<unsigned int>(kk + 15), static_cast<unsigned int>(a.K)))
            xv = *reinterpret_cast<const uint4*>(a.qx + static_cast<size_t>(tok) * a.K + kk);
          mma_s8_16832(d[j], wa[st].x, wb[st].x, wa[st].y, wb[st].y, xv.x, xv.y);
          mma_s8_16832(d[j], wa[st].z, wb[st].z, wa[st].w, wb[st].w, xv.z, xv.w);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kInt8MaxNB; ++j) {
      if (tb0 + j >= NB) break;
      const int t0 = (tb0 + j) * 8 + 2 * u;
      // d0, d1: row r0, tokens t0, t0 + 1; d2, d3: row r1
      if (r0 < a.N && t0 < a.M) atomicAdd(&a.acc[static_cast<size_t>(t0) * a.N + r0], d[j][0]);
      if (r0 < a.N && t0 + 1 < a.M) atomicAdd(&a.acc[static_cast<size_t>(t0 + 1) * a.N + r0], d[j][1]);
      if (r1 < a.N && t0 < a.M) atomicAdd(&a.acc[static_cast<size_t>(t0) * a.N + r1], d[j][2]);
      if (r1 < a.N && t0 + 1 < a.M) atomicAdd(&a.acc[static_cast<size_t>(t0 + 1) * a.N + r1], d[j][3]);
    }
  }
  // arrival on the row tile's counter; the last item runs the epilogue.  The
  // warp barrier orders every lane's atomics before lane 0's release (the
  // arrival) and, on the last item, lane 0's acquire before every lane's
  // reads of the sums.
  __syncwarp();
  unsigned prev = 0;
  if (lane == 0 && in_bounds(static_cast<unsigned int>(rt), static_cast<unsigned int>(a.row_tiles)))
    prev = atom_add_acq_rel_gpu(a.counter + rt, 1u);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  __syncwarp();
  if (prev != static_cast<unsigned>(a.slices - 1)) return;
  int8_epilogue(a, rt, lane);
}

}  // namespace w4
