// w4_gptq.cuh -- GPTQ error compensation at quantization time.
//
// "【推理与部署篇05】模型量化部署深度对比：GPTQ、AWQ、GGUF与FP8实战指南" §3.1: per
// layer, H = 2 X X^T from calibration activations; the columns are quantized
// one at a time and each column's error is spread over the columns not yet
// quantized through the inverse Hessian.  "大模型量化选型：五种主流方案对比与实战"
// §3: it is the Optimal Brain Surgeon update; the Hessian gets a small
// damping (percdamp 0.01) on its diagonal; §3.2: desc_act orders the columns
// by activation size.
//
// Device formulation.  With Hi = (damped H)^-1 and U its upper Cholesky
// factor (Hi = U^T U), eliminating column j from the inverse Hessian of the
// remaining columns leaves U's later rows unchanged, and the update of a
// remaining column k by column j's error e = w_j - dq(w_j) is
//   w_k -= e * Hi'_jk / Hi'_jj = (e / U_jj) * U_jk,
// so one factorization replaces the K eliminations.  U is obtained without
// forming Hi: for the reversal J (J_ij = [i + j = K - 1]), the lower
// Cholesky factor L' of J H J gives H = (J L' J)(J L' J)^T with J L' J upper,
// hence U = (J L' J)^-1 = J L'^-1 J.  Kernels:
//   prepare   diagonal (a never-activated channel gets H_kk = 1 and w_k = 0),
//             act-order permutation (stable, decreasing H_kk), damping
//             lambda = damp * mean(diag H), A = J P^T H P J + lambda I (fp64);
//   factor    blocked lower Cholesky of A (32 x 32 tiles: diagonal factor,
//             panel solve, trailing update), then the inverse T = L'^-1
//             (diagonal tiles inverted in parallel, then the off-diagonal
//             blocks by doubling: log2(K / 32) levels of two tile GEMMs), then
//             U = J T J in fp32;
//   quantize  lazy blocks of 128 columns: one thread per weight row applies
//             the in-block updates column by column in shared memory (and
//             decides codes, group scales and zero points there); a tiled
//             fp32 GEMM then applies the block's errors to every later column.
#pragma once

#include <cuda_bf16.h>

#include "w4_quant.cuh"

namespace w4 {

constexpr int kGptqB = 128;      // columns per lazy block
constexpr int kGptqRows = 128;   // weight rows (threads) per quantize CTA
constexpr int kChol = 32;        // factorization tile
constexpr size_t kGptqBlockSmem =
    static_cast<size_t>(kGptqB) * kGptqB * 4 + static_cast<size_t>(kGptqRows) * (kGptqB + 1) * 4;

// ------------------------------------------------------------------ H = 2 X^T X
// 64 x 64 output tiles (lower tiles only, mirrored), 256 threads x 4 x 4
// outputs, 16 calibration rows per shared-memory slice; fp32 accumulation.
__global__ void __launch_bounds__(256) gptq_hessian_kernel(const uint16_t* __restrict__ X, int n,
                                                            int K, float* __restrict__ H) {
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (bj > bi) return;
  __shared__ float As[16][64], Bs[16][64];
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  float acc[4][4] = {};
  for (int s0 = 0; s0 < n; s0 += 16) {
    for (int e = t; e < 16 * 64; e += 256) {
      const int r = e >> 6, c = e & 63, s = s0 + r;
      const int ci = bi * 64 + c, cj = bj * 64 + c;
      As[r][c] = (s < n && ci < K) ? __uint_as_float(static_cast<uint32_t>(X[static_cast<size_t>(s) * K + ci]) << 16) : 0.0f;
      Bs[r][c] = (s < n && cj < K) ? __uint_as_float(static_cast<uint32_t>(X[static_cast<size_t>(s) * K + cj]) << 16) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[r][ty * 4 + i];
        b[i] = Bs[r][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = bi * 64 + ty * 4 + i, c = bj * 64 + tx * 4 + j;
      if (r < K && c < K) {
        const float v = 2.0f * acc[i][j];
        H[static_cast<size_t>(r) * K + c] = v;
        H[static_cast<size_t>(c) * K + r] = v;
      }
    }
}

// ------------------------------------------------------------------ prepare
// d[k] = H_kk in fp64, with 1 for a channel whose H_kk is 0 (dead[k] = 1).
// A diagonal that is negative or not finite is not a Hessian: it is reported
// (device error word) and replaced by 1, so that the order below stays a
// permutation.
__global__ void gptq_diag_kernel(const float* __restrict__ H, int K, double* __restrict__ d,
                                 uint8_t* __restrict__ dead) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  float h = H[static_cast<size_t>(k) * K + k];
  if (!(h >= 0.0f) || isinf(h)) {
    set_dev_error(W4_DEV_ERR_INPUT);
    h = 1.0f;
  }
  dead[k] = h == 0.0f ? 1 : 0;
  d[k] = h == 0.0f ? 1.0 : static_cast<double>(h);
}

// Processing order: perm[position] = channel, pos[channel] = position.  With
// act-order the position of channel i is the number of channels with a larger
// d, plus those with an equal d and a smaller index (a stable sort).
__global__ void gptq_order_kernel(const double* __restrict__ d, int K, int act,
                                  int32_t* __restrict__ perm, int32_t* __restrict__ pos) {
  __shared__ double tile[256];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const double di = i < K ? d[i] : 0.0;
  int rank = 0;
  if (act) {
    for (int base = 0; base < K; base += 256) {
      const int j = base + threadIdx.x;
      tile[threadIdx.x] = j < K ? d[j] : 0.0;
      __syncthreads();
      const int lim = min(256, K - base);
      for (int e = 0; e < lim; ++e) {
        const double dj = tile[e];
        rank += (dj > di || (dj == di && base + e < i)) ? 1 : 0;
      }
      __syncthreads();
    }
  } else {
    rank = i;
  }
  if (i < K) {
    perm[rank] = i;
    pos[i] = rank;
  }
}

// lambda = damp * mean(d): one CTA, fixed summation order.
__global__ void gptq_damp_kernel(const double* __restrict__ d, int K, double damp,
                                 double* __restrict__ lambda) {
  __shared__ double part[256];
  double s = 0.0;
  for (int k = threadIdx.x; k < K; k += 256) s += d[k];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *lambda = damp * (part[0] / static_cast<double>(K));
}

// A[i][j] = H[p(i)][p(j)] (lower triangle), p(i) = perm[K - 1 - i]; the
// diagonal takes d (dead channels 1) plus lambda.
__global__ void gptq_build_kernel(const float* __restrict__ H, const double* __restrict__ d,
                                  const int32_t* __restrict__ perm,
                                  const double* __restrict__ lambda, int K,
                                  double* __restrict__ A) {
  const int j = blockIdx.x * 32 + (threadIdx.x & 31);
  const int i = blockIdx.y * 8 + (threadIdx.x >> 5);
  if (i >= K || j > i) return;
  const int pi = perm[K - 1 - i], pj = perm[K - 1 - j];
  A[static_cast<size_t>(i) * K + j] =
      i == j ? d[pi] + *lambda : static_cast<double>(H[static_cast<size_t>(pi) * K + pj]);
}

// Q[n][j] = W[n][perm[j]] (0 for a dead channel), fp32, processing order.
__global__ void gptq_gather_w_kernel(const float* __restrict__ W, const int32_t* __restrict__ perm,
                                     const uint8_t* __restrict__ dead, int N, int K,
                                     float* __restrict__ Q) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<size_t>(N) * K) return;
  const size_t n = idx / K;
  const int j = static_cast<int>(idx - n * K);
  const int c = perm[j];
  Q[idx] = dead[c] ? 0.0f : W[n * K + c];
}

// ------------------------------------------------------------------ factor
// Diagonal tile jb of the lower Cholesky factor, in place (32 x 32 threads).
// A non-positive pivot (H not positive definite) sets the device error word
// and continues with 1 so that nothing downstream reads a NaN.
__global__ void __launch_bounds__(1024) chol_diag_kernel(double* __restrict__ A, int K, int jb) {
  __shared__ double a[kChol][kChol + 1];
  const int r = threadIdx.x >> 5, c = threadIdx.x & 31;
  const size_t o = static_cast<size_t>(jb) * kChol;
  a[r][c] = c <= r ? A[(o + r) * K + o + c] : 0.0;
  for (int k = 0; k < kChol; ++k) {
    __syncthreads();
    if (r == k && c == k) {
      double v = a[k][k];
      if (!(v > 0.0)) {
        set_dev_error(W4_DEV_ERR_INPUT);
        v = 1.0;
      }
      a[k][k] = sqrt(v);
    }
    __syncthreads();
    if (c == k && r > k) a[r][k] /= a[k][k];
    __syncthreads();
    if (r > k && c > k && c <= r) a[r][c] -= a[r][k] * a[c][k];
  }
  __syncthreads();
  if (c <= r) A[(o + r) * K + o + c] = a[r][c];
}

// Panel: A[ib][jb] <- A[ib][jb] L[jb][jb]^-T for every tile row ib > jb.
// One thread per row of the tile, forward substitution along the row.
__global__ void __launch_bounds__(kChol) chol_panel_kernel(double* __restrict__ A, int K, int jb) {
  __shared__ double L[kChol][kChol + 1], Xs[kChol][kChol + 1];
  const int ib = jb + 1 + blockIdx.x;
  const int r = threadIdx.x;
  const size_t oj = static_cast<size_t>(jb) * kChol, oi = static_cast<size_t>(ib) * kChol;
  for (int c = 0; c < kChol; ++c) {
    L[r][c] = c <= r ? A[(oj + r) * K + oj + c] : 0.0;
    Xs[r][c] = A[(oi + r) * K + oj + c];
  }
  __syncthreads();
  for (int k = 0; k < kChol; ++k) {
    double x = Xs[r][k];
    for (int m = 0; m < k; ++m) x -= Xs[r][m] * L[k][m];
    Xs[r][k] = x / L[k][k];
  }
  for (int c = 0; c < kChol; ++c) A[(oi + r) * K + oj + c] = Xs[r][c];
}

// Trailing update: A[ib][kb] -= A[ib][jb] A[kb][jb]^T for jb < kb <= ib.
__global__ void __launch_bounds__(1024) chol_update_kernel(double* __restrict__ A, int K, int jb) {
  const int kb = jb + 1 + blockIdx.x, ib = jb + 1 + blockIdx.y;
  if (kb > ib) return;
  __shared__ double P[kChol][kChol + 1], Qt[kChol][kChol + 1];
  const int r = threadIdx.x >> 5, c = threadIdx.x & 31;
  const size_t oj = static_cast<size_t>(jb) * kChol, oi = static_cast<size_t>(ib) * kChol,
               ok = static_cast<size_t>(kb) * kChol;
  P[r][c] = A[(oi + r) * K + oj + c];
  Qt[r][c] = A[(ok + r) * K + oj + c];
  __syncthreads();
  if (ib == kb && c > r) return;
  double s = 0.0;
#pragma unroll 8
  for (int m = 0; m < kChol; ++m) s += P[r][m] * Qt[c][m];
  A[(oi + r) * K + ok + c] -= s;
}

// T[ib][ib] = L[ib][ib]^-1 for every diagonal tile; thread c computes column c
// by forward substitution.  The strictly upper part of each tile is zeroed.
__global__ void __launch_bounds__(kChol) trinv_diag_kernel(const double* __restrict__ L, int K,
                                                           double* __restrict__ T) {
  __shared__ double Ld[kChol][kChol + 1], X[kChol][kChol + 1];
  const int ib = blockIdx.x, c = threadIdx.x;
  const size_t o = static_cast<size_t>(ib) * kChol;
  for (int r = 0; r < kChol; ++r) Ld[r][c] = c <= r ? L[(o + r) * K + o + c] : 0.0;
  __syncthreads();
  for (int r = 0; r < kChol; ++r) {
    double s = r == c ? 1.0 : 0.0;
    if (r >= c) {
      for (int m = c; m < r; ++m) s -= Ld[r][m] * X[m][c];
      s /= Ld[r][r];
    } else {
      s = 0.0;
    }
    X[r][c] = s;
  }
  for (int r = 0; r < kChol; ++r) T[(o + r) * K + o + c] = X[r][c];
}

// The off-diagonal tiles of T = L^-1 by doubling.  At level s (in tiles),
// pair b joins the first block F = [2bs, 2bs + s) and the second block
// S = [2bs + s, min(2bs + 2s, nb)), whose inverses are complete; then
//   T[S][F] = -T[S][S] L[S][F] T[F][F],
// in two tile-GEMM launches over every pair of the level (grid: tile column
// j < s, tile row i < |S|, pair b).  P = L[S][F] T[F][F] goes to scratch, at
// tile (b s + i) s + j (only the last pair can have |S| < s).
__global__ void __launch_bounds__(1024) trinv_level_p_kernel(const double* __restrict__ L,
                                                             const double* __restrict__ T, int K,
                                                             int nb, int s,
                                                             double* __restrict__ P) {
  const int j = blockIdx.x, i = blockIdx.y, b = blockIdx.z;
  const int F0 = 2 * b * s, S0 = F0 + s;
  if (i >= min(s, nb - S0)) return;
  __shared__ double Lt[kChol][kChol + 1], Tt[kChol][kChol + 1];
  const int r = threadIdx.x >> 5, c = threadIdx.x & 31;
  const size_t oi = static_cast<size_t>(S0 + i) * kChol, oj = static_cast<size_t>(F0 + j) * kChol;
  double acc = 0.0;
  for (int k = j; k < s; ++k) {  // T[F][F] is lower triangular in tiles
    const size_t ok = static_cast<size_t>(F0 + k) * kChol;
    __syncthreads();
    Lt[r][c] = L[(oi + r) * K + ok + c];
    Tt[r][c] = T[(ok + r) * K + oj + c];
    __syncthreads();
#pragma unroll 8
    for (int m = 0; m < kChol; ++m) acc += Lt[r][m] * Tt[m][c];
  }
  P[((static_cast<size_t>(b) * s + i) * s + j) * (kChol * kChol) + r * kChol + c] = acc;
}

__global__ void __launch_bounds__(1024) trinv_level_t_kernel(const double* __restrict__ P, int K,
                                                             int nb, int s,
                                                             double* __restrict__ T) {
  const int j = blockIdx.x, i = blockIdx.y, b = blockIdx.z;
  const int F0 = 2 * b * s, S0 = F0 + s;
  if (i >= min(s, nb - S0)) return;
  __shared__ double At[kChol][kChol + 1], Pt[kChol][kChol + 1];
  const int r = threadIdx.x >> 5, c = threadIdx.x & 31;
  const size_t oi = static_cast<size_t>(S0 + i) * kChol;
  double acc = 0.0;
  for (int k = 0; k <= i; ++k) {  // T[S][S] is lower triangular in tiles
    const size_t ok = static_cast<size_t>(S0 + k) * kChol;
    __syncthreads();
    At[r][c] = T[(oi + r) * K + ok + c];
    Pt[r][c] = P[((static_cast<size_t>(b) * s + k) * s + j) * (kChol * kChol) + r * kChol + c];
    __syncthreads();
#pragma unroll 8
    for (int m = 0; m < kChol; ++m) acc -= At[r][m] * Pt[m][c];
  }
  T[(oi + r) * K + static_cast<size_t>(F0 + j) * kChol + c] = acc;
}

// U[a][b] = T[K-1-a][K-1-b] for b >= a (fp32): the upper Cholesky factor of
// the inverse of the damped, ordered Hessian.
__global__ void gptq_u_kernel(const double* __restrict__ T, int K, float* __restrict__ U) {
  const int b = blockIdx.x * 32 + (threadIdx.x & 31);
  const int a = blockIdx.y * 8 + (threadIdx.x >> 5);
  if (a >= K || b >= K || b < a) return;
  U[static_cast<size_t>(a) * K + b] =
      static_cast<float>(T[static_cast<size_t>(K - 1 - a) * K + (K - 1 - b)]);
}

// ------------------------------------------------------------------ quantize
// Columns j0 .. j0 + bw - 1 (bw <= kGptqB, a multiple of G; j0 a multiple of
// G).  Thread = weight row n; its block row lives in shared memory.  Per
// column: at a group start the RTN scale and zero point of the group's
// current (compensated) weights; the code; the error e = (w - dq) / U_jj;
// the in-block update of the later columns.  e goes to Et[c][n] for the
// trailing update, the code to codes_t[j][n] (processing order).
__global__ void __launch_bounds__(kGptqRows) gptq_block_kernel(
    const float* __restrict__ Q, const float* __restrict__ U, int N, int K, int G, int j0, int bw,
    float* __restrict__ Et, uint8_t* __restrict__ codes_t, uint16_t* __restrict__ scales,
    uint8_t* __restrict__ zeros) {
  extern __shared__ float sm_g[];
  float* Ub = sm_g;                                   // [bw][kGptqB]
  float* Qb = sm_g + kGptqB * kGptqB;                 // [kGptqRows][kGptqB + 1]
  const int t = threadIdx.x;
  const int n0 = blockIdx.x * kGptqRows;
  const unsigned long long kk = static_cast<unsigned long long>(K) * K;
  for (int e = t; e < bw * bw; e += kGptqRows) {
    const int a = e / bw, b = e - a * bw;
    const unsigned long long ui = static_cast<unsigned long long>(j0 + a) * K + j0 + b;
    Ub[a * kGptqB + b] = b >= a && in_bounds(ui, kk) ? U[ui] : 0.0f;
  }
  for (int e = t; e < kGptqRows * bw; e += kGptqRows) {
    const int r = e / bw, c = e - r * bw;
    const int n = n0 + r;
    const unsigned long long qi = static_cast<unsigned long long>(n) * K + j0 + c;
    Qb[r * (kGptqB + 1) + c] =
        n < N && in_bounds(qi, static_cast<unsigned long long>(N) * K) ? Q[qi] : 0.0f;
  }
  __syncthreads();
  const int n = n0 + t;
  const bool live = n < N;
  float* qr = Qb + t * (kGptqB + 1);
  const int ng = K / G;
  RtnParam p{};
  for (int c = 0; c < bw; ++c) {
    const int j = j0 + c;
    if (j % G == 0) {
      float mx = 0.0f, nx = 0.0f;
      for (int e = 0; e < G; ++e) {
        const float w = qr[c + e];
        mx = fmaxf(mx, w);
        nx = fmaxf(nx, -w);
      }
      p = rtn_param(mx, nx);
      if (live) {
        scales[static_cast<size_t>(n) * ng + j / G] = p.s16;
        zeros[static_cast<size_t>(n) * ng + j / G] = static_cast<uint8_t>(p.zp);
      }
    }
    const float w = qr[c];
    const uint32_t q = rtn_code(w, p);
    const float dq = __fmul_rn(__fsub_rn(static_cast<float>(q), p.zp), p.sf);  // exact
    const float e1 = __fdiv_rn(__fsub_rn(w, dq), Ub[c * kGptqB + c]);
    for (int k = c + 1; k < bw; ++k) qr[k] = fmaf(-e1, Ub[c * kGptqB + k], qr[k]);
    if (live) {
      Et[static_cast<size_t>(c) * N + n] = e1;
      codes_t[static_cast<size_t>(j) * N + n] = static_cast<uint8_t>(q);
    }
  }
}

// Trailing update after a block: Q[n][m] -= sum_{c < bw} Et[c][n] U[j0 + c][m]
// for every column m >= j0 + bw.  64 x 64 output tiles, 256 threads x 4 x 4,
// 16-deep slices of the block's errors.
__global__ void __launch_bounds__(256) gptq_trailing_kernel(float* __restrict__ Q,
                                                            const float* __restrict__ U,
                                                            const float* __restrict__ Et, int N,
                                                            int K, int j0, int bw) {
  __shared__ float Es[16][64], Us[16][64];
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  const int first = j0 + bw;
  const int m0 = first + blockIdx.x * 64, nb0 = blockIdx.y * 64;
  float acc[4][4] = {};
  for (int c0 = 0; c0 < bw; c0 += 16) {
    for (int e = t; e < 16 * 64; e += 256) {
      const int r = e >> 6, x = e & 63;
      Es[r][x] = nb0 + x < N ? Et[static_cast<size_t>(c0 + r) * N + nb0 + x] : 0.0f;
      Us[r][x] = m0 + x < K ? U[static_cast<size_t>(j0 + c0 + r) * K + m0 + x] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = Es[r][ty * 4 + i];
        b[i] = Us[r][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = nb0 + ty * 4 + i, m = m0 + tx * 4 + j;
      if (n < N && m < K) Q[static_cast<size_t>(n) * K + m] -= acc[i][j];
    }
}

// Wq[n][b] = code(2b) | code(2b + 1) << 4 in channel order, from the codes
// in processing order (codes_t[pos[k]][n]); threads run along n.
__global__ void gptq_pack_kernel(const uint8_t* __restrict__ codes_t,
                                 const int32_t* __restrict__ pos, int N, int K,
                                 uint8_t* __restrict__ Wq) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t half = static_cast<size_t>(K) / 2;
  if (idx >= half * N) return;
  const size_t b = idx / N;
  const size_t n = idx - b * N;
  const int p0 = pos[2 * b], p1 = pos[2 * b + 1];
  if (!in_bounds(static_cast<unsigned int>(p0), static_cast<unsigned int>(K)) ||
      !in_bounds(static_cast<unsigned int>(p1), static_cast<unsigned int>(K)))
    return;
  const uint32_t lo = codes_t[static_cast<size_t>(p0) * N + n];
  const uint32_t hi = codes_t[static_cast<size_t>(p1) * N + n];
  Wq[n * half + b] = static_cast<uint8_t>(lo | (hi << 4));
}

// g_idx[k] = pos[k] / G: the channel processed j-th belongs to group j / G.
__global__ void gptq_gidx_kernel(const int32_t* __restrict__ pos, int K, int G,
                                 int32_t* __restrict__ g_idx) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < K) g_idx[k] = pos[k] / G;
}

}  // namespace w4
