// w4_lib.cu -- the C ABI (include/w4.h): host-side argument checks and kernel
// launches.  One translation unit so that the per-device error word is a
// single object.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/w4.h"
#include "w4_gemm_kernel.cuh"
#include "w4_gemv_kernel.cuh"
#include "w4_gptq.cuh"
#include "w4_int8.cuh"
#include "w4_int8_tc.cuh"
#include "w4_prepack.cuh"
#include "w4_quant.cuh"
#include "w4_ptx.cuh"

using namespace w4;

namespace {

inline cudaStream_t as_stream(w4_stream s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}
inline bool valid_group(int G) { return G == 32 || G == 64 || G == 128; }
inline w4_status launch_status(cudaError_t e) { return e == cudaSuccess ? W4_OK : W4_ERR_CUDA; }
inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }
int sm_count();  // the current device's SMs (defined with the GEMM host code)

// A kernel's dynamic shared-memory limit is a per-device setting: raise it
// once on each device the kernel runs on (`done` holds one bit per device).
template <class Kernel>
cudaError_t ensure_smem_limit(Kernel* kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

bool int4_shape_ok(int N, int K, int G) {
  return N >= 1 && K >= 1 && valid_group(G) && K >= G && K % G == 0 && K % 2 == 0 &&
         static_cast<long long>(N) * K <= (1LL << 40);
}

// Failure-path check: one bounded wait on an mbarrier that nothing arrives
// on, with a short limit (about 1 ms): it must give up, set the device error
// word and return, leaving the context usable.
constexpr long long kSelftestWaitCycles = 2000000;

__global__ void wait_timeout_probe_kernel(long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, limit);
}

}  // namespace

extern "C" {

const char* w4_status_string(w4_status s) {
  switch (s) {
    case W4_OK: return "ok";
    case W4_ERR_INVALID_ARG: return "invalid argument";
    case W4_ERR_UNSUPPORTED: return "unsupported";
    case W4_ERR_CUDA: return "CUDA error";
    case W4_ERR_TIMEOUT: return "device pipeline wait timed out";
    case W4_ERR_DEVICE_INPUT: return "device found invalid input data";
    case W4_ERR_SCRATCH_LIMIT:
      return "workspace needed exceeds the static scratch (W4_STATIC_SCRATCH_BYTES)";
    case W4_ERR_BOUNDS:
      return "bounds-checked build: a kernel index fell outside its buffer (access skipped)";
    default: return "unknown status";
  }
}

int w4_version(void) { return 100; }

w4_status w4_device_status(w4_stream stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return W4_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(v)) != cudaSuccess) return W4_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return W4_ERR_CUDA;
  }
  if (v & W4_DEV_ERR_BOUNDS) return W4_ERR_BOUNDS;
  if (v & W4_DEV_ERR_TIMEOUT) return W4_ERR_TIMEOUT;
  if (v & W4_DEV_ERR_INPUT) return W4_ERR_DEVICE_INPUT;
  return W4_OK;
}

int w4_checked_build(void) { return kChecked ? 1 : 0; }

w4_status w4_selftest_wait_timeout(w4_stream stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, as_stream(stream)>>>(kSelftestWaitCycles);
  return launch_status(cudaGetLastError());
}

double w4_weight_bytes(int N, int K, int G) {
  if (!int4_shape_ok(N, K, G)) return 0.0;
  const double groups = static_cast<double>(N) * (K / G);
  return static_cast<double>(N) * K / 2.0 + groups * 2.0 + groups * 0.5;
}

// ---------------------------------------------------------------- INT4 RTN
}  // extern "C"

namespace {

template <bool SYM>
w4_status quantize_int4(const float* W, int N, int K, int G, const int32_t* g_idx, uint8_t* Wq,
                        uint16_t* scales, uint8_t* zeros, w4_stream stream) {
  if (!W || !Wq || !scales || !zeros) return W4_ERR_INVALID_ARG;
  if (!int4_shape_ok(N, K, G)) return W4_ERR_INVALID_ARG;
  if (!aligned(W, 4) || !aligned(scales, 2) || (g_idx && !aligned(g_idx, 4)))
    return W4_ERR_INVALID_ARG;
  const long long total = static_cast<long long>(N) * K;
  if (!g_idx && total % 128 == 0 && aligned(W, 16) && aligned(Wq, 2)) {
    // contiguous groups: the flat kernel, a persistent grid over 512-weight chunks
    const long long ngroups = total / G;
    const long long warps = (total + 511) / 512;
    const unsigned blocks = static_cast<unsigned>(
        std::min<long long>((warps + 7) / 8, static_cast<long long>(sm_count()) * 8));
    cudaStream_t st = as_stream(stream);
    switch (G) {
      case 32:
        rtn_quantize_flat_kernel<SYM, 32><<<blocks, 256, 0, st>>>(W, ngroups, Wq, scales, zeros);
        break;
      case 64:
        rtn_quantize_flat_kernel<SYM, 64><<<blocks, 256, 0, st>>>(W, ngroups, Wq, scales, zeros);
        break;
      default:
        rtn_quantize_flat_kernel<SYM, 128><<<blocks, 256, 0, st>>>(W, ngroups, Wq, scales, zeros);
        break;
    }
    return launch_status(cudaGetLastError());
  }
  const int ng = K / G;
  const size_t smem = static_cast<size_t>(ng) * 16;
  if (smem > 200 * 1024) return W4_ERR_UNSUPPORTED;
  static std::atomic<uint64_t> smem_set{0};
  if (ensure_smem_limit(rtn_quantize_kernel<SYM>, 200 * 1024, smem_set) != cudaSuccess) {
    cudaGetLastError();
    return W4_ERR_CUDA;
  }
  rtn_quantize_kernel<SYM>
      <<<N, 256, smem, as_stream(stream)>>>(W, N, K, G, g_idx, Wq, scales, zeros);
  return launch_status(cudaGetLastError());
}

}  // namespace

extern "C" {

w4_status w4_quantize_rtn(const float* W, int N, int K, int G, const int32_t* g_idx,
                          uint8_t* Wq, uint16_t* scales, uint8_t* zeros, w4_stream stream) {
  return quantize_int4<false>(W, N, K, G, g_idx, Wq, scales, zeros, stream);
}

w4_status w4_quantize_sym(const float* W, int N, int K, int G, const int32_t* g_idx,
                          uint8_t* Wq, uint16_t* scales, uint8_t* zeros, w4_stream stream) {
  return quantize_int4<true>(W, N, K, G, g_idx, Wq, scales, zeros, stream);
}

w4_status w4_awq_scale_weights(const float* W, const float* s, int N, int K, float* W_out,
                               w4_stream stream) {
  if (!W || !s || !W_out) return W4_ERR_INVALID_ARG;
  if (N < 1 || K < 1) return W4_ERR_INVALID_ARG;
  if (!aligned(W, 4) || !aligned(s, 4) || !aligned(W_out, 4)) return W4_ERR_INVALID_ARG;
  if (K % 4 == 0 && aligned(W, 16) && aligned(s, 16) && aligned(W_out, 16)) {
    // one CTA per row at a time, 8 resident per SM
    const int blocks = std::min(N, sm_count() * 8);
    awq_scale_weights_vec_kernel<<<static_cast<unsigned>(blocks), kAwqThreads, 0,
                                   as_stream(stream)>>>(
        reinterpret_cast<const float4*>(W), reinterpret_cast<const float4*>(s), N, K / 4,
        reinterpret_cast<float4*>(W_out));
    return launch_status(cudaGetLastError());
  }
  const size_t total = static_cast<size_t>(N) * K;
  const size_t blocks =
      std::min<size_t>((total + 255) / 256, static_cast<size_t>(sm_count()) * 16);
  awq_scale_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
      W, s, N, K, W_out);
  return launch_status(cudaGetLastError());
}

}  // extern "C"

// ---------------------------------------------------------------------------
// GPTQ: workspace regions (each 256-byte aligned).
namespace {

struct GptqLayout {
  size_t A, T, U, Q, E, codes, d, lambda, dead, perm, pos, total;
};

GptqLayout gptq_layout(int N, int K) {
  auto r = [](size_t v) { return (v + 255) / 256 * 256; };
  const size_t kk = static_cast<size_t>(K) * K, nk = static_cast<size_t>(N) * K;
  GptqLayout l{};
  size_t o = 0;
  l.A = o;      o += r(kk * 8);
  l.T = o;      o += r(kk * 8);
  l.U = o;      o += r(kk * 4);
  l.Q = o;      o += r(nk * 4);
  l.E = o;      o += r(static_cast<size_t>(kGptqB) * N * 4);
  l.codes = o;  o += r(nk);
  l.d = o;      o += r(static_cast<size_t>(K) * 8);
  l.lambda = o; o += 256;
  l.dead = o;   o += r(static_cast<size_t>(K));
  l.perm = o;   o += r(static_cast<size_t>(K) * 4);
  l.pos = o;    o += r(static_cast<size_t>(K) * 4);
  l.total = o;
  return l;
}

bool gptq_shape_ok(int N, int K, int G) {
  return int4_shape_ok(N, K, G) && K % kChol == 0 && K <= 65536;
}

}  // namespace

extern "C" {

size_t w4_gptq_workspace_bytes(int N, int K, int G) {
  if (!gptq_shape_ok(N, K, G)) return 0;
  return gptq_layout(N, K).total;
}

w4_status w4_gptq_hessian(const uint16_t* X, int n, int K, float* H, w4_stream stream) {
  if (!X || !H || n < 1 || K < 1 || K > 65536) return W4_ERR_INVALID_ARG;
  if (!aligned(X, 2) || !aligned(H, 4)) return W4_ERR_INVALID_ARG;
  const int t = ceil_div(K, 64);
  gptq_hessian_kernel<<<dim3(t, t), 256, 0, as_stream(stream)>>>(X, n, K, H);
  return launch_status(cudaGetLastError());
}

w4_status w4_gptq_quantize(const float* W, const float* H, int N, int K, int G, int act_order,
                           float damp, uint8_t* Wq, uint16_t* scales, uint8_t* zeros,
                           int32_t* g_idx, void* workspace, size_t workspace_bytes,
                           w4_stream stream) {
  if (!W || !H || !Wq || !scales || !zeros || !workspace) return W4_ERR_INVALID_ARG;
  if (act_order && !g_idx) return W4_ERR_INVALID_ARG;
  if (!gptq_shape_ok(N, K, G) || !(damp >= 0.0f)) return W4_ERR_INVALID_ARG;
  if (!aligned(W, 4) || !aligned(H, 4) || !aligned(scales, 2) || !aligned(workspace, 256) ||
      (g_idx && !aligned(g_idx, 4)))
    return W4_ERR_INVALID_ARG;
  const GptqLayout l = gptq_layout(N, K);
  if (workspace_bytes < l.total) return W4_ERR_INVALID_ARG;
  static std::atomic<uint64_t> smem_set{0};
  if (ensure_smem_limit(gptq_block_kernel, static_cast<int>(kGptqBlockSmem), smem_set) !=
      cudaSuccess) {
    cudaGetLastError();
    return W4_ERR_CUDA;
  }
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* A = reinterpret_cast<double*>(ws + l.A);
  double* T = reinterpret_cast<double*>(ws + l.T);
  float* U = reinterpret_cast<float*>(ws + l.U);
  float* Q = reinterpret_cast<float*>(ws + l.Q);
  float* E = reinterpret_cast<float*>(ws + l.E);
  uint8_t* codes = ws + l.codes;
  double* d = reinterpret_cast<double*>(ws + l.d);
  double* lambda = reinterpret_cast<double*>(ws + l.lambda);
  uint8_t* dead = ws + l.dead;
  int32_t* perm = reinterpret_cast<int32_t*>(ws + l.perm);
  int32_t* pos = reinterpret_cast<int32_t*>(ws + l.pos);

  // prepare: diagonal, order, damping, A = J P^T H P J + lambda I, Q = W P
  gptq_diag_kernel<<<ceil_div(K, 256), 256, 0, st>>>(H, K, d, dead);
  gptq_order_kernel<<<ceil_div(K, 256), 256, 0, st>>>(d, K, act_order ? 1 : 0, perm, pos);
  gptq_damp_kernel<<<1, 256, 0, st>>>(d, K, static_cast<double>(damp), lambda);
  gptq_build_kernel<<<dim3(ceil_div(K, 32), ceil_div(K, 8)), 256, 0, st>>>(H, d, perm, lambda,
                                                                            K, A);
  const size_t nk = static_cast<size_t>(N) * K;
  gptq_gather_w_kernel<<<static_cast<unsigned>((nk + 255) / 256), 256, 0, st>>>(W, perm, dead, N,
                                                                               K, Q);
  // factor: A = L' L'^T (lower, in place), T = L'^-1, U = J T J
  const int nb = K / kChol;
  for (int jb = 0; jb < nb; ++jb) {
    chol_diag_kernel<<<1, kChol * kChol, 0, st>>>(A, K, jb);
    const int rest = nb - jb - 1;
    if (rest > 0) {
      chol_panel_kernel<<<rest, kChol, 0, st>>>(A, K, jb);
      chol_update_kernel<<<dim3(rest, rest), kChol * kChol, 0, st>>>(A, K, jb);
    }
  }
  trinv_diag_kernel<<<nb, kChol, 0, st>>>(A, K, T);
  // off-diagonal blocks by doubling; P (at most K^2 / 4 doubles) borrows U's
  // region, which is written only after T is complete
  double* P = reinterpret_cast<double*>(U);
  for (int s = 1; s < nb; s *= 2) {
    const dim3 grid(s, s, ceil_div(nb, 2 * s));
    trinv_level_p_kernel<<<grid, kChol * kChol, 0, st>>>(A, T, K, nb, s, P);
    trinv_level_t_kernel<<<grid, kChol * kChol, 0, st>>>(P, K, nb, s, T);
  }
  gptq_u_kernel<<<dim3(ceil_div(K, 32), ceil_div(K, 8)), 256, 0, st>>>(T, K, U);
  // quantize: lazy blocks of kGptqB columns
  for (int j0 = 0; j0 < K; j0 += kGptqB) {
    const int bw = std::min(kGptqB, K - j0);
    gptq_block_kernel<<<ceil_div(N, kGptqRows), kGptqRows, kGptqBlockSmem, st>>>(
        Q, U, N, K, G, j0, bw, E, codes, scales, zeros);
    if (j0 + bw < K)
      gptq_trailing_kernel<<<dim3(ceil_div(K - j0 - bw, 64), ceil_div(N, 64)), 256, 0, st>>>(
          Q, U, E, N, K, j0, bw);
  }
  const size_t half = nk / 2;
  gptq_pack_kernel<<<static_cast<unsigned>((half + 255) / 256), 256, 0, st>>>(codes, pos, N, K,
                                                                              Wq);
  if (g_idx) gptq_gidx_kernel<<<ceil_div(K, 256), 256, 0, st>>>(pos, K, G, g_idx);
  return launch_status(cudaGetLastError());
}

}  // extern "C"

// ---------------------------------------------------------------------------
// LLM.int8: workspace regions (each 256-byte aligned).
namespace {

// Regions of the LLM.int8 workspace (each 256-byte aligned), all written by
// the call before they are read (the counters and the accumulator cleared by
// its first two kernels).
// More than this many tokens: the tensor-core (kind::i8) product.
constexpr int kInt8TcMinM = 33;

// The tensor-core product's tiling and split-K plan.
struct I8Plan {
  int MT, tiles_n, tiles_m, KS, splits;
};

I8Plan int8_tc_plan(int M, int N, int K) {
  I8Plan p{};
  p.MT = M <= 64 ? 64 : M <= 128 ? 128 : 256;
  p.tiles_n = (N + 127) / 128;
  p.tiles_m = (M + p.MT - 1) / p.MT;
  p.KS = (K + 127) / 128;
  const long long tiles = static_cast<long long>(p.tiles_n) * p.tiles_m;
  // K split by a cost model over the SMs, in stages of 4 MMAs: per CTA the
  // prologue and epilogue count 1.5 stages, a split tile's round trip at
  // least 12 more, and more when the last CTA's reduction needs more than
  // 8 L2 round trips (MT / 8 column chunks times one per 4 K ranges, about
  // 1.2 stages each); at most 16 ranges of at least 4 stages
  const long long sms = sm_count();
  const long long smax =
      tiles > 65536 ? 1 : std::min<long long>(16, std::max<long long>(1, p.KS / 4));
  double best = 1e30;
  p.splits = 1;
  for (long long s = 1; s <= smax; ++s) {
    const double rounds = static_cast<double>(p.MT / 8) * static_cast<double>((s + 3) / 4);
    const double rt = s > 1 ? std::max(12.0, 4.0 + 1.2 * rounds) : 0.0;
    const double cost = static_cast<double>((tiles * s + sms - 1) / sms) *
                        (static_cast<double>((p.KS + s - 1) / s) + 1.5 + rt);
    if (cost < best - 1e-9) {
      best = cost;
      p.splits = static_cast<int>(s);
    }
  }
  return p;
}

struct Int8Layout {
  size_t counter, acc, flag, list, cnt, part, olist, ocount, qx, sx, tcpart, total;
  int nscan;         // scan CTAs (kInt8ScanCh channels each)
  int counters;      // counters the scan clears
};

Int8Layout int8_layout(int M, int N, int K) {
  auto r = [](size_t v) { return (v + 255) / 256 * 256; };
  Int8Layout l{};
  l.nscan = (K + kInt8ScanCh - 1) / kInt8ScanCh;
  const bool tc = M >= kInt8TcMinM;
  const I8Plan tp = int8_tc_plan(M, N, K);
  const long long tiles = static_cast<long long>(tp.tiles_n) * tp.tiles_m;
  l.counters = std::max((N + 15) / 16, tc ? static_cast<int>(std::min<long long>(tiles, 65536)) : 0);
  size_t o = 0;
  l.counter = o; o += r(static_cast<size_t>(l.counters) * 4);
  l.acc = o;     o += tc ? 0 : r(static_cast<size_t>(M) * N * 4);
  l.flag = o;    o += r(static_cast<size_t>(K));
  l.list = o;    o += r(static_cast<size_t>(l.nscan) * kInt8ScanCh * 4);
  l.cnt = o;     o += r(static_cast<size_t>(l.nscan) * 4);
  l.part = o;    o += r(static_cast<size_t>(l.nscan) * M * 4);
  l.olist = o;   o += r(static_cast<size_t>(K) * 4);
  l.ocount = o;  o += 256;
  l.qx = o;      o += r(static_cast<size_t>(M) * K);
  l.sx = o;      o += r(static_cast<size_t>(M) * 4);
  l.tcpart = o;
  if (tc && tp.splits > 1)
    o += r(static_cast<size_t>(tiles) * tp.splits * tp.MT * kI8Rows * 4);
  l.total = o;
  return l;
}

// 3-D tensor map over an int8 [rows, K] matrix: {K, rows, 1}, box {128,
// box_rows, 1}, 128-byte swizzle (one 128-channel stage = one 128-byte row),
// rows past the end read as zero.
bool encode_i8_map(CUtensorMap* map, const int8_t* base, int rows, int K, int box_rows);

template <class C>
cudaError_t launch_i8_tc(const CUtensorMap& wmap, const CUtensorMap& xmap, const I8TcArgs& a,
                         int ctas, cudaStream_t st) {
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t attr_err = ensure_smem_limit(int8_tc_kernel<C>, C::kSmemBytes, smem_set);
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, int8_tc_kernel<C>, wmap, xmap, a);
}

bool int8_shape_ok(int M, int N, int K) {
  return M >= 1 && N >= 1 && K >= 64 && K % 64 == 0 && K <= 65536 &&
         static_cast<long long>(M) * N <= (1LL << 31) && static_cast<long long>(N) * K <= (1LL << 40);
}

}  // namespace

extern "C" {

w4_status llm_int8_quantize_weights(const float* W, int N, int K, int8_t* qw, float* sw,
                                    w4_stream stream) {
  if (!W || !qw || !sw || N < 1 || K < 1) return W4_ERR_INVALID_ARG;
  if (!aligned(W, 4) || !aligned(sw, 4)) return W4_ERR_INVALID_ARG;
  int8_quantize_weights_kernel<<<N, 256, 0, as_stream(stream)>>>(W, N, K, qw, sw);
  return launch_status(cudaGetLastError());
}

size_t llm_int8_workspace_bytes(int M, int N, int K) {
  if (!int8_shape_ok(M, N, K)) return 0;
  return int8_layout(M, N, K).total;
}

w4_status llm_int8_gemm(const uint16_t* X, const int8_t* qw, const float* sw, int M, int N, int K,
                        float threshold, uint16_t* Y, void* workspace, size_t workspace_bytes,
                        w4_stream stream) {
  if (!X || !qw || !sw || !Y || !workspace) return W4_ERR_INVALID_ARG;
  if (!int8_shape_ok(M, N, K) || !(threshold >= 0.0f)) return W4_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(qw, 16) || !aligned(sw, 4) || !aligned(Y, 2) ||
      !aligned(workspace, 256))
    return W4_ERR_INVALID_ARG;
  const Int8Layout l = int8_layout(M, N, K);
  if (workspace_bytes < l.total) return W4_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* flag = ws + l.flag;
  int32_t* list = reinterpret_cast<int32_t*>(ws + l.list);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + l.cnt);
  float* part = reinterpret_cast<float*>(ws + l.part);
  Int8Args a{};
  a.qw = qw;
  a.qx = reinterpret_cast<int8_t*>(ws + l.qx);
  a.sx = reinterpret_cast<float*>(ws + l.sx);
  a.sw = sw;
  a.X = X;
  a.olist = reinterpret_cast<int32_t*>(ws + l.olist);
  a.ocount = reinterpret_cast<int32_t*>(ws + l.ocount);
  a.acc = reinterpret_cast<int*>(ws + l.acc);
  a.counter = reinterpret_cast<unsigned int*>(ws + l.counter);
  a.Y = Y;
  a.M = M;
  a.N = N;
  a.K = K;
  // work items: (16-row tile, K slice), one wave of warps (kInt8CtasPerSm
  // CTAs of kInt8Warps per SM)
  a.row_tiles = ceil_div(N, 16);
  const int steps_total = K / 64;
  const int target = sm_count() * kInt8Warps * kInt8CtasPerSm;
  a.slices = std::min(steps_total, std::max(1, target / a.row_tiles));
  a.steps = ceil_div(steps_total, a.slices);
  a.slices = ceil_div(steps_total, a.steps);
  const long long items = static_cast<long long>(a.row_tiles) * a.slices;
  // three launches chained by programmatic dependent launch
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(l.nscan);
  cfg.blockDim = dim3(32 * std::min(M, 32));
  cudaError_t e = cudaLaunchKernelEx(&cfg, int8_scan_kernel, X, M, K, threshold, flag, list, cnt,
                                     part, a.counter, l.counters);
  if (e == cudaSuccess) {
    cfg.gridDim = dim3(M, ceil_div(K, 2048));
    cfg.blockDim = dim3(256);
    e = cudaLaunchKernelEx(&cfg, int8_quantize_x_kernel, X, static_cast<const uint8_t*>(flag),
                           static_cast<const float*>(part), static_cast<const int32_t*>(list),
                           static_cast<const int32_t*>(cnt), l.nscan, M, K,
                           const_cast<int8_t*>(a.qx), const_cast<float*>(a.sx),
                           const_cast<int32_t*>(a.olist), const_cast<int32_t*>(a.ocount), a.acc,
                           M >= kInt8TcMinM ? 0 : N);
  }
  if (e == cudaSuccess && M >= kInt8TcMinM) {
    // tensor-core product with the epilogue fused
    const I8Plan tp = int8_tc_plan(M, N, K);
    CUtensorMap wmap, xmap;
    if (!encode_i8_map(&wmap, qw, N, K, kI8Rows) || !encode_i8_map(&xmap, a.qx, M, K, tp.MT))
      return W4_ERR_CUDA;
    I8TcArgs t{};
    t.sx = a.sx;
    t.sw = sw;
    t.X = X;
    t.qw = qw;
    t.olist = a.olist;
    t.ocount = a.ocount;
    t.Y = Y;
    t.partial = reinterpret_cast<int*>(ws + l.tcpart);
    t.counter = a.counter;
    t.M = M;
    t.N = N;
    t.K = K;
    t.KS = tp.KS;
    t.tiles_n = tp.tiles_n;
    t.tiles_m = tp.tiles_m;
    t.splits = tp.splits;
    t.partial_count = (l.total - l.tcpart) / 4;
    const int ctas = tp.tiles_n * tp.tiles_m * tp.splits;
    switch (tp.MT) {
      case 64: e = launch_i8_tc<I8Cfg<64, 6>>(wmap, xmap, t, ctas, st); break;
      case 128: e = launch_i8_tc<I8Cfg<128, 5>>(wmap, xmap, t, ctas, st); break;
      default: e = launch_i8_tc<I8Cfg<256, 4>>(wmap, xmap, t, ctas, st); break;
    }
    return launch_status(e);
  }
  if (e == cudaSuccess) {
    cfg.gridDim = dim3(static_cast<unsigned>((items + kInt8Warps - 1) / kInt8Warps));
    cfg.blockDim = dim3(kInt8Warps * 32);
    // the epilogue's per-warp slice: one chunk of outlier channels for 16
    // rows and M tokens, and the chunk's in-bounds flags
    cfg.dynamicSmemBytes =
        M <= kInt8EpiDirectM
            ? 0
            : static_cast<size_t>(kInt8Warps) * ((16 + M) * kInt8EpiChunk + kInt8EpiChunk) * sizeof(float);
    e = cudaLaunchKernelEx(&cfg, int8_product_kernel, a);
  }
  return launch_status(e);
}

w4_status w4_dequant(const uint8_t* Wq, const uint16_t* scales, const uint8_t* zeros,
                     const int32_t* g_idx, int N, int K, int G, uint16_t* W_out,
                     w4_stream stream) {
  if (!Wq || !scales || !zeros || !W_out) return W4_ERR_INVALID_ARG;
  if (!int4_shape_ok(N, K, G) || K % 8 != 0) return W4_ERR_INVALID_ARG;
  if (!aligned(Wq, 4) || !aligned(W_out, 16) || !aligned(scales, 2) ||
      (g_idx && !aligned(g_idx, 4)))
    return W4_ERR_INVALID_ARG;
  if (!g_idx && aligned(Wq, 8)) {
    // contiguous groups: 16 weights (one group) per thread over the flat array
    const long long total16 = static_cast<long long>(N) * K / 16;
    const unsigned blocks = static_cast<unsigned>(ceil_div(total16, 256));
    cudaStream_t st = as_stream(stream);
    switch (G) {
      case 32:
        rtn_dequant_flat_kernel<32><<<blocks, 256, 0, st>>>(Wq, scales, zeros, total16, W_out);
        break;
      case 64:
        rtn_dequant_flat_kernel<64><<<blocks, 256, 0, st>>>(Wq, scales, zeros, total16, W_out);
        break;
      default:
        rtn_dequant_flat_kernel<128><<<blocks, 256, 0, st>>>(Wq, scales, zeros, total16, W_out);
        break;
    }
    return launch_status(cudaGetLastError());
  }
  const long long total = static_cast<long long>(N) * (K / 8);
  rtn_dequant_kernel<<<ceil_div(total, 256), 256, 0, as_stream(stream)>>>(Wq, scales, zeros,
                                                                           g_idx, N, K, G, W_out);
  return launch_status(cudaGetLastError());
}

// ---------------------------------------------------------------- prepack
size_t w4_prepacked_bytes(int N, int K, int G, int act_order) {
  if (!int4_shape_ok(N, K, G)) return 0;
  const size_t tiles = ceil_div(N, kTileRows), ks = ceil_div(K, kStageK);
  return tiles * ks * int4_stage_bytes(G) + (act_order ? static_cast<size_t>(K) * 4 : 0);
}

static int32_t* perm_region(uint8_t* Wp, int N, int K, int G) {
  const size_t tiles = ceil_div(N, kTileRows), ks = ceil_div(K, kStageK);
  return reinterpret_cast<int32_t*>(Wp + tiles * ks * int4_stage_bytes(G));
}

w4_status w4_prepack(const uint8_t* Wq, const uint16_t* scales, const uint8_t* zeros,
                     const int32_t* g_idx, int N, int K, int G, uint8_t* Wp, w4_stream stream) {
  if (!Wq || !scales || !zeros || !Wp) return W4_ERR_INVALID_ARG;
  if (!int4_shape_ok(N, K, G)) return W4_ERR_INVALID_ARG;
  if (!aligned(Wp, 16) || !aligned(scales, 2) || (g_idx && !aligned(g_idx, 4)))
    return W4_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  int32_t* perm = nullptr;
  if (g_idx) {
    perm = perm_region(Wp, N, K, G);
    act_order_perm_kernel<<<1, 1024, 0, st>>>(g_idx, K, G, perm);
    if (cudaGetLastError() != cudaSuccess) return W4_ERR_CUDA;
  }
  dim3 grid(ceil_div(K, kStageK), ceil_div(N, kTileRows));
  int4_prepack_kernel<<<grid, 256, 0, st>>>(Wq, scales, zeros, perm, N, K, G, Wp);
  return launch_status(cudaGetLastError());
}

w4_status w4_unprepack(const uint8_t* Wp, int N, int K, int G, int act_order, uint8_t* Wq,
                       uint16_t* scales, uint8_t* zeros, int32_t* perm, w4_stream stream) {
  if (!Wp || !Wq || !scales || !zeros) return W4_ERR_INVALID_ARG;
  if (!int4_shape_ok(N, K, G) || !aligned(Wp, 16)) return W4_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  dim3 grid(ceil_div(K, kStageK), ceil_div(N, kTileRows));
  int4_unprepack_kernel<<<grid, 256, 0, st>>>(Wp, N, K, G, Wq, scales, zeros);
  if (cudaGetLastError() != cudaSuccess) return W4_ERR_CUDA;
  if (act_order && perm) {
    const int32_t* src = perm_region(const_cast<uint8_t*>(Wp), N, K, G);
    if (cudaMemcpyAsync(perm, src, static_cast<size_t>(K) * 4, cudaMemcpyDeviceToDevice, st) !=
        cudaSuccess)
      return W4_ERR_CUDA;
  }
  return W4_OK;
}

// ---------------------------------------------------------------- NF4
void nf4_levels(float out[16]) {
  if (out) std::memcpy(out, kNf4LevelBitsHost, sizeof(kNf4LevelBitsHost));
}

static bool nf4_shape_ok(int N, int K, int blocksize, int dq_group) {
  return N >= 1 && K >= 64 && K % 64 == 0 && blocksize == 64 && dq_group >= 1 &&
         dq_group <= 1024 && static_cast<long long>(N) * K <= (1LL << 40);
}

}  // extern "C"

namespace {

// mean == nullptr: the plain double quantization; otherwise the
// mean-offset one, with the runs' means written to / read from `mean`.
template <int TABLE>
w4_status blockwise_quantize(const float* W, int N, int K, int blocksize, int dq_group,
                             uint8_t* Wq, uint8_t* absmax_q, float* s2, float* mean,
                             w4_stream stream) {
  if (!W || !Wq || !absmax_q || !s2) return W4_ERR_INVALID_ARG;
  if (!nf4_shape_ok(N, K, blocksize, dq_group)) return W4_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(Wq, 16) || !aligned(s2, 4) || !aligned(mean, 4))
    return W4_ERR_INVALID_ARG;
  const long long nb = static_cast<long long>(N) * K / 64;
  const int runs = ceil_div(nb, dq_group);
  const size_t smem = (512 + static_cast<size_t>(dq_group) + 64) * sizeof(float);
  if (mean)
    nf4_quantize_kernel<TABLE, true>
        <<<runs, kNf4QThreads, smem, as_stream(stream)>>>(W, nb, dq_group, Wq, absmax_q, s2, mean);
  else
    nf4_quantize_kernel<TABLE, false>
        <<<runs, kNf4QThreads, smem, as_stream(stream)>>>(W, nb, dq_group, Wq, absmax_q, s2, nullptr);
  return launch_status(cudaGetLastError());
}

w4_status blockwise_dequant(const uint8_t* Wq, const uint8_t* absmax_q, const float* s2,
                            const float* mean, int N, int K, int blocksize, int dq_group,
                            int table, uint16_t* W_out, w4_stream stream) {
  if (!Wq || !absmax_q || !s2 || !W_out) return W4_ERR_INVALID_ARG;
  if (!nf4_shape_ok(N, K, blocksize, dq_group)) return W4_ERR_INVALID_ARG;
  if (!aligned(Wq, 4) || !aligned(W_out, 16) || !aligned(s2, 4) || !aligned(mean, 4))
    return W4_ERR_INVALID_ARG;
  const long long total8 = static_cast<long long>(N) * K / 8;
  if (mean)
    nf4_dequant_kernel<true><<<ceil_div(total8, 256), 256, 0, as_stream(stream)>>>(
        Wq, absmax_q, s2, mean, total8, dq_group, table, W_out);
  else
    nf4_dequant_kernel<false><<<ceil_div(total8, 256), 256, 0, as_stream(stream)>>>(
        Wq, absmax_q, s2, nullptr, total8, dq_group, table, W_out);
  return launch_status(cudaGetLastError());
}

}  // namespace

extern "C" {

w4_status nf4_quantize(const float* W, int N, int K, int blocksize, int dq_group, uint8_t* Wq,
                       uint8_t* absmax_q, float* s2, w4_stream stream) {
  return blockwise_quantize<kTableNf4>(W, N, K, blocksize, dq_group, Wq, absmax_q, s2, nullptr,
                                       stream);
}

w4_status nf4_dequant(const uint8_t* Wq, const uint8_t* absmax_q, const float* s2, int N, int K,
                      int blocksize, int dq_group, uint16_t* W_out, w4_stream stream) {
  return blockwise_dequant(Wq, absmax_q, s2, nullptr, N, K, blocksize, dq_group, kTableNf4,
                           W_out, stream);
}

w4_status fp4_quantize(const float* W, int N, int K, int blocksize, int dq_group, uint8_t* Wq,
                       uint8_t* absmax_q, float* s2, w4_stream stream) {
  return blockwise_quantize<kTableFp4>(W, N, K, blocksize, dq_group, Wq, absmax_q, s2, nullptr,
                                       stream);
}

w4_status fp4_dequant(const uint8_t* Wq, const uint8_t* absmax_q, const float* s2, int N, int K,
                      int blocksize, int dq_group, uint16_t* W_out, w4_stream stream) {
  return blockwise_dequant(Wq, absmax_q, s2, nullptr, N, K, blocksize, dq_group, kTableFp4,
                           W_out, stream);
}

w4_status nf4_quantize_meandq(const float* W, int N, int K, int blocksize, int dq_group,
                              uint8_t* Wq, int8_t* absmax_q, float* mean, float* s2,
                              w4_stream stream) {
  if (!mean) return W4_ERR_INVALID_ARG;
  return blockwise_quantize<kTableNf4>(W, N, K, blocksize, dq_group, Wq,
                                       reinterpret_cast<uint8_t*>(absmax_q), s2, mean, stream);
}

w4_status nf4_dequant_meandq(const uint8_t* Wq, const int8_t* absmax_q, const float* mean,
                             const float* s2, int N, int K, int blocksize, int dq_group,
                             uint16_t* W_out, w4_stream stream) {
  if (!mean) return W4_ERR_INVALID_ARG;
  return blockwise_dequant(Wq, reinterpret_cast<const uint8_t*>(absmax_q), s2, mean, N, K,
                           blocksize, dq_group, kTableNf4, W_out, stream);
}

void fp4_levels(float out[16]) {
  if (out) std::memcpy(out, kFp4LevelsHost, sizeof(kFp4LevelsHost));
}

size_t nf4_prepacked_bytes(int N, int K) {
  if (!nf4_shape_ok(N, K, 64, 256)) return 0;
  return static_cast<size_t>(ceil_div(N, kTileRows)) * ceil_div(K, kStageK) * nf4_stage_bytes();
}

w4_status nf4_prepack(const uint8_t* Wq, const uint8_t* absmax_q, int N, int K, uint8_t* Wp,
                      w4_stream stream) {
  if (!Wq || !absmax_q || !Wp) return W4_ERR_INVALID_ARG;
  if (!nf4_shape_ok(N, K, 64, 256) || !aligned(Wp, 16)) return W4_ERR_INVALID_ARG;
  dim3 grid(ceil_div(K, kStageK), ceil_div(N, kTileRows));
  nf4_prepack_kernel<<<grid, 256, 0, as_stream(stream)>>>(Wq, absmax_q, N, K, Wp);
  return launch_status(cudaGetLastError());
}

}  // extern "C"

#include "w4_gemm_host.inc"
