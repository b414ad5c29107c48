// Microbenchmark: the cost of one tcgen05.mma (kind::f16, bf16 in, fp32
// accumulate, cta_group::1) as a function of its shape, on every SM at once.
// One CTA per SM (the shared-memory request keeps it alone) allocates 512
// tensor-memory columns; one thread issues kMma MMAs back to back (A from
// tensor memory or from shared memory, B from shared memory, zero operands,
// 1 or 4 accumulators in turn), commits, and waits for the commit with the
// library's bounded mbarrier wait.  Reported: SM cycles per MMA (issue of
// the batch and issue-to-completion) and the implied dense FLOP rate over
// 148 SMs at the measured SM clock.  This is what the decode path's choice
// of warp-level MMA rests on: a narrow (N = 8..16) tensor-core MMA costs the
// SM as much as a wide one.
#include <cstdint>
#include <cstdio>

#include <cuda_runtime.h>

#include "../csrc/w4_ptx.cuh"
using namespace w4;

constexpr int kMma = 512;
constexpr int kSmemBytes = 160 * 1024;  // one CTA per SM

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

// mode 0: A in tensor memory (TS); mode 1: A in shared memory (SS)
__global__ void __launch_bounds__(128, 1) probe(int mode, int M, int N, int nacc, long long* out) {
  extern __shared__ __align__(1024) uint8_t sm[];
  uint8_t* buf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t holder;
  // operands: 96 KB of zeros (A tile at buf, B tile at buf + 32 KB)
  for (int i = threadIdx.x; i < 96 * 1024 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(buf)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(&holder, 512);
    tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = holder;
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_bf16_f32(M, N);
    const uint32_t base = smem_u32(buf);
    const uint64_t adesc = smem_desc_sw128(base);
    const uint64_t bdesc = smem_desc_sw128(base + 32768);
    const uint32_t dstride = N <= 64 ? 64 : 256;  // accumulator columns apart
    const long long t0 = clock64();
    for (int i = 0; i < kMma; ++i) {
      const uint32_t d = tmem + static_cast<uint32_t>((i % nacc) * dstride) % 256;
      if (mode == 0)
        mma_bf16_ts(d, tmem + 256 + (i % 4) * 8, bdesc + ((i & 3) * 2), idesc, i >= nacc);
      else
        mma_ss(d, adesc + ((i & 3) * 2), bdesc + ((i & 3) * 2), idesc, i >= nacc);
    }
    const long long t1 = clock64();
    mma_commit(&bar);
    mbar_wait(&bar, 0);
    const long long t2 = clock64();
    if (blockIdx.x == 0) {
      out[0] = t1 - t0;
      out[1] = t2 - t0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(tmem, 512);
}

// Issue pattern: A and B from shared memory, M = 128, `issuers` warps (1 or
// 2) each issuing kMma MMAs from one thread; with 1 issuer it alternates
// over `nacc` accumulators 256 columns apart, with 2 each issuer keeps its
// own accumulator (columns 0 and 256).  Each issuer commits to its own
// mbarrier and waits for it (bounded).  out[0]: cycles of the slower issuer.
__global__ void __launch_bounds__(128, 1) probe_issue(int N, int issuers, int nacc, int a_tmem, long long* out) {
  extern __shared__ __align__(1024) uint8_t sm[];
  uint8_t* buf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar[2];
  __shared__ uint32_t holder;
  __shared__ long long cyc[2];
  for (int i = threadIdx.x; i < 96 * 1024 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(buf)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_barrier_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(&holder, 512);
    tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = holder;
  const int warp = threadIdx.x >> 5;
  if (warp < issuers && (threadIdx.x & 31) == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, N);
    const uint32_t base = smem_u32(buf);
    const uint64_t adesc = smem_desc_sw128(base);
    const uint64_t bdesc = smem_desc_sw128(base + 32768);
    const long long t0 = clock64();
    for (int i = 0; i < kMma; ++i) {
      if (a_tmem) {
        // A from tensor memory (columns 384..415, shared by the issuers),
        // accumulators of N <= 128 at columns 0 and 128
        const uint32_t col = static_cast<uint32_t>(issuers == 2 ? warp : i % nacc) * 128u;
        mma_bf16_ts(tmem + col, tmem + 384 + (i % 4) * 8, bdesc + ((i & 3) * 2), idesc,
                    i >= (issuers == 2 ? 1 : nacc));
      } else {
        const uint32_t col = issuers == 2 ? static_cast<uint32_t>(warp) * 256u
                                          : static_cast<uint32_t>(i % nacc) * 256u;
        mma_ss(tmem + col, adesc + ((i & 3) * 2), bdesc + ((i & 3) * 2), idesc, i >= (issuers == 2 ? 1 : nacc));
      }
    }
    mma_commit(&bar[warp]);
    mbar_wait(&bar[warp], 0);
    cyc[warp] = clock64() - t0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && blockIdx.x == 0) out[0] = issuers == 2 && cyc[1] > cyc[0] ? cyc[1] : cyc[0];
  if (threadIdx.x < 32) tmem_dealloc(tmem, 512);
}

// SM clock (GHz) from one CTA spinning on clock64 against the global timer.
__global__ void clock_probe(double* ghz) {
  unsigned long long g0, g1;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(g0));
  const long long c0 = clock64();
  while (clock64() - c0 < 20000000) {
  }
  const long long c1 = clock64();
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(g1));
  *ghz = static_cast<double>(c1 - c0) / static_cast<double>(g1 - g0);
}

int main() {
  long long* d;
  double* dg;
  cudaMalloc(&d, 16);
  cudaMalloc(&dg, 8);
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  cudaFuncSetAttribute(probe, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  clock_probe<<<1, 1>>>(dg);
  double ghz = 0;
  cudaMemcpy(&ghz, dg, 8, cudaMemcpyDeviceToHost);
  printf("SM clock %.3f GHz, %d SMs, %d MMAs per CTA\n", ghz, sms, kMma);
  const int Ns[] = {16, 32, 64, 128, 256};
  for (int mode = 0; mode < 2; ++mode)
    for (int M : {128, 64})
      for (int N : Ns)
        for (int nacc : {1, 4}) {
          if (M == 64 && mode == 0) continue;  // A from tensor memory only at M = 128
          if (nacc == 4 && N > 64) continue;
          probe<<<sms, 128, kSmemBytes>>>(mode, M, N, nacc, d);
          long long h[2];
          const cudaError_t e = cudaMemcpy(h, d, 16, cudaMemcpyDeviceToHost);
          if (e != cudaSuccess) {
            printf("error %s\n", cudaGetErrorString(e));
            return 1;
          }
          const double cyc = static_cast<double>(h[1]) / kMma;
          const double tflops = 2.0 * M * N * 16 / cyc * ghz * 1e9 * sms / 1e12;
          printf("%s M=%3d N=%3d acc=%d: issue %6.1f cycles/MMA, complete %6.1f cycles/MMA, %7.1f TFLOP/s\n",
                 mode == 0 ? "A in TMEM" : "A in SMEM", M, N, nacc,
                 static_cast<double>(h[0]) / kMma, cyc, tflops);
        }
  // issue pattern: one thread alternating two N = 256 accumulators, and two
  // issuing warps with one accumulator each
  cudaFuncSetAttribute(probe_issue, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  struct Case { int N, issuers, nacc, a_tmem; };
  const Case cases[] = {{256, 1, 1, 0}, {256, 1, 2, 0}, {256, 2, 1, 0}, {128, 1, 1, 0}, {128, 2, 1, 0},
                        {64, 2, 1, 0},  {128, 1, 1, 1}, {128, 2, 1, 1}, {64, 2, 1, 1}};
  for (const Case& c : cases) {
    probe_issue<<<sms, 128, kSmemBytes>>>(c.N, c.issuers, c.nacc, c.a_tmem, d);
    long long h = 0;
    const cudaError_t e = cudaMemcpy(&h, d, 8, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
      printf("error %s\n", cudaGetErrorString(e));
      return 1;
    }
    const double mmas = static_cast<double>(kMma) * c.issuers;
    const double cyc = static_cast<double>(h) / mmas;
    const double tflops = 2.0 * 128 * c.N * 16 / cyc * ghz * 1e9 * sms / 1e12;
    printf("A in %s M=128 N=%3d, %d issuer(s), %d accumulator(s) each issuer: %6.1f cycles/MMA per SM, %7.1f TFLOP/s\n",
           c.a_tmem ? "TMEM" : "SMEM", c.N, c.issuers, c.issuers == 2 ? 1 : c.nacc, cyc, tflops);
  }
  return 0;
}
