// w4_gemm_kernel.cuh -- the warp-specialised tcgen05 kernel (see w4_gemm.cuh).
#pragma once

#include "w4_gemm.cuh"

namespace w4 {

// CTA mask of a pair's multicast commits: ranks 0 and 1 of the cluster
constexpr uint16_t kPairCtas = 0x3;

template <class C>
__global__ void __launch_bounds__(C::kThreads, C::kMinBlocks)
    w4_tc_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* xs = smem;                                   // STAGES x kXStageBytes
  uint8_t* wsl = xs + C::STAGES * C::kXStageBytes;      // STAGES x kWSlot
  uint64_t* bars = reinterpret_cast<uint64_t*>(wsl + C::STAGES * C::kWSlot);
  uint64_t* full = bars;                                // X + W landed       (tx)
  uint64_t* empty = full + C::STAGES;                   // MMAs done reading  (commit)
  uint64_t* afull = empty + C::STAGES;                  // A slot written     (8 warps)
  uint64_t* aempty = afull + C::kASlots;                // A slot consumed    (commit)
  uint64_t* accf = aempty + C::kASlots;                 // accumulator ready  (commit)
  uint64_t* epi1 = accf + 1;                            // partials stored    (8 warps)
  uint64_t* epi2 = epi1 + 1;                            // last-arrival known (1)
  uint64_t* xfull = epi2 + 1;                           // pair: both X halves landed (tx)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(xfull + (C::PAIR ? C::STAGES : 0));
  int* last_flag = reinterpret_cast<int*>(tmem_holder + 1);
  float* Ts = reinterpret_cast<float*>(                   // NF4 levels [16], 256-byte aligned
      (reinterpret_cast<uintptr_t>(tmem_holder + 4) + 255) & ~static_cast<uintptr_t>(255));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA pair: rank 0 (the leader) issues the MMAs; the barriers of the
  // shared MMA stream (xfull, afull) live in the leader's shared memory.
  const uint32_t rank = C::PAIR ? cluster_ctarank() : 0u;
  // CTA order: groups of group_m token tiles; inside a group the token tile
  // runs fastest, so the CTAs that read one weight tile (and split range)
  // run together and share it through L2, as do the weight tiles of a wave
  // for the group's activation tiles.
  // Two work splits: every tile in `splits` K ranges (tail_splits == 0), or
  // the first head_tiles tiles whole and the remaining (tail) tiles in
  // tail_splits K ranges each, so that the last partial wave of CTAs still
  // spreads over the SMs.  pbase: the partial slot of K range 0 of this
  // tile; cidx: its arrival counter.
  int mtile, nt, split, nsplit, cidx;
  size_t pbase;
  // For a CTA pair every count below is in pair tiles of 256 weight rows
  // (tiles_n / 2 of them); the CTA then takes 128-row tile 2 nt + rank.
  {
    const int b = static_cast<int>(C::PAIR ? blockIdx.x >> 1 : blockIdx.x);
    const int tn = C::PAIR ? args.tiles_n >> 1 : args.tiles_n;
    const int ns = args.tail_splits == 0 ? tn * args.splits : tn;
    int lt = b;  // CTA position in the group order (tail: the tile's)
    if (args.tail_splits == 0) {
      nsplit = args.splits;
    } else if (b < args.head_tiles) {
      nsplit = 1;
    } else {
      const int t = b - args.head_tiles;
      nsplit = args.tail_splits;
      lt = args.head_tiles + t / nsplit;
    }
    const int gsize = args.group_m * ns;
    const int grp = lt / gsize;
    const int gm = min(args.group_m, args.tiles_m - grp * args.group_m);
    const int lin = lt - grp * gsize;
    mtile = grp * args.group_m + lin % gm;
    const int nts = lin / gm;
    if (args.tail_splits == 0) {
      nt = nts / nsplit;
      split = nts % nsplit;
      if (C::PAIR) nt = 2 * nt + static_cast<int>(rank);
      cidx = mtile * args.tiles_n + nt;
      pbase = static_cast<size_t>(cidx) * nsplit;
    } else {
      nt = C::PAIR ? 2 * nts + static_cast<int>(rank) : nts;
      split = b < args.head_tiles ? 0 : (b - args.head_tiles) % nsplit;
      cidx = C::PAIR ? 2 * (lt - args.head_tiles) + static_cast<int>(rank) : lt - args.head_tiles;
      pbase = static_cast<size_t>(cidx) * nsplit;
    }
  }
  const int s0 = static_cast<int>(static_cast<long long>(split) * args.KS / nsplit);
  const int s1 = static_cast<int>(static_cast<long long>(split + 1) * args.KS / nsplit);
  const int nst = s1 - s0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < C::kASlots; ++i) {
      mbar_init(&afull[i], C::PAIR ? 2 * C::kDqWarps : C::kDqWarps);
      mbar_init(&aempty[i], 1);
    }
    mbar_init(accf, 1);
    mbar_init(epi1, C::kDqWarps);
    mbar_init(epi2, 1);
    if (C::PAIR)
      for (int i = 0; i < C::STAGES; ++i) mbar_init(&xfull[i], 1);
    fence_barrier_init();
    grid_dep_launch();  // the next kernel on the stream may start its prologue
  }
  if (C::FMT == kFmtNf4 && threadIdx.x < 16) Ts[threadIdx.x] = level_value(args.table, threadIdx.x);
  // the level addresses need a 256-byte-aligned table (bounds-checked build: verified)
  if (C::FMT == kFmtNf4 && kChecked && threadIdx.x == 0) in_bounds(smem_u32(Ts) & 0xFFu, 1u);
  if (warp == 1) {
    if constexpr (C::PAIR) {
      tmem_alloc_pair(tmem_holder, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  // a pair: the peer's copies and arrivals may target this CTA's barriers
  // as soon as it passes here, so both CTAs' initialisations come first
  if constexpr (C::PAIR)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&xmap);
      const uint64_t pol_w = policy_evict_first();  // weights are read once per M tile
      const uint64_t pol_x = policy_evict_last();   // X is shared by every CTA
      const uint8_t* wsrc =
          args.Wp + (static_cast<size_t>(nt) * args.KS + s0) * C::kWStageBytes;
      // bounds-checked build: a stage outside Wp is flagged and replaced by the
      // first stage (so that the barrier still completes)
      auto stage_src = [&](int it) -> const uint8_t* {
        const unsigned long long off = (static_cast<unsigned long long>(nt) * args.KS + s0 + it) *
                                       C::kWStageBytes;
        return in_bounds(off + C::kWStageBytes - 1, args.wp_bytes)
                   ? wsrc + static_cast<size_t>(it) * C::kWStageBytes
                   : args.Wp;
      };
      // The weights do not depend on the previous kernel: start streaming the
      // first ring's worth before waiting for it, then add the X tiles.
      // full[s] counts this CTA's weight bytes (and for a single CTA its X
      // bytes); a pair's X halves are counted on the leader's xfull[s], which
      // the leader alone arms, with both halves' bytes.
      constexpr uint32_t kFullBytes = C::PAIR ? C::kWStageBytes : C::kXStageBytes + C::kWStageBytes;
      const int first = nst < C::STAGES ? nst : C::STAGES;
      for (int it = 0; it < first; ++it) {
        mbar_arrive_expect_tx(&full[it], kFullBytes);
        bulk_g2s(wsl + it * C::kWSlot, stage_src(it), C::kWStageBytes, &full[it], pol_w);
      }
      grid_dep_wait();
      int issued = 0;
      for (int it = 0; it < nst; ++it) {
        const int s = it % C::STAGES;
        if (it >= C::STAGES) {
          if (!mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1)) break;
          mbar_arrive_expect_tx(&full[s], kFullBytes);
          bulk_g2s(wsl + s * C::kWSlot, stage_src(it), C::kWStageBytes, &full[s], pol_w);
        }
        if constexpr (C::PAIR) {
          if (rank == 0) mbar_arrive_expect_tx(&xfull[s], 2 * C::kXStageBytes);
          tma_load_3d_pair(xs + s * C::kXStageBytes, &xmap, 0,
                           mtile * C::MT + static_cast<int>(rank) * C::kXTok, (s0 + it) * 2,
                           mapa_shared(smem_u32(&xfull[s]), 0), pol_x);
        } else {
          tma_load_3d(xs + s * C::kXStageBytes, &xmap, 0, mtile * C::MT, (s0 + it) * 2,
                      &full[s], pol_x);
        }
        ++issued;
      }
      if (issued < first) {
        // stopped early: the weight copies of the first ring are still counted
        for (int it = issued; it < first; ++it) mbar_wait(&full[it], 0);
      }
      // never leave with copies in flight: wait for the last issued stages
      // (the leader's xfull also covers the peer's halves)
      for (int it = issued - 1; it >= 0 && it >= issued - C::STAGES; --it) {
        mbar_wait(&full[it % C::STAGES], (it / C::STAGES) & 1);
        if (C::PAIR && rank == 0) mbar_wait(&xfull[it % C::STAGES], (it / C::STAGES) & 1);
      }
      // a pair: the leader's MMA completions arrive on this CTA's empty
      // barriers from the other SM; wait for the last ones before leaving
      if (C::PAIR && issued == nst)
        for (int it = nst - 1; it >= 0 && it >= nst - C::STAGES; --it)
          mbar_wait(&empty[it % C::STAGES], (it / C::STAGES) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // (a pair: the leader's thread alone; its MMAs span both CTAs, and each
    // commit arrives on the barrier at the same offset in both)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(C::PAIR ? 256 : 128, C::MT);
      const uint32_t d_tmem = tmem + C::kDCol;
      for (int it = 0; it < nst; ++it) {
        const int s = it % C::STAGES;
        const int a = it % C::kASlots;
        if (!mbar_wait(C::PAIR ? &xfull[s] : &full[s], (it / C::STAGES) & 1)) break;
        if (!mbar_wait(&afull[a], (it / C::kASlots) & 1)) break;
        tc_fence_after();
        const uint32_t xaddr = smem_u32(xs + s * C::kXStageBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc =
              smem_desc_sw128(xaddr + (kk >> 2) * C::kXBoxBytes + (kk & 3) * 32);
          const uint32_t a_tmem = tmem + C::kACol + a * 64 + kk * 8;
          const int acc = kk % C::kAcc;
          if constexpr (C::PAIR)
            mma_bf16_ts_pair(d_tmem, a_tmem, bdesc, idesc, (it > 0 || kk > 0) ? 1u : 0u);
          else
            mma_bf16_ts(d_tmem + acc * C::MT, a_tmem, bdesc, idesc,
                        (it > 0 || kk >= C::kAcc) ? 1u : 0u);
        }
        if constexpr (C::PAIR) {
          mma_commit_pair(&empty[s], kPairCtas);
          mma_commit_pair(&aempty[a], kPairCtas);
        } else {
          mma_commit(&empty[s]);
          mma_commit(&aempty[a]);
        }
      }
      // also on an early exit, so that TMEM is quiet before dealloc
      if constexpr (C::PAIR)
        mma_commit_pair(accf, kPairCtas);
      else
        mma_commit(accf);
    }
  } else {
    // ------------------------------------------------------------ dequant
    // warp (quadrant q, half h) owns TMEM lanes 32q..32q+31 = row groups 2q,
    // 2q+1, and channel blocks 4h..4h+3 of every stage
    const int dw = warp - 2;        // 0..7
    const int quad = warp & 3;      // TMEM lane quadrant this warp may access
    const int h = dw >> 2;          // 64-channel half of each stage
    const int row = quad * 32 + lane;  // accumulator lane owned in the epilogue
    const int n = nt * kTileRows + row;
    const int g = lane >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    for (int it = 0; it < nst && ok; ++it) {
      const int s = it % C::STAGES;
      const int a = it % C::kASlots;
      // warp-uniform waits: the tcgen05 loads/stores below are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (it / C::STAGES) & 1))) {
        ok = false;
        break;
      }
      const uint8_t* wb = wsl + s * C::kWSlot;
      uint32_t out[2][16];
#pragma unroll
      for (int rgl = 0; rgl < 2; ++rgl) {
        const int rg = quad * 2 + rgl;
        const uint4 cw = *reinterpret_cast<const uint4*>(wb + code_word_offset(rg, 4 * h, lane));
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
        if constexpr (C::FMT == kFmtInt4) {
          constexpr int gps = kStageK / C::G;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int gl = ((4 * h + w) * 16) / C::G;
            const uint32_t sp = *reinterpret_cast<const uint32_t*>(wb + scale_pair_offset(rg, gl, g, gps));
            const uint32_t zp = wb[zero_pair_offset(rg, gl, g, gps)];
            // (the compiler merges the loads and parameter math shared by words)
            Int4Dq p0, p1;
            int4_dq_params2(sp, zp, p0, p1);
            int4_dq_word(words[w], p0, p1, &out[rgl][4 * w]);
          }
        } else {
          const int blk_in_row = (s0 + it) * 2 + h;
          const uint32_t cp = *reinterpret_cast<const uint16_t*>(wb + absmax_pair_offset(rg, h, g));
          const int r0 = nt * kTileRows + rg * 16 + g;
          float a0 = 0.0f, a1 = 0.0f;
          if (blk_in_row * 64 < args.K) {
            const long long kb64 = args.K / 64;
            if (r0 < args.N) {
              unsigned long long i0 =
                  fast_div(static_cast<unsigned long long>(r0) * kb64 + blk_in_row, args.by_dq);
              if (!in_bounds(i0, args.s2_count)) i0 = 0;
              a0 = absmax_from_code<C::MEAN>(cp, __ldg(args.s2 + i0),
                                             C::MEAN ? __ldg(args.mean + i0) : 0.0f);
            }
            if (r0 + 8 < args.N) {
              unsigned long long i1 =
                  fast_div(static_cast<unsigned long long>(r0 + 8) * kb64 + blk_in_row, args.by_dq);
              if (!in_bounds(i1, args.s2_count)) i1 = 0;
              a1 = absmax_from_code<C::MEAN>(cp >> 8, __ldg(args.s2 + i1),
                                             C::MEAN ? __ldg(args.mean + i1) : 0.0f);
            }
          }
#pragma unroll
          for (int w = 0; w < 4; ++w) nf4_dq_word(words[w], a0, a1, smem_u32(Ts), &out[rgl][4 * w]);
        }
      }
      if (it >= C::kASlots) {
        if (!__all_sync(0xffffffffu, mbar_wait(&aempty[a], ((it / C::kASlots) - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();  // the MMAs that read this slot are complete
      }
#pragma unroll
      for (int rgl = 0; rgl < 2; ++rgl)
        tmem_st_16x256b_x4(tmem + lane_base + (static_cast<uint32_t>(16 * rgl) << 16) + C::kACol +
                               a * 64 + h * 32,
                           out[rgl]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (C::PAIR)
          mbar_arrive_cluster(mapa_shared(smem_u32(&afull[a]), 0));  // the leader's
        else
          mbar_arrive(&afull[a]);
      }
    }
    // a pair: the last slot releases arrive from the other SM; wait for them
    // before the CTA can leave
    if (C::PAIR && ok)
      for (int it = nst - 1; it >= 0 && it >= nst - C::kASlots; --it)
        mbar_wait(&aempty[it % C::kASlots], (it / C::kASlots) & 1);

    // ------------------------------------------------------------ epilogue
    if (ok && __all_sync(0xffffffffu, mbar_wait(accf, 0))) {
      tc_fence_after();
      grid_dep_wait();  // Y and the workspace may still be in use by the previous kernel
      constexpr int kHalfCols = C::MT / 2;
      const int m_base = mtile * C::MT + h * kHalfCols;
      float* part = args.partial + ((pbase + split) * C::MT + h * kHalfCols) * kTileRows;
      // columns per tensor-memory wait: 32 with one accumulator (every
      // tile of 64 tokens or more), else 8 per accumulator, summed in order
      constexpr int kCw = C::kAcc == 1 && kHalfCols % 32 == 0 ? 32 : 8;
#pragma unroll 1
      for (int cb = 0; cb < kHalfCols; cb += kCw) {
        float sum[kCw];
        if constexpr (kCw == 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + C::kDCol + h * kHalfCols + cb, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) sum[j] = __uint_as_float(v[j]);
        } else {
#pragma unroll
          for (int ai = 0; ai < C::kAcc; ++ai) {
            uint32_t v[8];
            tmem_ld8(tmem + lane_base + C::kDCol + ai * C::MT + h * kHalfCols + cb, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              sum[j] = ai == 0 ? __uint_as_float(v[j]) : sum[j] + __uint_as_float(v[j]);
          }
        }
#pragma unroll
        for (int j = 0; j < kCw; ++j) {
          const int m = m_base + cb + j;
          const float acc = sum[j];
          if (nsplit == 1) {
            if (m < args.M && n < args.N)
              args.Y[static_cast<size_t>(m) * args.N + n] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(acc));
          } else if (in_bounds(static_cast<unsigned long long>(part - args.partial) +
                                   (cb + j) * kTileRows + row,
                               args.partial_floats)) {
            part[(cb + j) * kTileRows + row] = acc;
          }
        }
      }
      tc_fence_before();
      if (nsplit > 1) {
        // the last CTA of this tile to arrive sums the partials in split order
        // (mbarriers with bounded waits, not bar.sync, so that a warp that gave
        // up earlier cannot leave the others blocked)
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(epi1);
        bool have_flag = true;
        if (threadIdx.x == 64) {
          if (mbar_wait(epi1, 0) && in_bounds(cidx, 65536)) {
            const unsigned prev = atomicAdd(args.counter + cidx, 1u);
            *last_flag = (prev == static_cast<unsigned>(nsplit - 1)) ? 1 : 0;
          } else {
            *last_flag = 0;
          }
          mbar_arrive(epi2);
        }
        have_flag = __all_sync(0xffffffffu, mbar_wait(epi2, 0));
        if (have_flag && *last_flag) {
          __threadfence();
          const float* base = args.partial + pbase * C::MT * kTileRows;
          // kCb columns of kSu K ranges at a time: kCb * kSu loads in flight per
          // L2 round trip (one range at a time, a 16-range tile took 128 round
          // trips); the sums are still taken in range order
          constexpr int kCb = kHalfCols < 8 ? kHalfCols : 8;
          constexpr int kSu = 4;
#pragma unroll 1
          for (int c0 = 0; c0 < kHalfCols; c0 += kCb) {
            const int ml0 = h * kHalfCols + c0;
            float acc[kCb];
#pragma unroll
            for (int j = 0; j < kCb; ++j) acc[j] = 0.0f;
#pragma unroll 1
            for (int sp0 = 0; sp0 < nsplit; sp0 += kSu) {
              float v[kSu][kCb];
              bool ok[kSu];
#pragma unroll
              for (int u = 0; u < kSu; ++u) {
                const float* src =
                    base + (static_cast<size_t>(sp0 + u) * C::MT + ml0) * kTileRows + row;
                ok[u] = sp0 + u < nsplit &&
                        in_bounds(static_cast<unsigned long long>(src - args.partial) +
                                      (kCb - 1) * kTileRows,
                                  args.partial_floats);
#pragma unroll
                for (int j = 0; j < kCb; ++j) v[u][j] = ok[u] ? __ldcg(src + j * kTileRows) : 0.0f;
              }
#pragma unroll
              for (int u = 0; u < kSu; ++u)
#pragma unroll
                for (int j = 0; j < kCb; ++j)
                  if (ok[u]) acc[j] += v[u][j];
            }
#pragma unroll
            for (int j = 0; j < kCb; ++j) {
              const int m = mtile * C::MT + ml0 + j;
              if (m < args.M && n < args.N)
                args.Y[static_cast<size_t>(m) * args.N + n] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]));
            }
          }
          if (threadIdx.x == 64) args.counter[cidx] = 0u;  // leave the workspace zeroed
        }
      }
    }
  }

  if constexpr (C::PAIR) {
    // neither CTA of a pair leaves (or frees its tensor memory) while the
    // other may still reach its shared or tensor memory
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
      mbar_wait(accf, 0);  // every issued MMA has completed
      tc_fence_after();
      tmem_dealloc_pair(tmem, C::kTmemCols);
    }
  } else {
    __syncthreads();
    if (warp == 1) {
      mbar_wait(accf, 0);  // every issued MMA has completed
      tc_fence_after();
      tmem_dealloc(tmem, C::kTmemCols);
    }
  }
}

// The activation prologue, run before a GEMM whose X needs rewriting:
//   X'[m, j] = X[m, c],  c = perm[j] with act-order, else c = j,
// and with the AWQ factor s ("大模型量化选型：五种主流方案对比与实战" §4.1:
// the weights are quantized as W s, the activations enter as X / s)
//   X'[m, j] = bf16_rne(fp32(X[m, c]) / s[c])        (IEEE division).
// 8 consecutive outputs per thread (one 16-byte store); K % 8 == 0, X and X'
// 16-byte aligned, s 16-byte aligned.  Without PERM each thread reads only
// the 8 inputs it writes, so X' may be X itself.  The GEMM launched after it
// may start at once (programmatic dependent launch) and stream its weights
// while this runs; it reads X' only after its dependency wait.
template <bool PERM, bool SCALE>
__global__ void __launch_bounds__(256) x_prologue_kernel(const uint16_t* X,
                                                         const int32_t* __restrict__ perm,
                                                         const float* __restrict__ s, int M,
                                                         int K, uint16_t* Xp) {
  grid_dep_launch();
  const size_t k8 = static_cast<size_t>(K) / 8;
  const size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<size_t>(M) * k8) return;
  const size_t m = t / k8;
  const int j0 = static_cast<int>(t - m * k8) * 8;
  const uint16_t* xr = X + m * K;
  uint32_t v[8];
  int c[8];
  if (PERM) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = perm[j0 + e];
      if (!in_bounds(static_cast<unsigned int>(c[e]), static_cast<unsigned int>(K))) c[e] = 0;
      v[e] = xr[c[e]];
    }
  } else {
    const uint4 w = *reinterpret_cast<const uint4*>(xr + j0);
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = j0 + e;
      v[e] = (wv[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
    }
  }
  if (SCALE) {
    float sv[8];
    if (PERM) {
#pragma unroll
      for (int e = 0; e < 8; ++e) sv[e] = s[c[e]];
    } else {
      const float4 a = *reinterpret_cast<const float4*>(s + j0);
      const float4 b = *reinterpret_cast<const float4*>(s + j0 + 4);
      sv[0] = a.x; sv[1] = a.y; sv[2] = a.z; sv[3] = a.w;
      sv[4] = b.x; sv[5] = b.y; sv[6] = b.z; sv[7] = b.w;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float q = __fdiv_rn(__uint_as_float(v[e] << 16), sv[e]);
      v[e] = __bfloat16_as_ushort(__float2bfloat16_rn(q));
    }
  }
  uint4 o;
  o.x = v[0] | (v[1] << 16);
  o.y = v[2] | (v[3] << 16);
  o.z = v[4] | (v[5] << 16);
  o.w = v[6] | (v[7] << 16);
  *reinterpret_cast<uint4*>(Xp + m * K + j0) = o;
}

}  // namespace w4
