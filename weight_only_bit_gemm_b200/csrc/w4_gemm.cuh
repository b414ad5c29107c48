// w4_gemm.cuh -- fused unpack -> dequant -> tcgen05 MMA for the W4A16 / NF4
// linear layer, Y = X . W_hat^T, computed as the swapped product
// Y^T = W_hat . X^T so that the dequantized weight tile is the MMA's A
// operand and lives in tensor memory:
//
//   warp 0      producer: one bulk copy of the prepacked weight stage and two
//               TMA tiles of X per stage into a shared-memory ring
//   warp 1      tensor-memory allocation and the single MMA-issuing thread
//   warps 2..9  dequantize: each thread owns one weight row (TMEM lane) and
//               one 64-channel half of a stage, turns 32 packed bytes into 64
//               bf16 values and writes them to TMEM with tcgen05.st; at the
//               end they read the fp32 accumulator back and store Y (or a
//               split-K partial)
//
// "这不是理论课...LLM量化实操手册" §4.2 measures a separate 4-bit decode +
// dequant kernel next to the cuBLASLt matmul; here the two are one kernel and
// the dequantized tile never leaves the SM.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "w4_prepack.cuh"
#include "w4_ptx.cuh"
#include "w4_quant.cuh"

namespace w4 {

enum WeightFormat : int { kFmtInt4 = 0, kFmtNf4 = 1 };

template <int MT_, int STAGES_, int FMT_, int G_, bool MEAN_ = false, bool PAIR_ = false>
struct GemmCfg {
  static constexpr int MT = MT_;          // tokens per tile (MMA N)
  static constexpr int STAGES = STAGES_;  // shared-memory ring depth
  static constexpr int FMT = FMT_;
  static constexpr int G = G_;            // INT4 group size (ignored for NF4)
  static constexpr bool MEAN = MEAN_;     // NF4 layout: mean-offset absmax constants
  // CTA pair (cluster of 2, cta_group::2): the pair computes 256 weight rows
  // x MT tokens with one MMA stream issued by the even CTA; each CTA holds its
  // 128 weight rows (dequantized into its own tensor memory) and half of the
  // tile's tokens (MT / 2 rows of the activation boxes), so each CTA streams
  // half the activation bytes per MMA of a single-CTA tile.
  static constexpr bool PAIR = PAIR_;
  static constexpr int kXTok = PAIR ? MT / 2 : MT;    // token rows of this CTA's boxes
  static constexpr int kXBoxBytes = kXTok * 128;      // [kXTok][64] bf16, 128-byte rows
  static constexpr int kXStageBytes = 2 * kXBoxBytes;  // 128 channels
  static constexpr int kWStageBytes = FMT == kFmtInt4 ? int4_stage_bytes(G) : nf4_stage_bytes();
  static constexpr int kWSlot = (kWStageBytes + 127) / 128 * 128;
  static constexpr int kASlots = PAIR ? 4 : 3;        // TMEM A ring (64 columns each)
  // Independent accumulators: consecutive MMAs of a stage write different
  // ones, so that narrow (decode) tiles are not serialised on the
  // accumulator dependency; the epilogue sums them in a fixed order.
  static constexpr int kAcc = MT <= 16 ? 4 : MT <= 32 ? 2 : 1;
  static constexpr int kDCol = 0;
  static constexpr int kACol = kAcc * MT;             // A slots after the accumulators
  static constexpr int kColsNeeded = kAcc * MT + kASlots * 64;
  static constexpr int kTmemCols = kColsNeeded <= 32 ? 32
                                   : kColsNeeded <= 64 ? 64
                                   : kColsNeeded <= 128 ? 128
                                   : kColsNeeded <= 256 ? 256 : 512;
  static constexpr int kDqWarps = 8;
  static constexpr int kThreads = 64 + kDqWarps * 32;
  // full, empty (STAGES each), afull, aempty (kASlots each), accf, epi1,
  // epi2, and for a pair xfull (STAGES: the activation halves of both CTAs)
  static constexpr int kNumBars = (PAIR ? 3 : 2) * STAGES + 2 * kASlots + 3;
  static constexpr int kSmemBytes =
      1024 /* alignment slack */ + STAGES * (kXStageBytes + kWSlot) + kNumBars * 8 + 16 + 64 +
      256 /* NF4 level table alignment */;
  static constexpr int kMinBlocks =
      !PAIR && kTmemCols <= 256 && kSmemBytes <= 113 * 1024 ? 2 : 1;
  static_assert(!PAIR || (MT == 256 && kAcc == 1), "CTA pairs: 256-token tiles");
  static_assert(MT % 16 == 0 && MT >= 16 && MT <= 256, "MMA N for M=128 is 16..256 step 16");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(kColsNeeded <= 512, "tensor memory");
};

// bf16x2 arithmetic on 32-bit registers (low half = first element).
__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// (lo, hi) fp32 -> bf16x2, round to nearest even
__device__ __forceinline__ uint32_t bf2_from_f32(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Exact INT4 dequant of one 32-bit word (8 codes, see w4_prepack.cuh):
//   w_hat = bf16_rne((q - z) * s)
// with the fp16 scale s split as s_hi + s_lo, both exact in bf16 (s_lo has at
// most 3 significant bits).  q becomes the bf16 value 128 + q by OR-ing the
// code into the mantissa of 128.0; d = (128+q) - (128+z) is exact; d * s_lo is
// exact (at most 7 significant bits); and one fused multiply-add
// d * s_hi + d * s_lo rounds the exact product d * s once to bf16.
// The three constants are bf16x2 bit patterns with equal halves.
struct Int4Dq {
  uint32_t zm, shi, slo;
};

// The constants of both rows of a lane at once, from the packed fp16 scale
// pair sp = s(r0) | s(r1) << 16 and the zero byte zp = z(r0) | z(r1) << 4.
__device__ __forceinline__ void int4_dq_params2(uint32_t sp, uint32_t zp, Int4Dq& p0, Int4Dq& p1) {
  float s0, s1;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "cvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
      : "=f"(s0), "=f"(s1)
      : "r"(sp));
  p0.shi = bf2_from_f32(s0, s0);
  p1.shi = bf2_from_f32(s1, s1);
  const float l0 = s0 - __uint_as_float(p0.shi << 16);  // exact
  const float l1 = s1 - __uint_as_float(p1.shi << 16);
  p0.slo = bf2_from_f32(l0, l0);
  p1.slo = bf2_from_f32(l1, l1);
  const uint32_t t = zp * 0x00010001u;  // z(r0) at bits 0 and 16, z(r1) at 4 and 20
  p0.zm = (t & 0x000F000Fu) | 0x43004300u;
  p1.zm = ((t >> 4) & 0x000F000Fu) | 0x43004300u;
}

// Pairs 0 and 1 of the word belong to row r0 (params p0), pairs 2 and 3 to
// row r1 (params p1).  One asm block, so that each pair costs exactly one
// LOP3 (plus one shift for pairs 1..3) and three bf16x2 instructions.
__device__ __forceinline__ void int4_dq_word(uint32_t w, const Int4Dq& p0, const Int4Dq& p1,
                                             uint32_t* out) {
  const uint32_t mask = 0x000F000Fu, magic = 0x43004300u;
  asm("{\n\t.reg .b32 t0, t1, t2, t3, d0, d1, d2, d3, l0, l1, l2, l3;\n\t"
      "lop3.b32 t0, %4, %5, %6, 0xEA;\n\t"
      "shr.b32 t1, %4, 4;\n\t"
      "lop3.b32 t1, t1, %5, %6, 0xEA;\n\t"
      "shr.b32 t2, %4, 8;\n\t"
      "lop3.b32 t2, t2, %5, %6, 0xEA;\n\t"
      "shr.b32 t3, %4, 12;\n\t"
      "lop3.b32 t3, t3, %5, %6, 0xEA;\n\t"
      "sub.rn.bf16x2 d0, t0, %7;\n\t"
      "sub.rn.bf16x2 d1, t1, %7;\n\t"
      "sub.rn.bf16x2 d2, t2, %10;\n\t"
      "sub.rn.bf16x2 d3, t3, %10;\n\t"
      "mul.rn.bf16x2 l0, d0, %9;\n\t"
      "mul.rn.bf16x2 l1, d1, %9;\n\t"
      "mul.rn.bf16x2 l2, d2, %12;\n\t"
      "mul.rn.bf16x2 l3, d3, %12;\n\t"
      "fma.rn.bf16x2 %0, d0, %8, l0;\n\t"
      "fma.rn.bf16x2 %1, d1, %8, l1;\n\t"
      "fma.rn.bf16x2 %2, d2, %11, l2;\n\t"
      "fma.rn.bf16x2 %3, d3, %11, l3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w), "r"(mask), "r"(magic), "r"(p0.zm), "r"(p0.shi), "r"(p0.slo), "r"(p1.zm),
        "r"(p1.shi), "r"(p1.slo));
}

// NF4 dequant of one word: w_hat = bf16_rne(fp32(T[q] * a')), with the 16
// levels T in shared memory at the 256-byte-aligned shared address tb (so
// that a level's address is tb with its low byte replaced by 4q), a0 / a1 the
// reconstructed absmax of rows r0 / r1.  One asm block: two shift + mask
// pairs put 4q of all eight codes into the bytes of two registers (t0: codes
// 0, 2, 4, 6; t1: codes 1, 3, 5, 7), one byte permute per code makes its
// address; then one shared load and one fp32 multiply per code and one
// conversion per pair.  The pairs are (code i, code i + 4), i = 0..3, as the
// prepacked layout orders them for the MMA fragment.
__device__ __forceinline__ void nf4_dq_word(uint32_t w, float a0, float a1, uint32_t tb,
                                            uint32_t* out) {
  asm("{\n\t.reg .b32 t0, t1, o0, o1, o2, o3, o4, o5, o6, o7;\n\t"
      ".reg .f32 v0, v1, v2, v3, v4, v5, v6, v7;\n\t"
      "shl.b32 t0, %4, 2;\n\t  and.b32 t0, t0, 0x3C3C3C3C;\n\t"
      "shr.b32 t1, %4, 2;\n\t  and.b32 t1, t1, 0x3C3C3C3C;\n\t"
      "prmt.b32 o0, t0, %7, 0x7650;\n\t prmt.b32 o1, t0, %7, 0x7652;\n\t"
      "prmt.b32 o2, t1, %7, 0x7650;\n\t prmt.b32 o3, t1, %7, 0x7652;\n\t"
      "prmt.b32 o4, t0, %7, 0x7651;\n\t prmt.b32 o5, t0, %7, 0x7653;\n\t"
      "prmt.b32 o6, t1, %7, 0x7651;\n\t prmt.b32 o7, t1, %7, 0x7653;\n\t"
      "ld.shared.f32 v0, [o0];\n\t ld.shared.f32 v1, [o1];\n\t"
      "ld.shared.f32 v2, [o2];\n\t ld.shared.f32 v3, [o3];\n\t"
      "ld.shared.f32 v4, [o4];\n\t ld.shared.f32 v5, [o5];\n\t"
      "ld.shared.f32 v6, [o6];\n\t ld.shared.f32 v7, [o7];\n\t"
      "mul.rn.f32 v0, v0, %5;\n\t mul.rn.f32 v1, v1, %5;\n\t"
      "mul.rn.f32 v2, v2, %5;\n\t mul.rn.f32 v3, v3, %5;\n\t"
      "mul.rn.f32 v4, v4, %6;\n\t mul.rn.f32 v5, v5, %6;\n\t"
      "mul.rn.f32 v6, v6, %6;\n\t mul.rn.f32 v7, v7, %6;\n\t"
      "cvt.rn.bf16x2.f32 %0, v1, v0;\n\t"
      "cvt.rn.bf16x2.f32 %1, v3, v2;\n\t"
      "cvt.rn.bf16x2.f32 %2, v5, v4;\n\t"
      "cvt.rn.bf16x2.f32 %3, v7, v6;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w), "f"(a0), "f"(a1), "r"(tb)
      : "memory");
}

struct GemmArgs {
  const uint8_t* Wp;      // prepacked weights (tiles x stages blocks)
  const float* s2;        // NF4 second-level scales (NF4 only)
  const float* mean;      // NF4 mean-offset double quantization: run means
  uint16_t* Y;            // bf16 [M, N]
  float* partial;         // split-K partials [tile][split][MT][128]
  unsigned int* counter;  // split-K arrival counters [tile]
  int M, N, K;
  int KS;                 // stages per tile row = ceil(K / 128)
  int tiles_n;
  int splits;             // K ranges of every tile (tail_splits == 0)
  int head_tiles;         // tail_splits > 0: tiles (in CTA order) computed whole,
  int tail_splits;        //   then each remaining tile in tail_splits K ranges
  int tiles_m;            // token tiles
  int group_m;            // token tiles per group of the CTA order (see the kernel)
  FastDivIdx by_dq;        // NF4: 64-block index -> s2 index (double-quant run)
  int table;              // NF4 layout: level table (kTableNf4 / kTableFp4)
  // buffer extents, read only by the bounds-checked build
  unsigned long long wp_bytes, partial_floats, s2_count;
};

}  // namespace w4
