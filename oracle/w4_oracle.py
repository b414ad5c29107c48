"""Oracle: group-wise INT4 (asymmetric and symmetric RTN, GPTQ) and NF4 / FP4
(block-wise, double-quantized) weight quantization, the LLM.int8 mixed
decomposition, the AWQ per-input-channel factor,
packing, dequantization and the fp64 matmul reference.

TEST INFRASTRUCTURE ONLY -- see the package docstring for who may import it.

Page titles cited below (the five source pages):

* [Survey]     "大模型量化选型：五种主流方案对比与实战"
* [Primer]     the aicoding.csdn.net primer whose first heading is
               "一、量化究竟做了什么"
* [Handbook]   "这不是理论课，是能立刻上手的LLM量化实操手册"
* [Guide]      "开源模型量化实战指南：GGUF、GPTQ、AWQ选型与本地部署"
* [Comparison] "【推理与部署篇05】模型量化部署深度对比：GPTQ、AWQ、GGUF与FP8实战指南"

Readings taken where the pages leave a step open (each is listed, with its
reason, in the design notes):

R1  the group range includes 0 (``mn = min(min w, 0)``, ``mx = max(max w, 0)``)
    so that the zero point always fits in 4 bits;
R2  the scale is stored in fp16 and every later step uses the fp16 value; a
    zero scale becomes 1.0;
R3  "round" is round-half-to-even (``numpy.rint``);
R4  nibble order: even k in the low nibble of byte k // 2;
R5  the dequantized weight is the bf16 (round-to-nearest-even) of the exact
    fp32 product ``(q - zp) * scale``;
R6  NF4 levels are the normal-quantile construction with an exact zero
    (8 positive, 7 negative quantiles, normalised to [-1, 1]);
R7  an NF4 value on a midpoint takes the lower code;
R8  double quantization: per run of 256 consecutive blocks,
    ``s2 = max(absmax) / 255``, ``c = rint(absmax / s2)`` in [0, 255],
    ``absmax' = c * s2`` in fp32; codes are chosen with the unquantized absmax;
R9  NF4 dequant is ``bf16(fp32(T[q] * absmax'))``;
R20 mean-offset double quantization (the variant of R8): per run, the mean
    of the constants (fp64 sum in block order, one rounding to fp32) is
    subtracted and the residuals take the symmetric 8-bit formula
    (``max|d| / 127``, codes in [-127, 127]); ``absmax' = fp32(c * s2) + mean``;
R14 symmetric INT4: ``scale = fp16(max|w| / 7)``, codes ``rint(w / scale)``
    clamped to [-7, 7] and stored + 8 (zero point 8, code 0 unused);
R15 AWQ: the factor s is an input (found offline); weights enter
    quantization as the fp32 product ``w * s_k``, activations the GEMM as
    ``bf16(fp32(x / s_k))``;
R17 FP4: E2M1 codes (sign bit 3, exponent bits 2..1, mantissa bit 0) with
    magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 divided by 6; nearest magnitude,
    the lower on a midpoint; sign bit only for a nonzero magnitude; blocks,
    double quantization and dequantization as NF4;
R18 GPTQ: H = 2 X^T X (fp64); dead channels H_kk = 0 -> 1 and w_k = 0;
    act-order = stable sort by decreasing H_kk; damping 0.01 * mean(diag H);
    the update uses the inverse Hessian of the remaining columns, eliminated
    one column at a time; group parameters from the compensated weights at
    the group's first column; codes decided in fp32;
R19 LLM.int8: per-row weight absmax/127, outlier channels |x| > 6.0 in any
    token of the call, per-token activation absmax/127 over the other
    channels, exact INT8 sum scaled by s_x s_w plus the outlier channels'
    product with bf16 dequantized INT8 weights.

All floating-point steps are numpy float32 operations (IEEE, round to nearest
even) unless stated as fp64; the matmul accumulates in fp64.

NF4 levels: the pages print no table.  The tests pin what the pages fix (16
levels, strictly increasing, an exact zero, -1 and +1 at the ends, spacing
smallest near zero) and, to one fp32 ulp, the digits of R6's construction
against an independent fp64 evaluation of it (bisection on the normal CDF
written through erfc, not the library inverse CDF used here).  Agreement
with any NF4 table published elsewhere is not claimed.
"""
from __future__ import annotations

import math
import statistics
from fractions import Fraction

import numpy as np

__all__ = [
    "bf16_round_bits", "bf16_bits_to_f64", "bf16_bits_to_f32",
    "group_index", "rtn_params", "quantize_rtn", "pack_nibbles", "unpack_nibbles",
    "dequant_rtn_f32", "dequant_rtn", "nf4_table", "nf4_midpoints", "nf4_absmax",
    "nf4_codes", "nf4_double_quant", "nf4_quantize", "nf4_dequant", "matmul_ref",
    "nf4_double_quant_mean", "nf4_absmax_mean_dequant", "nf4_quantize_meandq",
    "nf4_dequant_meandq",
    "matmul_exact_small", "ulp_bf16", "tolerance", "check_matmul",
    "weight_bytes", "code_bytes", "nf4_weight_bytes",
    "sym_params", "quantize_sym", "awq_scale_weights", "awq_scale_activations",
    "fp4_table", "fp4_midpoints", "fp4_codes", "fp4_quantize", "fp4_dequant",
    "gptq_hessian", "gptq_prepare", "gptq_eliminate", "gptq_quantize", "gptq_loss",
    "int8_quantize_weights", "int8_outliers", "int8_quantize_activations", "int8_mixed_ref",
]

F32 = np.float32


# ---------------------------------------------------------------------------
# bf16 rounding (R5): keep the top 16 bits of the fp32 pattern, rounding the
# discarded low 16 bits to nearest, ties to the even result.
# ---------------------------------------------------------------------------

def bf16_round_bits(f: np.ndarray) -> np.ndarray:
    """fp32 values -> bf16 bit patterns (uint16), round to nearest even.

    Finite inputs only (no NaN handling is needed: the path never produces
    NaN from finite inputs)."""
    u = np.ascontiguousarray(f, dtype=F32).view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = (u + np.uint64(0x7FFF) + keep_lsb) >> np.uint64(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(F32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


# ---------------------------------------------------------------------------
# INT4 asymmetric round-to-nearest, group-wise along K.
# [Comparison] §2.3 gives the asymmetric min-max formulas for 8 bits
# (scale = (max - min)/255, zero_point = round(-min/scale), range [0, 255]);
# with 4 bits the denominator is 2^4 - 1 = 15 and the range is [0, 15].
# [Comparison] §2.2 and [Primer] §二 give per-group granularity (one scale per
# group of G weights, G = 128/64/32); [Primer] §四 names plain rounding (RTN).
# ---------------------------------------------------------------------------

def group_index(K: int, G: int, g_idx: np.ndarray | None) -> np.ndarray:
    """Group id of every input channel k.  Without act-order the groups are the
    contiguous runs [gG, (g+1)G); with act-order ([Survey] §3.2 desc_act,
    [Guide] §3.2: inference must reorder) channel k belongs to g_idx[k]."""
    if K % G:
        raise ValueError("K must be a multiple of G")
    if g_idx is None:
        return np.arange(K, dtype=np.int64) // G
    g = np.asarray(g_idx).astype(np.int64)
    if g.shape != (K,):
        raise ValueError("g_idx must have shape [K]")
    if g.size and (g.min() < 0 or g.max() >= K // G):
        raise ValueError("g_idx values must lie in [0, K/G)")
    return g


def _group_minmax(W: np.ndarray, G: int, gk: np.ndarray, contiguous: bool):
    N, K = W.shape
    ng = K // G
    if contiguous:
        Wg = W.reshape(N, ng, G)
        return Wg.min(axis=2), Wg.max(axis=2)
    mn = np.zeros((N, ng), F32)
    mx = np.zeros((N, ng), F32)
    for g in range(ng):
        cols = np.nonzero(gk == g)[0]
        if cols.size:
            sub = W[:, cols]
            mn[:, g] = sub.min(axis=1)
            mx[:, g] = sub.max(axis=1)
    return mn, mx


def rtn_params(W: np.ndarray, G: int, g_idx: np.ndarray | None = None):
    """Per (row, group) fp16 scale and zero point (R1, R2, R3).

    Returns (scale_fp16 [N, K/G], zero_uint8 [N, K/G])."""
    W = np.ascontiguousarray(W, dtype=F32)
    N, K = W.shape
    gk = group_index(K, G, g_idx)
    mn, mx = _group_minmax(W, G, gk, g_idx is None)
    mn = np.minimum(mn, F32(0))                      # R1
    mx = np.maximum(mx, F32(0))
    s32 = (mx - mn) / F32(15.0)                      # scale = (max - min) / (2^4 - 1)
    s16 = s32.astype(np.float16)                     # R2: stored fp16 (round to nearest even)
    s16[s16 == 0] = np.float16(1.0)
    sf = s16.astype(F32)
    zp = np.clip(np.rint(-mn / sf), 0, 15)           # zero_point = round(-min / scale)
    return s16, zp.astype(np.uint8)


def quantize_rtn(W: np.ndarray, G: int, g_idx: np.ndarray | None = None):
    """Codes q = clamp(round(w / scale) + zp, 0, 15) (one uint8 per weight).

    Returns (codes uint8 [N, K], scale fp16 [N, K/G], zero uint8 [N, K/G])."""
    W = np.ascontiguousarray(W, dtype=F32)
    N, K = W.shape
    gk = group_index(K, G, g_idx)
    s16, zp = rtn_params(W, G, g_idx)
    sk = s16.astype(F32)[:, gk]
    zk = zp.astype(F32)[:, gk]
    q = np.clip(np.rint(W / sk) + zk, 0, 15)
    return q.astype(np.uint8), s16, zp


# ---------------------------------------------------------------------------
# Symmetric (absmax) quantization.  [Comparison] §2.3 gives the symmetric form
# for 8 bits: scale = max|w| / 127, values in [-127, 127]; [Survey] §1's worked
# example divides a maximum of 80 by 127.  With b bits the levels are
# [-(2^(b-1) - 1), 2^(b-1) - 1].  For b = 4 the code stored is q + 8 in
# [1, 15] with zero point 8, the same canonical format as asymmetric RTN, so
# dequant and the GEMM take it unchanged.  Readings: the scale is stored in
# fp16 like the asymmetric one (R2), a zero scale becomes 1.0, round half to
# even (R3).
# ---------------------------------------------------------------------------

def sym_params(W: np.ndarray, G: int, g_idx: np.ndarray | None = None, bits: int = 4):
    """Per (row, group) fp32 scale max|w| / (2^(bits-1) - 1) and its fp16 value.

    Returns (scale_fp32 [N, K/G], scale_fp16 [N, K/G])."""
    W = np.ascontiguousarray(W, dtype=F32)
    N, K = W.shape
    gk = group_index(K, G, g_idx)
    mn, mx = _group_minmax(W, G, gk, g_idx is None)
    amax = np.maximum(np.abs(mn), np.abs(mx))
    qmax = F32(2 ** (bits - 1) - 1)
    s32 = amax / qmax
    s16 = s32.astype(np.float16)
    s16[s16 == 0] = np.float16(1.0)
    return s32, s16


def quantize_sym(W: np.ndarray, G: int, g_idx: np.ndarray | None = None):
    """4-bit symmetric codes: q = clamp(round(w / scale), -7, 7), stored q + 8.

    Returns (codes uint8 [N, K] in [1, 15], scale fp16 [N, K/G], zero uint8
    [N, K/G] = 8)."""
    W = np.ascontiguousarray(W, dtype=F32)
    N, K = W.shape
    gk = group_index(K, G, g_idx)
    _, s16 = sym_params(W, G, g_idx, 4)
    sk = s16.astype(F32)[:, gk]
    q = np.clip(np.rint(W / sk), -7, 7) + 8
    return q.astype(np.uint8), s16, np.full(s16.shape, 8, np.uint8)


# ---------------------------------------------------------------------------
# AWQ per-input-channel factor.  [Survey] §4.1 and [Comparison] §4.1: the
# weights are quantized as W * s (a factor s_k > 0 per input channel, found
# offline) and the activations enter as X / s, so (X / s)(W s)^T = X W^T
# before quantization; the runtime is the same W4A16 GEMM.  Readings: W * s is
# an fp32 product, X / s an fp32 division of the bf16 value, each rounded to
# nearest even (the latter then to bf16).
# ---------------------------------------------------------------------------

def awq_scale_weights(W: np.ndarray, s: np.ndarray) -> np.ndarray:
    """W[n, k] * s[k] in fp32."""
    return (np.asarray(W, dtype=F32) * np.asarray(s, dtype=F32)[None, :]).astype(F32)


def awq_scale_activations(x_bits: np.ndarray, s: np.ndarray) -> np.ndarray:
    """bf16 bits of fp32(x[m, k] / s[k])."""
    x = bf16_bits_to_f32(x_bits)
    return bf16_round_bits((x / np.asarray(s, dtype=F32)[None, :]).astype(F32))


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte, even k in the low nibble (R4); [Guide] §1.1:
    an INT4 value takes half a byte."""
    c = np.asarray(codes, dtype=np.uint8)
    if c.shape[-1] % 2:
        raise ValueError("K must be even")
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def dequant_rtn_f32(Wq: np.ndarray, scales: np.ndarray, zeros: np.ndarray, G: int,
                    g_idx: np.ndarray | None = None) -> np.ndarray:
    """Exact fp32 value (q - zp) * scale before the bf16 rounding.  The product
    of a |q - zp| <= 15 integer and an 11-bit fp16 significand is exact in fp32."""
    q = unpack_nibbles(Wq).astype(F32)
    K = q.shape[1]
    gk = group_index(K, G, g_idx)
    sk = np.asarray(scales, dtype=np.float16).astype(F32)[:, gk]
    zk = np.asarray(zeros, dtype=np.uint8).astype(F32)[:, gk]
    return (q - zk) * sk


def dequant_rtn(Wq, scales, zeros, G, g_idx=None) -> np.ndarray:
    """Dequantized weight as bf16 bits [N, K] (R5); the pages dequantize to the
    bf16 compute dtype before the matmul ([Survey] §6.2, [Primer] §七)."""
    return bf16_round_bits(dequant_rtn_f32(Wq, scales, zeros, G, g_idx))


# ---------------------------------------------------------------------------
# NF4.  [Survey] §6.1: 16 levels placed at quantiles of the normal
# distribution, denser near zero; [Comparison] §6.2: non-uniform, follows the
# normal CDF; [Survey] §6.3: block-wise, one scale per 64 weights by default;
# [Survey] §6.2 and [Comparison] §6.1: double quantization of the scales.
# ---------------------------------------------------------------------------

def nf4_table() -> np.ndarray:
    """16 NF4 levels (R6), evaluated in fp64, rounded once to fp32.

    Quantile points: delta = 1 - (1/30 + 1/32)/2.  Eight positive levels at
    the first 8 of 9 equally spaced probabilities from delta down to 1/2,
    seven negative levels (mirrored) at the first 7 of 8 such probabilities,
    plus an exact zero; divided by the largest level so the table spans
    [-1, 1]."""
    nd = statistics.NormalDist()
    delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    pos = [nd.inv_cdf(delta + (0.5 - delta) * i / 8.0) for i in range(8)]
    neg = [-nd.inv_cdf(delta + (0.5 - delta) * i / 7.0) for i in range(7)]
    levels = sorted(neg + [0.0] + pos)
    top = nd.inv_cdf(delta)
    return np.array([v / top for v in levels], dtype=np.float64).astype(F32)


def nf4_midpoints() -> np.ndarray:
    """Decision thresholds t_i = fp32((T[i] + T[i+1]) / 2), i = 0..14."""
    T = nf4_table().astype(np.float64)
    return ((T[:-1] + T[1:]) / 2.0).astype(F32)


def _blocks(W: np.ndarray, blocksize: int) -> np.ndarray:
    flat = np.ascontiguousarray(W, dtype=F32).reshape(-1)
    if flat.size % blocksize:
        raise ValueError("N*K must be a multiple of the block size")
    return flat.reshape(-1, blocksize)


def nf4_absmax(W: np.ndarray, blocksize: int = 64) -> np.ndarray:
    """fp32 absmax of each block of `blocksize` consecutive row-major weights."""
    return np.abs(_blocks(W, blocksize)).max(axis=1)


def nf4_codes(W: np.ndarray, blocksize: int = 64) -> np.ndarray:
    """Code of each weight: v = w / absmax (fp32 divide; 0 if absmax is 0),
    q = number of thresholds t_i with v > t_i (R7).  Returns uint8 [N, K]."""
    B = _blocks(W, blocksize)
    a = np.abs(B).max(axis=1)
    safe = np.where(a > 0, a, F32(1.0)).astype(F32)
    v = np.where(a[:, None] > 0, B / safe[:, None], F32(0.0)).astype(F32)
    q = np.searchsorted(nf4_midpoints(), v, side="left")   # count of t_i < v
    return q.astype(np.uint8).reshape(np.shape(W))


def nf4_double_quant(absmax: np.ndarray, dq_group: int = 256):
    """R8: returns (c uint8 [nblocks], s2 fp32 [ceil(nblocks/dq_group)])."""
    a = np.asarray(absmax, dtype=F32)
    nb = a.size
    nruns = (nb + dq_group - 1) // dq_group
    c = np.empty(nb, np.uint8)
    s2 = np.empty(nruns, F32)
    for r in range(nruns):
        run = a[r * dq_group:(r + 1) * dq_group]
        s = run.max() / F32(255.0)
        if s == 0:
            s = F32(1.0)
        s2[r] = s
        c[r * dq_group:(r + 1) * dq_group] = np.clip(np.rint(run / s), 0, 255).astype(np.uint8)
    return c, s2


def nf4_quantize(W: np.ndarray, blocksize: int = 64, dq_group: int = 256):
    """Returns (packed codes uint8 [N, K/2], absmax codes uint8 [N*K/blocksize],
    s2 fp32 [ceil(N*K/blocksize/dq_group)])."""
    q = nf4_codes(W, blocksize)
    c, s2 = nf4_double_quant(nf4_absmax(W, blocksize), dq_group)
    return pack_nibbles(q), c, s2


def nf4_dequant(Wq: np.ndarray, absmax_q: np.ndarray, s2: np.ndarray,
                blocksize: int = 64, dq_group: int = 256) -> np.ndarray:
    """R9: bf16 bits [N, K] of fp32(T[q] * absmax'), absmax' = fp32(c * s2)."""
    q = unpack_nibbles(Wq)
    shape = q.shape
    qb = q.reshape(-1, blocksize)
    nb = qb.shape[0]
    c = np.asarray(absmax_q, dtype=np.uint8)[:nb].astype(F32)
    s = np.asarray(s2, dtype=F32)[np.arange(nb) // dq_group]
    a_dq = c * s                                              # fp32 product
    vals = nf4_table()[qb] * a_dq[:, None]                    # fp32 product
    return bf16_round_bits(vals.reshape(shape))


# ---------------------------------------------------------------------------
# R20: mean-offset double quantization of the NF4 block constants.
# [Survey] §6.2 and [Primer] §七: the per-block absmax constants are
# quantized a second time to save memory; [Comparison] §6 names the switch
# (bnb_4bit_use_double_quant).  The pages do not say how.  This variant
# centres each run of dq_group constants on the run's mean before the second
# quantization, so that the 8 bits cover the spread of the constants rather
# than their whole range, and stores the residuals with the pages' own
# symmetric 8-bit formula ([Comparison] §2.3: scale = max|x| / 127,
# q = round(x / scale) in [-127, 127]).  Per run the mean and the scale are
# kept in fp32.  Codes of the weights are still chosen with the unquantized
# absmax (as in R8).
# ---------------------------------------------------------------------------

def nf4_double_quant_mean(absmax: np.ndarray, dq_group: int = 256):
    """R20: returns (c int8 [nblocks], mean fp32 [runs], s2 fp32 [runs]).

    Per run of dq_group consecutive blocks (the last run may be shorter):
      mean = fp32(S / n), S the fp64 sum of the run's fp32 constants added
             in block order, n the number of blocks in the run;
      d    = fp32(a - mean);
      s2   = fp32(max |d| / 127), 1 if that is 0;
      c    = clamp(rint(d / s2), -127, 127) (fp32 divide)."""
    a = np.asarray(absmax, dtype=F32)
    nb = a.size
    nruns = (nb + dq_group - 1) // dq_group
    c = np.empty(nb, np.int8)
    mean = np.empty(nruns, F32)
    s2 = np.empty(nruns, F32)
    for r in range(nruns):
        run = a[r * dq_group:(r + 1) * dq_group]
        total = 0.0                                   # Python float: fp64
        for v in run:
            total += float(v)
        mu = F32(total / len(run))
        d = (run - mu).astype(F32)
        s = F32(np.abs(d).max() / F32(127.0))
        if s == 0:
            s = F32(1.0)
        mean[r] = mu
        s2[r] = s
        c[r * dq_group:(r + 1) * dq_group] = np.clip(np.rint(d / s), -127, 127).astype(np.int8)
    return c, mean, s2


def nf4_absmax_mean_dequant(c: np.ndarray, mean: np.ndarray, s2: np.ndarray,
                            dq_group: int = 256) -> np.ndarray:
    """R20: absmax' = fp32(fp32(c * s2) + mean), per block (fp32 [nblocks])."""
    cc = np.asarray(c, dtype=np.int8).astype(F32)
    run = np.arange(cc.size) // dq_group
    prod = (cc * np.asarray(s2, F32)[run]).astype(F32)          # fp32 product
    return (prod + np.asarray(mean, F32)[run]).astype(F32)      # fp32 sum


def nf4_quantize_meandq(W: np.ndarray, blocksize: int = 64, dq_group: int = 256):
    """NF4 with R20 constants.  Returns (packed codes uint8 [N, K/2],
    absmax codes int8 [N*K/blocksize], mean fp32 [runs], s2 fp32 [runs])."""
    q = nf4_codes(W, blocksize)
    c, mean, s2 = nf4_double_quant_mean(nf4_absmax(W, blocksize), dq_group)
    return pack_nibbles(q), c, mean, s2


def nf4_dequant_meandq(Wq: np.ndarray, absmax_q: np.ndarray, mean: np.ndarray,
                       s2: np.ndarray, blocksize: int = 64, dq_group: int = 256) -> np.ndarray:
    """R9 with R20 constants: bf16 bits [N, K] of fp32(T[q] * absmax')."""
    q = unpack_nibbles(Wq)
    shape = q.shape
    qb = q.reshape(-1, blocksize)
    nb = qb.shape[0]
    a_dq = nf4_absmax_mean_dequant(np.asarray(absmax_q)[:nb], mean, s2, dq_group)
    vals = nf4_table()[qb] * a_dq[:, None]                    # fp32 product
    return bf16_round_bits(vals.reshape(shape))


# ---------------------------------------------------------------------------
# FP4: the other 4-bit type of the same block-wise scheme.  [Survey] §6.3
# names NF4 and FP4 as the two 4-bit formats of that scheme; [Survey] §6.1
# says plain FP4 keeps three significant bits with uneven spacing;
# [Comparison] §7.2 gives the 4-bit float layout [S:1][E:2][M:1] (E2M1).
# Readings (R17): code bit 3 is the sign, bits 2..1 the exponent e, bit 0
# the mantissa m; magnitude m/2 for e = 0, else 2^(e-1) (1 + m/2), i.e.
# 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7; the table is divided by 6 so
# that it spans [-1, 1] like NF4's and the block absmax maps to code 7.  A
# value takes the nearest magnitude (the lower one on a midpoint) and the
# sign bit only when that magnitude is not zero.  Blocks, double
# quantization and dequantization are NF4's (R8, R9) with this table.
# ---------------------------------------------------------------------------

def fp4_table() -> np.ndarray:
    """16 FP4 levels, fp32: code c -> sign * magnitude(e, m) / 6 (R17), each
    the single fp32 rounding of an exact quotient."""
    out = np.empty(16, dtype=F32)
    for c in range(16):
        e, m = (c >> 1) & 3, c & 1
        mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1.0 + 0.5 * m)   # exact in fp32
        v = F32(mag) / F32(6.0)
        out[c] = -v if c & 8 else v
    return out


def fp4_midpoints() -> np.ndarray:
    """Magnitude thresholds t_i = fp32((T[i] + T[i+1]) / 2), i = 0..6, over
    the ascending positive levels T[0..7]."""
    T = fp4_table()[:8].astype(np.float64)
    return ((T[:-1] + T[1:]) / 2.0).astype(F32)


def fp4_codes(W: np.ndarray, blocksize: int = 64) -> np.ndarray:
    """Code of each weight: v = w / absmax (fp32; 0 if absmax is 0),
    magnitude code = number of thresholds below |v|, plus 8 when v < 0 and
    that magnitude is not zero.  Returns uint8 [N, K]."""
    B = _blocks(W, blocksize)
    a = np.abs(B).max(axis=1)
    safe = np.where(a > 0, a, F32(1.0)).astype(F32)
    v = np.where(a[:, None] > 0, B / safe[:, None], F32(0.0)).astype(F32)
    mag = np.searchsorted(fp4_midpoints(), np.abs(v), side="left")
    q = np.where((v < 0) & (mag > 0), mag + 8, mag)
    return q.astype(np.uint8).reshape(np.shape(W))


def fp4_quantize(W: np.ndarray, blocksize: int = 64, dq_group: int = 256):
    """As nf4_quantize with the FP4 codes: (packed codes, absmax codes, s2)."""
    q = fp4_codes(W, blocksize)
    c, s2 = nf4_double_quant(nf4_absmax(W, blocksize), dq_group)
    return pack_nibbles(q), c, s2


def fp4_dequant(Wq: np.ndarray, absmax_q: np.ndarray, s2: np.ndarray,
                blocksize: int = 64, dq_group: int = 256) -> np.ndarray:
    """bf16 bits [N, K] of fp32(T_fp4[q] * absmax'), absmax' = fp32(c * s2)."""
    q = unpack_nibbles(Wq)
    shape = q.shape
    qb = q.reshape(-1, blocksize)
    nb = qb.shape[0]
    c = np.asarray(absmax_q, dtype=np.uint8)[:nb].astype(F32)
    s = np.asarray(s2, dtype=F32)[np.arange(nb) // dq_group]
    a_dq = c * s                                              # fp32 product
    vals = fp4_table()[qb] * a_dq[:, None]                    # fp32 product
    return bf16_round_bits(vals.reshape(shape))


# ---------------------------------------------------------------------------
# GPTQ error compensation at quantization time.  [Comparison] §3.1: per layer,
# H = 2 X X^T from calibration activations; Q = W; for each column in turn
# (by importance): quantize it, take the error, spread it over the columns not
# yet quantized through the (inverse) Hessian, "remaining -= err / H_diag *
# H_row".  [Survey] §3 (GPTQ): this is the Optimal Brain Surgeon update, it
# needs the inverse of H, and a small damping (percdamp, 0.01) is added to
# H's diagonal so that it stays invertible.  [Survey] §3.2: desc_act orders
# the columns by activation size; group_size 128 shares one scale and zero
# point per group.  Readings (R18):
#   H = 2 X^T X in fp64 for X [n, K] (rows = calibration tokens);
#   a channel with H_kk = 0 (never activated) gets H_kk = 1 and w_k = 0;
#   act-order = a stable sort of the channels by decreasing H_kk;
#   damping H += lambda I, lambda = 0.01 * mean(diag H);
#   "H_diag" and "H_row" are those of the inverse Hessian of the columns not
#   yet quantized: Hi = H^-1, and after column j, Hi loses row and column j
#   by Gaussian elimination (Hi_F <- Hi_F - Hi_Fj Hi_jF / Hi_jj, which is
#   the inverse of H restricted to the remaining columns);
#   a group's scale and zero point come from its (already compensated)
#   weights when its first column is reached, by the RTN rule (R1-R3) on
#   their fp32 values; codes are decided in fp32; the error uses the fp32
#   dequantized value (q - z) * scale; the compensation runs in fp64.
# ---------------------------------------------------------------------------

def gptq_hessian(x_bits: np.ndarray) -> np.ndarray:
    """H = 2 X^T X in fp64 for bf16 calibration activations X [n, K]."""
    x = bf16_bits_to_f64(x_bits)
    return 2.0 * (x.T @ x)


def gptq_prepare(H: np.ndarray, act_order: bool, damp: float = 0.01):
    """Dead channels, order and damping (R18).  Returns (H' fp64 in the
    processing order, perm int64 [K] = processing position -> channel, dead
    bool [K])."""
    H = np.array(H, dtype=np.float64, copy=True)
    K = H.shape[0]
    d = np.diag(H).copy()
    dead = d == 0
    H[dead, dead] = 1.0
    d[dead] = 1.0
    perm = np.argsort(-d, kind="stable") if act_order else np.arange(K)
    H = H[np.ix_(perm, perm)]
    H[np.diag_indices(K)] += damp * float(np.mean(np.diag(H)))
    return H, perm.astype(np.int64), dead


def gptq_eliminate(Hi: np.ndarray, j: int) -> np.ndarray:
    """Remove column j from the inverse Hessian of the columns j.. : returns
    the inverse Hessian of the columns j+1.. (Gaussian elimination)."""
    r = Hi[j, j + 1:]
    return Hi[j + 1:, j + 1:] - np.outer(Hi[j + 1:, j], r) / Hi[j, j]


def gptq_quantize(W: np.ndarray, H: np.ndarray, G: int, act_order: bool = False,
                  damp: float = 0.01, follow: np.ndarray | None = None,
                  record: dict | None = None):
    """INT4 codes with GPTQ error compensation (R18).

    Returns (codes uint8 [N, K], scale fp16 [N, K/G], zero uint8 [N, K/G],
    g_idx int32 [K] or None): the canonical format of ``quantize_rtn``; with
    act-order the channel processed j-th belongs to group j // G.

    Observation hook for comparing another implementation step by step (the
    arithmetic is unchanged): with ``follow`` (codes uint8 [N, K], canonical
    channel order) the error of each column is computed from those codes
    instead of this function's own, so that the compensated weights track the
    other implementation's decisions; ``record`` (a dict) then receives
    'own' (this function's own code decisions, canonical order) and 'tie'
    (the distance of w / s to the nearest half-integer, in code units, for
    each decision)."""
    W = np.array(W, dtype=np.float64, copy=True)
    N, K = W.shape
    if K % G:
        raise ValueError("K must be a multiple of G")
    Hp, perm, dead = gptq_prepare(H, act_order, damp)
    W[:, dead] = 0.0
    Q = W[:, perm]                                  # working copy, processing order
    Hi = np.linalg.inv(Hp)
    codes = np.zeros((N, K), dtype=np.uint8)
    s16 = np.zeros((N, K // G), dtype=np.float16)
    zp = np.zeros((N, K // G), dtype=np.uint8)
    for j in range(K):
        g = j // G
        if j % G == 0:                              # group parameters, compensated weights
            s16[:, g:g + 1], zp[:, g:g + 1] = rtn_params(Q[:, j:j + G].astype(F32), G)
        sf = s16[:, g].astype(F32)
        zf = zp[:, g].astype(F32)
        w32 = Q[:, j].astype(F32)
        ratio = w32 / sf
        q = np.clip(np.rint(ratio) + zf, 0, 15)      # decided in fp32
        codes[:, j] = q.astype(np.uint8)
        if record is not None:
            record.setdefault("own", np.zeros((N, K), np.uint8))[:, perm[j]] = codes[:, j]
            record.setdefault("tie", np.zeros((N, K)))[:, perm[j]] = np.abs(
                np.abs(ratio.astype(np.float64) - np.rint(ratio)) - 0.5)
        if follow is not None:
            q = np.asarray(follow)[:, perm[j]].astype(F32)
            codes[:, j] = q.astype(np.uint8)
        deq = ((q - zf) * sf).astype(F32).astype(np.float64)
        err = (Q[:, j] - deq) / Hi[0, 0]
        Q[:, j + 1:] -= np.outer(err, Hi[0, 1:])    # spread over the remaining columns
        Hi = gptq_eliminate(Hi, 0)
    out = np.zeros_like(codes)
    out[:, perm] = codes
    if act_order:
        g_idx = np.empty(K, dtype=np.int32)
        g_idx[perm] = (np.arange(K) // G).astype(np.int32)
        return out, s16, zp, g_idx
    return out, s16, zp, None


def gptq_loss(W: np.ndarray, what_bits: np.ndarray, H: np.ndarray) -> float:
    """Layer output error tr((W - W_hat) H (W - W_hat)^T) in fp64 (the
    quantity the compensation lowers; H undamped)."""
    D = np.asarray(W, dtype=np.float64) - bf16_bits_to_f64(what_bits)
    return float(np.einsum("nk,kl,nl->", D, np.asarray(H, np.float64), D))


# ---------------------------------------------------------------------------
# LLM.int8 mixed decomposition.  [Survey] §2.1: vector-wise quantization (one
# scale per column of the weight matrix, i.e. per output feature: row n of
# W [N, K] here) and mixed-precision decomposition (the feature dimensions
# where the activations exceed 6.0 in magnitude go through a 16-bit matmul,
# the rest through INT8, and the two results are added).  [Comparison] §6.1:
# llm_int8_threshold = 6.0 and no 16-bit copy of the weights is kept.
# Readings (R19):
#   s_w[n] = max_k |w| / 127 (fp32; 1 if 0), q_w = clamp(rint(w / s_w), +-127);
#   O = {k : |x[m, k]| > threshold for some token m of the call};
#   s_x[m] = max_{k not in O} |x[m, k]| / 127 (1 if 0);
#   q_x = clamp(rint(x / s_x), +-127) outside O and 0 inside O;
#   y[m, n] = (sum_k q_x q_w) s_x[m] s_w[n] + sum_{k in O} x[m, k] w16[n, k],
#   w16 = bf16(fp32(q_w s_w)) (the 16-bit weights of the outlier channels are
#   the dequantized INT8 ones); the INT8 sum is exact (int64 here).
# ---------------------------------------------------------------------------

def int8_quantize_weights(W: np.ndarray):
    """Per output row: (q_w int8 [N, K], s_w fp32 [N])."""
    W = np.ascontiguousarray(W, dtype=F32)
    s = (np.abs(W).max(axis=1) / F32(127.0)).astype(F32)
    s[s == 0] = F32(1.0)
    q = np.clip(np.rint(W / s[:, None]), -127, 127).astype(np.int8)
    return q, s


def int8_outliers(x_bits: np.ndarray, threshold: float = 6.0) -> np.ndarray:
    """Outlier channels of a call: bool [K], |x| > threshold for some token."""
    x = bf16_bits_to_f32(x_bits)
    return np.any(np.abs(x) > F32(threshold), axis=0)


def int8_quantize_activations(x_bits: np.ndarray, outliers: np.ndarray):
    """Per token over the non-outlier channels: (q_x int8 [M, K], s_x fp32 [M])."""
    x = bf16_bits_to_f32(x_bits)
    keep = ~np.asarray(outliers, dtype=bool)
    a = np.where(keep[None, :], np.abs(x), F32(0)).max(axis=1)
    s = (a / F32(127.0)).astype(F32)
    s[s == 0] = F32(1.0)
    q = np.clip(np.rint(x / s[:, None]), -127, 127)
    q = np.where(keep[None, :], q, 0).astype(np.int8)
    return q, s


def int8_mixed_ref(x_bits: np.ndarray, q_w: np.ndarray, s_w: np.ndarray,
                   threshold: float = 6.0):
    """(y_ref fp64 [M, N], abs_ref fp64 [M, N]) of the decomposed product."""
    O_ = int8_outliers(x_bits, threshold)
    q_x, s_x = int8_quantize_activations(x_bits, O_)
    acc = q_x.astype(np.int64) @ q_w.astype(np.int64).T                 # exact
    sx = s_x.astype(np.float64)[:, None]
    sw = s_w.astype(np.float64)[None, :]
    y_int = acc.astype(np.float64) * sx * sw
    a_int = (np.abs(q_x).astype(np.int64) @ np.abs(q_w).astype(np.int64).T) * sx * sw
    w16 = bf16_bits_to_f64(bf16_round_bits((q_w[:, O_].astype(F32) * s_w[:, None]).astype(F32)))
    x = bf16_bits_to_f64(x_bits)[:, O_]
    return y_int + x @ w16.T, a_int + np.abs(x) @ np.abs(w16).T


# ---------------------------------------------------------------------------
# Matmul reference: y[m, n] = sum_k x[m, k] * w_hat[n, k] in fp64, and the
# tolerance |y - y_ref| <= 1e-3 * sum_k |x w_hat| + ulp_bf16(y_ref).
# ---------------------------------------------------------------------------

def matmul_ref(x_bits: np.ndarray, what_bits: np.ndarray):
    """(y_ref, abs_ref) in fp64 for bf16 X [M, K] and bf16 W_hat [N, K]."""
    x = bf16_bits_to_f64(x_bits)
    w = bf16_bits_to_f64(what_bits)
    return x @ w.T, np.abs(x) @ np.abs(w).T


def matmul_exact_small(x_bits: np.ndarray, what_bits: np.ndarray) -> list:
    """Exact rational products and sums by pure-Python loops (tiny inputs)."""
    x = bf16_bits_to_f32(x_bits)
    w = bf16_bits_to_f32(what_bits)
    M, K = x.shape
    N = w.shape[0]
    out = []
    for m in range(M):
        row = []
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                acc += Fraction(float(x[m, k])) * Fraction(float(w[n, k]))
            row.append(acc)
        out.append(row)
    return out


def ulp_bf16(y: np.ndarray) -> np.ndarray:
    """Spacing of the bf16 grid at |y| (8 significant bits); at 0 and in the
    subnormal range it is the smallest subnormal, 2^-133."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.where(a > 0, e, -200.0)
    return np.where(e < -126, 2.0 ** -133, np.exp2(e - 7))


def tolerance(y_ref: np.ndarray, abs_ref: np.ndarray) -> np.ndarray:
    return 1e-3 * np.asarray(abs_ref, np.float64) + ulp_bf16(y_ref)


def check_matmul(y_bits: np.ndarray, y_ref: np.ndarray, abs_ref: np.ndarray):
    """Returns (ok, worst error / tolerance ratio)."""
    y = bf16_bits_to_f64(y_bits)
    err = np.abs(y - y_ref)
    tol = tolerance(y_ref, abs_ref)
    ratio = float((err / tol).max()) if err.size else 0.0
    return bool(np.all(err <= tol)), ratio


# ---------------------------------------------------------------------------
# Storage sizes.  [Primer] opening: a 7B model is ~14 GB in FP16 and ~3.5 GB in
# 4 bits; [Survey] §6.2 and [Comparison] §1: 70B goes from 140 GB to ~35 GB;
# [Handbook] §4.1: codes (params x bits / 8), plus one fp16 scale and one zero
# per group of 128.
# ---------------------------------------------------------------------------

def code_bytes(n_params: int, bits: int = 4) -> int:
    return n_params * bits // 8


def weight_bytes(N: int, K: int, G: int, zero_bytes: float = 0.5,
                 scale_bytes: float = 2.0) -> float:
    """Bytes of one INT4 layer: codes + per-group scale + per-group zero.
    This library stores zeros as 4-bit values (0.5 B); the handbook's worked
    example counts them at 2 B like the scales."""
    groups = N * (K // G)
    return code_bytes(N * K) + groups * scale_bytes + groups * zero_bytes


def nf4_weight_bytes(N: int, K: int, blocksize: int = 64, dq_group: int = 256) -> float:
    nb = N * K // blocksize
    return code_bytes(N * K) + nb + 4 * math.ceil(nb / dq_group)
