/*
 * w4.h -- C ABI of the group-wise 4-bit weight-only linear layer for NVIDIA
 * B200 (sm_100a):  Y[M,N] = X[M,K] . dequant(Wq)^T
 *
 * Source pages (cited by title and section):
 *   [Survey]     "大模型量化选型：五种主流方案对比与实战"
 *   [Primer]     aicoding.csdn.net primer, "一、量化究竟做了什么" onwards
 *   [Handbook]   "这不是理论课，是能立刻上手的LLM量化实操手册"
 *   [Guide]      "开源模型量化实战指南：GGUF、GPTQ、AWQ选型与本地部署"
 *   [Comparison] "【推理与部署篇05】模型量化部署深度对比：GPTQ、AWQ、GGUF与FP8实战指南"
 *
 * Conventions for every entry point
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them.  Arrays are dense, row-major,
 *     16-byte aligned unless stated otherwise.
 *   - fp16 and bf16 values are passed as their uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work and returns; results are ready when the stream
 *     has reached that point.
 *   - Return value: W4_OK, or an error found on the host BEFORE anything is
 *     launched (bad sizes, null or misaligned pointers, unsupported shapes),
 *     or W4_ERR_CUDA if a launch failed.  Errors that only the device can see
 *     (g_idx out of range, a pipeline wait that timed out) set a per-device
 *     error word that w4_device_status() reads.
 *   - No CPU fallback: every computation runs in this library's kernels.
 *
 * Layouts
 *   W       fp32 [N, K]        row n = output channel, K contiguous
 *   Wq      uint8 [N, K/2]     two 4-bit codes per byte, even k in the low
 *                              nibble ([Guide] §1.1: INT4 is half a byte)
 *   scales  fp16 [N, K/G]      one scale per (row, group)
 *   zeros   uint8 [N, K/G]     one zero point per (row, group), value 0..15
 *   g_idx   int32 [K]          act-order group of each input channel, or NULL
 *   X       bf16 [M, K]        activations
 *   Y       bf16 [M, N]        output
 *   Wp      uint8 opaque       pre-shuffled weights (w4_prepack / nf4_prepack)
 */
#ifndef W4_H_
#define W4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int w4_status;
typedef void* w4_stream; /* a cudaStream_t */

enum {
  W4_OK = 0,
  W4_ERR_INVALID_ARG = 1, /* null/misaligned pointer, size out of range      */
  W4_ERR_UNSUPPORTED = 2, /* valid but not supported by this library         */
  W4_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed            */
  W4_ERR_TIMEOUT = 4,     /* a device pipeline wait gave up (device status)  */
  W4_ERR_DEVICE_INPUT = 5, /* the device found bad input data (device status) */
  W4_ERR_SCRATCH_LIMIT = 6, /* w4a16_gemm_static_scratch: the call needs more
                               workspace than W4_STATIC_SCRATCH_BYTES          */
  W4_ERR_BOUNDS = 7        /* bounds-checked build only (device status): a
                              kernel index fell outside its buffer; the access
                              was skipped, so outputs are not to be trusted   */
};

/* Human-readable name of a status code (static string, never NULL). */
const char* w4_status_string(w4_status s);

/* ABI version (major * 100 + minor). */
int w4_version(void);

/* Waits for `stream`, then returns and clears the error word that kernels of
 * this library set on the current device: W4_OK, W4_ERR_BOUNDS (bounds-checked
 * build only), W4_ERR_TIMEOUT or W4_ERR_DEVICE_INPUT, in that order of
 * precedence (or W4_ERR_CUDA if the synchronisation itself failed). */
w4_status w4_device_status(w4_stream stream);

/* 1 for the bounds-checked build of this library (libw4b200_checked.so,
 * compiled with W4_CHECKED: every global access of every kernel is checked
 * against the extent of its buffer implied by the call's arguments; a
 * violation is recorded as W4_ERR_BOUNDS and the access skipped), 0 for the
 * normal build.  The two builds export the same functions. */
int w4_checked_build(void);

/* Failure-path check (no counterpart on the pages): launches one thread that
 * runs this library's bounded pipeline wait on a barrier nothing arrives on,
 * with a limit of about 1 ms instead of the kernels' 2 s.  The wait gives up,
 * sets the device error word and returns; the next w4_device_status(stream)
 * returns W4_ERR_TIMEOUT and the context stays usable.  Nothing faults. */
w4_status w4_selftest_wait_timeout(w4_stream stream);

/* ------------------------------------------------------------------------
 * INT4 asymmetric round-to-nearest quantization, group-wise along K.
 * [Comparison] §2.3: scale = (max - min) / (2^b - 1), zero_point =
 * round(-min / scale), codes in [0, 2^b - 1] (printed for b = 8; here b = 4);
 * [Comparison] §2.2 / [Primer] §二: one scale per group of G weights;
 * [Primer] §四: plain rounding (RTN).  Per (row n, group g):
 *   mn = min(min_k w, 0), mx = max(max_k w, 0)                     (fp32)
 *   scale = fp16((mx - mn) / 15), or 1.0 if that is 0
 *   zp = clamp(rint(-mn / scale), 0, 15)
 *   q_k = clamp(rint(w_k / scale) + zp, 0, 15)     (rint: half to even)
 * Group g is {k : k / G == g}, or {k : g_idx[k] == g} when g_idx is given
 * (GPTQ act-order, [Survey] §3.2 desc_act).
 *   W        in   fp32 [N, K]
 *   N, K, G  N >= 1; G in {32, 64, 128}; K >= G, K % G == 0, K % 2 == 0
 *   g_idx    in   int32 [K], values in [0, K/G), or NULL.  Out-of-range
 *                 values are skipped and reported as W4_ERR_DEVICE_INPUT.
 *   Wq       out  uint8 [N, K/2]
 *   scales   out  fp16 bits [N, K/G]
 *   zeros    out  uint8 [N, K/G]
 * Bit-exact with the CPU definition above.  w must be finite and every group
 * must have (mx - mn) / 15 < 65520, so that the fp16 scale is finite (true
 * whenever |w| < 491000). */
w4_status w4_quantize_rtn(const float* W, int N, int K, int G, const int32_t* g_idx,
                          uint8_t* Wq, uint16_t* scales, uint8_t* zeros,
                          w4_stream stream);

/* INT4 symmetric (absmax) quantization, group-wise along K, in the same
 * canonical format as w4_quantize_rtn (so w4_dequant, w4_prepack and
 * w4a16_gemm take it unchanged).  [Comparison] §2.3: symmetric scale =
 * max|w| / (2^(b-1) - 1), values in [-(2^(b-1) - 1), 2^(b-1) - 1] (printed
 * for b = 8: /127; [Survey] §1 works 80 / 127 = 0.63); here b = 4:
 *   scale = fp16(max_k |w_k| / 7), or 1.0 if that is 0
 *   q_k = clamp(rint(w_k / scale), -7, 7) + 8      (codes 1..15; 0 unused)
 *   zero point = 8 for every group
 * Arguments, group definition (g_idx), error behaviour and preconditions as
 * for w4_quantize_rtn, with max|w| / 7 < 65520 in every group. */
w4_status w4_quantize_sym(const float* W, int N, int K, int G, const int32_t* g_idx,
                          uint8_t* Wq, uint16_t* scales, uint8_t* zeros,
                          w4_stream stream);

/* AWQ per-input-channel factor ([Survey] §4.1, [Comparison] §4.1): the
 * weights of input channel k are quantized as w * s_k and the activations
 * enter the product as x / s_k, so (X / s)(W s)^T = X W^T before
 * quantization; the effective weight is round(W s / scale) scale / s.  s is
 * an input (found offline by the calibration search the pages describe).
 *   W      in   fp32 [N, K]
 *   s      in   fp32 [K], finite and nonzero (not checked)
 *   W_out  out  fp32 [N, K] = fp32(W[n, k] * s[k]) (round to nearest even);
 *               may be W itself
 * Quantize W_out with w4_quantize_rtn or w4_quantize_sym, then prepack. */
w4_status w4_awq_scale_weights(const float* W, const float* s, int N, int K, float* W_out,
                               w4_stream stream);

/* X_out[m, k] = bf16_rne(fp32(X[m, k]) / s[k]) (IEEE division): the
 * activation side of the AWQ factor, as w4a16_awq_gemm applies it.
 *   X, X_out  bf16 [M, K], 16-byte aligned, K % 8 == 0; X_out may be X
 *   s         fp32 [K], 16-byte aligned                                    */
w4_status w4_awq_scale_activations(const uint16_t* X, const float* s, int M, int K,
                                   uint16_t* X_out, w4_stream stream);

/* GPTQ error compensation at quantization time ([Comparison] §3.1; [Survey]
 * §3, §3.2).  The layer's columns are quantized one at a time (INT4, the
 * asymmetric RTN rule of w4_quantize_rtn per group) and each column's error
 * is spread over the columns not yet quantized through the inverse of the
 * damped Hessian H' = H + lambda I, lambda = damp * mean(diag H):
 *   Hi = H'^-1 over the remaining columns; for column j:
 *     q_j = quantize(w_j);  e = (w_j - dq(q_j)) / Hi_jj
 *     w_k -= e * Hi_jk for every later k;  Hi loses row/column j (Gaussian
 *     elimination, i.e. Hi becomes the inverse of H' without column j).
 * A group's scale and zero point are taken from its current (compensated)
 * weights when its first column is reached.  A channel with H_kk = 0 gets
 * H_kk = 1 and weight 0.  With act_order the columns are taken in the order
 * of decreasing H_kk (stable), group g holds the channels processed in
 * positions [gG, (g+1)G), and g_idx receives that map (the act-order format
 * of w4_quantize_rtn / w4_prepack).  The device computes Hi's upper Cholesky
 * factor once in fp64 and runs the column updates in fp32; the result agrees
 * with an fp64 evaluation of the steps above up to rounding (a weight near a
 * rounding boundary may take the neighbouring code).
 *   W         in   fp32 [N, K]
 *   H         in   fp32 [K, K], symmetric positive semi-definite (e.g. from
 *                  w4_gptq_hessian); a negative or non-finite diagonal entry
 *                  or a non-positive pivot is reported as W4_ERR_DEVICE_INPUT
 *   G         32, 64 or 128; K % G == 0, K % 32 == 0, K <= 65536
 *   damp      >= 0 (the pages use 0.01)
 *   Wq, scales, zeros  out, as w4_quantize_rtn
 *   g_idx     out  int32 [K]; required with act_order, else may be NULL
 *                  (then receives k / G)
 *   workspace device memory of w4_gptq_workspace_bytes(N, K, G) bytes,
 *             256-byte aligned, contents irrelevant (about 20 K^2 + 9 N K B) */
size_t w4_gptq_workspace_bytes(int N, int K, int G);
w4_status w4_gptq_quantize(const float* W, const float* H, int N, int K, int G, int act_order,
                           float damp, uint8_t* Wq, uint16_t* scales, uint8_t* zeros,
                           int32_t* g_idx, void* workspace, size_t workspace_bytes,
                           w4_stream stream);

/* H = 2 X^T X ([Comparison] §3.1: H = 2 X X^T with X the calibration
 * activations as columns), fp32 accumulation.
 *   X  in   bf16 [n, K] (n calibration tokens);  H  out  fp32 [K, K]     */
w4_status w4_gptq_hessian(const uint16_t* X, int n, int K, float* H, w4_stream stream);

/* LLM.int8 mixed decomposition ([Survey] §2.1: one weight scale per output
 * feature; input channels whose activation exceeds the threshold in magnitude
 * go through a 16-bit product, the others through INT8, and the results are
 * added; [Comparison] §6.1: threshold 6.0, no 16-bit weight copy kept).
 *   llm_int8_quantize_weights:  s_w[n] = max_k |w[n,k]| / 127 (1 if 0),
 *     q_w = clamp(rint(w / s_w), -127, 127)
 *     W in fp32 [N, K];  qw out int8 [N, K];  sw out fp32 [N]
 *   llm_int8_gemm, per call:
 *     O = {k : |x[m,k]| > threshold for some m}
 *     s_x[m] = max over k not in O of |x[m,k]| / 127 (1 if 0)
 *     q_x = clamp(rint(x / s_x), -127, 127) outside O, 0 on O
 *     y[m,n] = (sum_k q_x q_w) s_x[m] s_w[n]             (exact int32 sum)
 *            + sum_{k in O} x[m,k] bf16(q_w[n,k] s_w[n])  (fp32)
 *     X bf16 [M, K], 16-byte aligned; qw 16-byte aligned; K % 64 == 0,
 *     K <= 65536; Y bf16 [M, N]; threshold >= 0 (the pages use 6.0);
 *     workspace of llm_int8_workspace_bytes(M, N, K) bytes, 256-byte aligned,
 *     contents irrelevant (the call clears what it needs cleared); the call
 *     leaves it dirty, so it must not be the workspace of w4a16_gemm /
 *     nf4_gemm (which must stay zeroed).  Calls that share a workspace must
 *     be ordered on one stream.  Three launches (outlier scan, token
 *     quantization, INT8 product with the 16-bit outlier part in its last
 *     work item per row tile) chained by programmatic dependent launch; the
 *     INT8 product uses warp-level s8 MMAs.                                 */
w4_status llm_int8_quantize_weights(const float* W, int N, int K, int8_t* qw, float* sw,
                                    w4_stream stream);
size_t llm_int8_workspace_bytes(int M, int N, int K);
w4_status llm_int8_gemm(const uint16_t* X, const int8_t* qw, const float* sw, int M, int N, int K,
                        float threshold, uint16_t* Y, void* workspace, size_t workspace_bytes,
                        w4_stream stream);

/* Dequantization to the bf16 compute dtype ([Survey] §6.2, [Primer] §七):
 *   w_hat[n,k] = bf16_rne( float(q - zp) * float(scale) )
 * (the fp32 product is exact, so there is exactly one rounding).
 *   Wq, scales, zeros, g_idx   in, as produced by w4_quantize_rtn
 *   W_out                      out  bf16 bits [N, K]                        */
w4_status w4_dequant(const uint8_t* Wq, const uint16_t* scales, const uint8_t* zeros,
                     const int32_t* g_idx, int N, int K, int G, uint16_t* W_out,
                     w4_stream stream);

/* Bytes of the canonical INT4 storage of one [N, K] layer: codes N*K/2,
 * fp16 scales 2 B and 4-bit zero points 0.5 B per group ([Handbook] §4.1
 * counts codes as params*bits/8 plus per-group constants). */
double w4_weight_bytes(int N, int K, int G);

/* ------------------------------------------------------------------------
 * Pre-shuffled device layout (no counterpart on the pages: it is the
 * B200-specific part).  Wp holds, for each tile of 128 output rows and each
 * stage of 128 input channels, one contiguous block that a single bulk copy
 * brings into shared memory:
 *   codes   8192 B in warp-MMA fragment order: for row group rg < 8 (16
 *           rows), channel block kb < 8 (16 channels) and lane t < 32
 *           (g = t / 4, u = t % 4) the 32-bit word at byte offset
 *           (((rg * 2 + kb / 4) * 32 + t) * 4 + kb % 4) * 4 holds rows
 *           r0 = 16 rg + g, r1 = r0 + 8 x channels c = 16 kb + 4 u .. c + 3
 *           as four pairs j: bits 4j..4j+3 and 16+4j..19+4j hold
 *           (r0, c, c+1), (r0, c+2, c+3), (r1, c, c+1), (r1, c+2, c+3)
 *   scales  fp16 [rg][group within the stage][g][2] (rows r0, r1)
 *   zeros   uint8 [rg][group][g] = z(r0) | z(r1) << 4
 *           (stage block: 8512 / 8832 / 9472 B for G = 128 / 64 / 32)
 * Rows >= N and channels >= K are padding (code 0, scale 0, zero 0).  With
 * act_order, the channels are taken in the order that makes each group
 * contiguous (a stable sort of k by g_idx[k]) and that permutation, int32
 * [K], follows the tiles.  Act-order needs exactly G channels per group
 * (the GPTQ layout); otherwise the device reports W4_ERR_DEVICE_INPUT.   */
size_t w4_prepacked_bytes(int N, int K, int G, int act_order);

/* Canonical (Wq, scales, zeros, g_idx) -> Wp.  Wp must hold
 * w4_prepacked_bytes(N, K, G, g_idx != NULL) bytes. */
w4_status w4_prepack(const uint8_t* Wq, const uint16_t* scales, const uint8_t* zeros,
                     const int32_t* g_idx, int N, int K, int G, uint8_t* Wp,
                     w4_stream stream);

/* Inverse of w4_prepack for the permuted-channel view: writes the codes,
 * scales and zeros in the prepacked channel order (identical to the
 * canonical arrays when act_order == 0) and, if perm != NULL and act_order,
 * the channel permutation int32 [K]. */
w4_status w4_unprepack(const uint8_t* Wp, int N, int K, int G, int act_order,
                       uint8_t* Wq, uint16_t* scales, uint8_t* zeros, int32_t* perm,
                       w4_stream stream);

/* ------------------------------------------------------------------------
 * W4A16 linear: Y = X . w_hat^T with w_hat as in w4_dequant, bf16 products,
 * fp32 accumulation, bf16 (round to nearest even) output.  Two kernels,
 * chosen by M ([Survey] §4.3: AWQ ships a "GEMV" kernel for single requests
 * and a "GEMM" kernel for batches): M <= 32 streams the packed weights once
 * through warp-level MMAs; M > 32 runs tcgen05 tensor-core MMAs with the
 * dequantized weight tile in tensor memory (Y^T = W_hat . X^T), M in tiles
 * of 64..256 tokens.  The kernels use programmatic dependent launch and
 * start reading Wp before the kernel before them on the stream has
 * finished: Wp is constant model state and must not be written by that
 * kernel (this library's prepack kernels make their writes visible before
 * they exit, so prepack followed by a GEMM is fine).
 *   X          in   bf16 [M, K], 16-byte aligned, K % 64 == 0
 *   Wp         in   from w4_prepack (act_order must match)
 *   M, N, K, G M >= 1, N >= 1; with M <= 32 (the decode kernel) N is at most
 *              2097152 (65536 groups of 32 rows, one arrival counter each):
 *              larger N returns W4_ERR_UNSUPPORTED, launching nothing
 *   Y          out  bf16 [M, N]
 *   workspace  device scratch of at least w4_workspace_bytes(M,N,K,G,act_order)
 *              bytes, 256-byte aligned, ZEROED ONCE before its first use; the
 *              library leaves it zeroed after every call (split-K counters).
 *              Calls that share a workspace must be ordered on one stream.
 *              w4_workspace_bytes returns 0 for an invalid or unsupported
 *              shape.                                                       */
size_t w4_workspace_bytes(int M, int N, int K, int G, int act_order);
w4_status w4a16_gemm(const uint16_t* X, const uint8_t* Wp, int M, int N, int K, int G,
                     int act_order, uint16_t* Y, void* workspace, size_t workspace_bytes,
                     w4_stream stream);

/* ------------------------------------------------------------------------
 * W4A16 linear for AWQ weights: Y = (X / s) . w_hat^T, with w_hat from
 * weights quantized as W s (w4_awq_scale_weights).  The division is done
 * once, by a prologue kernel that writes bf16(x / s_k) into the workspace
 * (the same pass that applies the act-order permutation), and the weight
 * stream and GEMM kernels are w4a16_gemm's; the result is identical to
 * w4_awq_scale_activations followed by w4a16_gemm.
 *   s          in   fp32 [K], 16-byte aligned, finite and nonzero
 *   workspace  at least w4_awq_workspace_bytes(M, N, K, G, act_order)
 *   all other arguments as for w4a16_gemm                                  */
size_t w4_awq_workspace_bytes(int M, int N, int K, int G, int act_order);
w4_status w4a16_awq_gemm(const uint16_t* X, const float* s, const uint8_t* Wp, int M, int N,
                         int K, int G, int act_order, uint16_t* Y, void* workspace,
                         size_t workspace_bytes, w4_stream stream);

/* ------------------------------------------------------------------------
 * w4a16_gemm without a caller workspace.  The pages describe no such call; it
 * computes exactly what w4a16_gemm computes, for callers that cannot allocate
 * device memory when they call: a runtime that plans all of HBM at start-up,
 * a caller that cannot pay cudaFree's device-wide synchronisation, or plain C
 * code without a device allocator.  It allocates nothing (no cudaMalloc /
 * cudaFree, no allocating library routine): its workspace is a file-scope
 * device array of W4_STATIC_SCRATCH_BYTES (16 MiB), one copy per device.
 *   Arguments, layouts and results as for w4a16_gemm (minus the workspace).
 *   Limit: returns W4_ERR_SCRATCH_LIMIT, launching nothing, when
 *          w4_workspace_bytes(M, N, K, G, act_order) > W4_STATIC_SCRATCH_BYTES
 *          (every decode shape M <= 32 up to N * K = 28672 * 8192 fits; large
 *          prefill shapes that split K do not: use w4a16_gemm there).
 *   First call on a device: looks up that device's copy of the array (which
 *          may load the module on the device) with the device current, and
 *          returns W4_ERR_CUDA if that fails.  Make the first call on each
 *          device before any stream capture.  The address is cached per
 *          device together with the context it was found in; a call that
 *          finds another context current (after cudaDeviceReset, or after
 *          the primary context was released and created again) looks it up
 *          again, so that call too should come before any capture.
 *   Each call clears (cudaMemsetAsync on `stream`) the arrival counters it
 *          uses before its kernel runs.
 *   One array per device: calls whose executions can overlap on the same
 *          device (different streams, or different host threads) race on it
 *          and give wrong results.  Order them on one stream.              */
#define W4_STATIC_SCRATCH_BYTES 16777216u /* 16 MiB */
w4_status w4a16_gemm_static_scratch(const uint16_t* X, const uint8_t* Wp, int M, int N, int K,
                                    int G, int act_order, uint16_t* Y, w4_stream stream);

/* ------------------------------------------------------------------------
 * NF4 ([Survey] §6.1: 16 levels at normal-distribution quantiles, denser near
 * zero; [Comparison] §6.2; [Survey] §6.3: block-wise absmax, one scale per 64
 * weights; [Survey] §6.2 / [Comparison] §6.1: double quantization of the
 * scales).  Blocks are 64 consecutive weights of a row (K % 64 == 0).
 *   a = max |w| over the block (fp32); v = w / a (0 if a == 0);
 *   q = #{ i < 15 : v > t_i }, t_i = (T[i] + T[i+1]) / 2  (lower code on ties)
 *   per run of dq_group consecutive blocks: s2 = max(a) / 255 (1 if 0),
 *   c = clamp(rint(a / s2), 0, 255), a' = fp32(c * s2)
 *   w_hat = bf16_rne(fp32(T[q] * a'))
 *   W          in   fp32 [N, K]
 *   blocksize  64 (only value supported); dq_group in [1, 1024]
 *   Wq         out  uint8 [N, K/2]
 *   absmax_q   out  uint8 [N*K/64]
 *   s2         out  fp32 [ceil(N*K/64/dq_group)]                           */
w4_status nf4_quantize(const float* W, int N, int K, int blocksize, int dq_group,
                       uint8_t* Wq, uint8_t* absmax_q, float* s2, w4_stream stream);
w4_status nf4_dequant(const uint8_t* Wq, const uint8_t* absmax_q, const float* s2, int N,
                      int K, int blocksize, int dq_group, uint16_t* W_out,
                      w4_stream stream);

/* The 16 NF4 levels this library uses (host memory, fp32). */
void nf4_levels(float out[16]);

/* NF4 pre-shuffled layout: as for INT4 (same codes block per 128 rows x 128
 * channels) followed by the absmax codes uint8 [rg][64-block in stage (2)]
 * [g][2] (rows r0, r1); stage block 8448 B.  s2 stays in its canonical
 * array. */
size_t nf4_prepacked_bytes(int N, int K);
w4_status nf4_prepack(const uint8_t* Wq, const uint8_t* absmax_q, int N, int K,
                      uint8_t* Wp, w4_stream stream);

/* Y = X . w_hat^T for NF4 weights (same kernel family as w4a16_gemm).
 *   X bf16 [M,K]; Wp from nf4_prepack; s2 as from nf4_quantize; Y bf16 [M,N].
 *   Workspace rules, the decode limit N <= 2097152 at M <= 32 and the 0 that
 *   nf4_workspace_bytes returns for an unsupported shape are w4a16_gemm's. */
size_t nf4_workspace_bytes(int M, int N, int K);
w4_status nf4_gemm(const uint16_t* X, const uint8_t* Wp, const float* s2, int M, int N,
                   int K, int dq_group, uint16_t* Y, void* workspace,
                   size_t workspace_bytes, w4_stream stream);

/* ------------------------------------------------------------------------
 * NF4 with mean-offset double quantization of the block constants.  The
 * pages ask for the constants to be quantized a second time ([Survey] §6.2,
 * the [Primer]'s §七, [Comparison] §6 bnb_4bit_use_double_quant) without
 * saying how; this variant centres each run of dq_group constants on the
 * run's mean and stores the residuals with the pages' symmetric 8-bit
 * formula ([Comparison] §2.3: max|x| / 127, round):
 *   mu = fp32(S / n), S the fp64 sum of the run's a in block order, n the
 *        run's block count (the last run may be shorter);
 *   d = fp32(a - mu); s2 = fp32(max|d| / 127) (1 if 0);
 *   c = clamp(rint(d / s2), -127, 127) (int8); a' = fp32(fp32(c * s2) + mu)
 *   w_hat = bf16_rne(fp32(T[q] * a')); codes q as for nf4_quantize.
 *   absmax_q   out  int8 [N*K/64]
 *   mean, s2   out  fp32 [ceil(N*K/64/dq_group)] each
 *   all other arguments, layouts and errors as for nf4_quantize / nf4_dequant.
 * Prepack the codes and the int8 constants with nf4_prepack (it moves the
 * constant bytes unchanged; pass absmax_q as bytes) and multiply with
 * nf4_gemm_meandq, which takes the run means beside s2 and otherwise the
 * arguments, workspace and limits of nf4_gemm.                             */
w4_status nf4_quantize_meandq(const float* W, int N, int K, int blocksize, int dq_group,
                              uint8_t* Wq, int8_t* absmax_q, float* mean, float* s2,
                              w4_stream stream);
w4_status nf4_dequant_meandq(const uint8_t* Wq, const int8_t* absmax_q, const float* mean,
                             const float* s2, int N, int K, int blocksize, int dq_group,
                             uint16_t* W_out, w4_stream stream);
w4_status nf4_gemm_meandq(const uint16_t* X, const uint8_t* Wp, const float* mean,
                          const float* s2, int M, int N, int K, int dq_group, uint16_t* Y,
                          void* workspace, size_t workspace_bytes, w4_stream stream);

/* ------------------------------------------------------------------------
 * FP4: the second 4-bit type of the block-wise scheme ([Survey] §6.3: the
 * library offers NF4 and FP4; [Survey] §6.1: plain FP4 has three significant
 * bits and uneven spacing), with the 4-bit float layout [S:1][E:2][M:1]
 * ([Comparison] §7.2).  Code bit 3 = sign, bits 2..1 = exponent e, bit 0 =
 * mantissa m; magnitude m/2 (e = 0) or 2^(e-1)(1 + m/2), i.e. 0, 0.5, 1, 1.5,
 * 2, 3, 4, 6 for codes 0..7; table T = magnitude / 6 (fp32), so T spans
 * [-1, 1] and a block's absmax maps to code 7.
 *   v = w / a as for NF4; magnitude code = #{ i < 7 : |v| > t_i },
 *   t_i = fp32((T[i] + T[i+1]) / 2) (the lower magnitude on a midpoint);
 *   q = magnitude code + 8 if v < 0 and that code is not 0, else the code.
 * Blocks, double quantization, dequantization (w_hat = bf16(fp32(T[q] a'))),
 * arguments, layouts and errors are those of nf4_quantize / nf4_dequant.
 * The prepacked layout is NF4's: prepack with nf4_prepack
 * (nf4_prepacked_bytes), size the workspace with nf4_workspace_bytes.      */
w4_status fp4_quantize(const float* W, int N, int K, int blocksize, int dq_group,
                       uint8_t* Wq, uint8_t* absmax_q, float* s2, w4_stream stream);
w4_status fp4_dequant(const uint8_t* Wq, const uint8_t* absmax_q, const float* s2, int N,
                      int K, int blocksize, int dq_group, uint16_t* W_out,
                      w4_stream stream);

/* The 16 FP4 levels this library uses (host memory, fp32). */
void fp4_levels(float out[16]);

/* Y = X . w_hat^T for FP4 weights: the NF4 kernels with the FP4 table.
 *   Arguments as for nf4_gemm; Wp from nf4_prepack of fp4_quantize output. */
w4_status fp4_gemm(const uint16_t* X, const uint8_t* Wp, const float* s2, int M, int N,
                   int K, int dq_group, uint16_t* Y, void* workspace,
                   size_t workspace_bytes, w4_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* W4_H_ */
