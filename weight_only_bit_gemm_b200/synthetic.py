"""Seeded synthetic inputs for the 4-bit weight-only linear layer.

This module only draws random numbers and lays them out; it holds none of the
quantization arithmetic.  Both the CPU oracle and the CUDA path are fed from
the same host arrays produced here.

The pages measure trained LLaMA/Qwen layers.  No weights or datasets exist
here, so these draws stand in for them with the layer shapes and value
distributions the workloads name:

* ``W``: fp32 ``standard_normal * sigma`` of shape ``[N, K]`` (row = output
  channel, K contiguous), optionally with a fraction of input channels
  (K-index columns) multiplied by a factor.
* ``X``: fp32 ``standard_normal`` of shape ``[M, K]``, optionally with a
  fraction of K-channels multiplied by a factor (activation outliers, as in
  "大模型量化选型：五种主流方案对比与实战" §1: a few channels reach 20..100),
  then rounded to bf16 (round-to-nearest-even) and returned as the bf16 bit
  pattern in a ``uint16`` array.
* ``g_idx``: the act-order group map ``g_idx[perm[j]] = j // G`` for a seeded
  permutation ``perm`` of ``range(K)``.
* calibration activations for GPTQ's Hessian: fp32 ``standard_normal`` ``[n, K]``
  plus ``rank`` shared factors (``standard_normal [n, rank] @ standard_normal
  [rank, K]``), so that channels are correlated as real activations are,
  rounded to bf16;
* ``s``: the AWQ per-input-channel factor, fp32 ``[K]`` uniform in
  ``[lo, hi]`` (default 0.95..1.05, the range
  "【推理与部署篇05】模型量化部署深度对比" §4.1 gives for important and
  secondary channels); the search that finds it offline is not run here.

Generators (``numpy.random.default_rng`` keyed by integer lists):
``[seed, tag, K, N]`` for W (draw order: W, then the outlier columns),
``[seed, tag, K, N, M]`` for X (X, then its outlier channels) and
``[seed, tag, K, N, 7]`` for the act-order permutation and
``[seed, tag, K, N, 11]`` for the AWQ factor and ``[seed, tag, K, n, 13]`` for the
calibration activations.
"""
from __future__ import annotations

import numpy as np
import torch


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([int(k) for k in key])


def draw_w(N: int, K: int, sigma: float = 0.02, *, seed: int = 0, tag: int = 0,
           outlier_frac: float = 0.0, outlier_scale: float = 1.0) -> np.ndarray:
    """fp32 weights ``[N, K]`` ~ N(0, sigma^2); ``round(outlier_frac*K)``
    input channels (distinct, seeded) are multiplied by ``outlier_scale``."""
    rng = _rng(seed, tag, K, N)
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(sigma)
    n_out = int(round(outlier_frac * K))
    if n_out > 0:
        cols = rng.choice(K, size=n_out, replace=False)
        w[:, cols] *= np.float32(outlier_scale)
    return w


def draw_perm(K: int, *, seed: int = 0, tag: int = 0, N: int = 0) -> np.ndarray:
    """Seeded permutation of ``range(K)`` (its own generator stream)."""
    return _rng(seed, tag, K, N, 7).permutation(K).astype(np.int64)


def draw_awq_s(K: int, *, seed: int = 0, tag: int = 0, N: int = 0, lo: float = 0.95,
               hi: float = 1.05) -> np.ndarray:
    """fp32 per-input-channel factor ``[K]`` uniform in ``[lo, hi]``."""
    return _rng(seed, tag, K, N, 11).uniform(lo, hi, K).astype(np.float32)


def draw_calib_x(n: int, K: int, *, seed: int = 0, tag: int = 0, rank: int = 4) -> np.ndarray:
    """bf16 calibration activations ``[n, K]`` (uint16 bits) with ``rank``
    shared factors."""
    rng = _rng(seed, tag, K, n, 13)
    x = rng.standard_normal((n, K), dtype=np.float32)
    if rank > 0:
        x += rng.standard_normal((n, rank), dtype=np.float32) @ \
            rng.standard_normal((rank, K), dtype=np.float32)
    return to_bf16_bits(x)


def act_order_g_idx(perm: np.ndarray, G: int) -> np.ndarray:
    """``g_idx[perm[j]] = j // G``: channel perm[j] is the j-th one quantized."""
    K = perm.shape[0]
    g = np.empty(K, dtype=np.int32)
    g[perm] = (np.arange(K) // G).astype(np.int32)
    return g


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even, via torch's CPU cast) -> uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 values."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def draw_x(M: int, K: int, *, seed: int = 0, tag: int = 0, N: int = 0,
           outlier_frac: float = 0.0, outlier_scale: float = 1.0) -> np.ndarray:
    """bf16 activations ``[M, K]`` (uint16 bit patterns)."""
    rng = _rng(seed, tag, K, N, M)
    x = rng.standard_normal((M, K), dtype=np.float32)
    n_out = int(round(outlier_frac * K))
    if n_out > 0:
        cols = rng.choice(K, size=n_out, replace=False)
        x[:, cols] *= np.float32(outlier_scale)
    return to_bf16_bits(x)


# ---------------------------------------------------------------------------
# Workload catalogue: the five layer-shape families and their distributions.
# ---------------------------------------------------------------------------

TINY = dict(name="tiny single linear", tag=1, shapes=[(512, 512)], Ms=[1], G=128,
            sigma=0.02)
LLAMA7B_DECODE = dict(name="Llama-7B decode GEMV", tag=2,
                      shapes=[(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)],
                      Ms=[1, 4, 16], G=128, sigma=0.02,
                      x_outlier_frac=0.001, x_outlier_scale=50.0)
NF4_DECODE = dict(name="NF4 decode/small batch", tag=3,
                  shapes=[(4096, 14336), (14336, 4096)], Ms=[1, 8, 32],
                  blocksize=64, dq_group=256, sigma=0.02)
PREFILL_70B = dict(name="70B MLP prefill", tag=4, shapes=[(8192, 28672), (28672, 8192)],
                   Ms=[512, 2048, 8192], G=128, sigma=0.015,
                   w_outlier_frac=0.01, w_outlier_scale=8.0)
ACT_ORDER_13B = dict(name="13B MLP act-order", tag=5, shapes=[(5120, 13824), (13824, 5120)],
                     Ms=[1, 16, 256], G=32, G_sweep=[64, 128], sigma=0.02)

# Symmetric INT4 weights quantized after the AWQ factor (W s), activations
# divided by it: the Llama-7B decode shapes, with the activation outliers
# that motivate AWQ.
AWQ_SYM_DECODE = dict(name="Llama-7B decode GEMV, AWQ factor + symmetric INT4", tag=6,
                      shapes=[(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)],
                      Ms=[1, 4, 16], G=128, sigma=0.02,
                      x_outlier_frac=0.001, x_outlier_scale=50.0, awq_lo=0.95, awq_hi=1.05)

# FP4 (E2M1) weights in the NF4 block-wise layout, on the NF4 decode shapes.
FP4_DECODE = dict(name="FP4 decode/small batch", tag=7,
                  shapes=[(4096, 14336), (14336, 4096)], Ms=[1, 8, 32],
                  blocksize=64, dq_group=256, sigma=0.02)

WORKLOADS = [TINY, LLAMA7B_DECODE, NF4_DECODE, PREFILL_70B, ACT_ORDER_13B, AWQ_SYM_DECODE,
             FP4_DECODE]


def layer_w(wl: dict, K: int, N: int, seed: int = 0) -> np.ndarray:
    return draw_w(N, K, wl["sigma"], seed=seed, tag=wl["tag"],
                  outlier_frac=wl.get("w_outlier_frac", 0.0),
                  outlier_scale=wl.get("w_outlier_scale", 1.0))


def layer_x(wl: dict, M: int, K: int, N: int, seed: int = 0) -> np.ndarray:
    return draw_x(M, K, seed=seed, tag=wl["tag"], N=N,
                  outlier_frac=wl.get("x_outlier_frac", 0.0),
                  outlier_scale=wl.get("x_outlier_scale", 1.0))


def layer_awq_s(wl: dict, K: int, N: int, seed: int = 0) -> np.ndarray:
    return draw_awq_s(K, seed=seed, tag=wl["tag"], N=N, lo=wl.get("awq_lo", 0.95),
                      hi=wl.get("awq_hi", 1.05))
