"""ctypes binding of ``libw4b200.so`` (C ABI in ``include/w4.h``).

Argument marshalling only: every computation runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (torch provides device memory and the
current stream); there is no CPU path, and importing this module fails loudly
when the library has not been built.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libw4b200.so")
LIB_CHECKED_PATH = os.path.join(_PKG, "libw4b200_checked.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "w4.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m weight_only_bit_gemm_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

_SIGS = {
    "w4_status_string": (ctypes.c_char_p, [_i]),
    "w4_version": (_i, []),
    "w4_checked_build": (_i, []),
    "w4_device_status": (_i, [_p]),
    "w4_selftest_wait_timeout": (_i, [_p]),
    "w4_weight_bytes": (ctypes.c_double, [_i, _i, _i]),
    "w4_quantize_rtn": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p]),
    "w4_quantize_sym": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p]),
    "w4_awq_scale_weights": (_i, [_p, _p, _i, _i, _p, _p]),
    "w4_awq_scale_activations": (_i, [_p, _p, _i, _i, _p, _p]),
    "w4_gptq_workspace_bytes": (_sz, [_i, _i, _i]),
    "w4_gptq_quantize": (_i, [_p, _p, _i, _i, _i, _i, ctypes.c_float, _p, _p, _p, _p, _p, _sz,
                              _p]),
    "w4_gptq_hessian": (_i, [_p, _i, _i, _p, _p]),
    "llm_int8_quantize_weights": (_i, [_p, _i, _i, _p, _p, _p]),
    "llm_int8_workspace_bytes": (_sz, [_i, _i, _i]),
    "llm_int8_gemm": (_i, [_p, _p, _p, _i, _i, _i, ctypes.c_float, _p, _p, _sz, _p]),
    "w4_dequant": (_i, [_p, _p, _p, _p, _i, _i, _i, _p, _p]),
    "w4_prepacked_bytes": (_sz, [_i, _i, _i, _i]),
    "w4_prepack": (_i, [_p, _p, _p, _p, _i, _i, _i, _p, _p]),
    "w4_unprepack": (_i, [_p, _i, _i, _i, _i, _p, _p, _p, _p, _p]),
    "w4_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "w4a16_gemm": (_i, [_p, _p, _i, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "w4a16_gemm_static_scratch": (_i, [_p, _p, _i, _i, _i, _i, _i, _p, _p]),
    "w4_awq_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "w4a16_awq_gemm": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "nf4_quantize": (_i, [_p, _i, _i, _i, _i, _p, _p, _p, _p]),
    "nf4_dequant": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _p]),
    "nf4_levels": (None, [_p]),
    "nf4_prepacked_bytes": (_sz, [_i, _i]),
    "nf4_prepack": (_i, [_p, _p, _i, _i, _p, _p]),
    "nf4_workspace_bytes": (_sz, [_i, _i, _i]),
    "nf4_gemm": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "nf4_quantize_meandq": (_i, [_p, _i, _i, _i, _i, _p, _p, _p, _p, _p]),
    "nf4_dequant_meandq": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _p, _p]),
    "nf4_gemm_meandq": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "fp4_quantize": (_i, [_p, _i, _i, _i, _i, _p, _p, _p, _p]),
    "fp4_dequant": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _p]),
    "fp4_levels": (None, [_p]),
    "fp4_gemm": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _p, _sz, _p]),
}
def _bind(handle):
    for name, (res, args) in _SIGS.items():
        f = getattr(handle, name)
        f.restype = res
        f.argtypes = args
    return handle


_bind(lib)
_checked = None


def checked_library():
    """The bounds-checked build (libw4b200_checked.so), loaded on first use;
    ImportError if it has not been built."""
    global _checked
    if _checked is None:
        if not os.path.exists(LIB_CHECKED_PATH):
            raise ImportError(f"{LIB_CHECKED_PATH} is missing: build it with "
                              "`python -m weight_only_bit_gemm_b200.build --checked`")
        _checked = _bind(ctypes.CDLL(LIB_CHECKED_PATH))
    return _checked


@contextlib.contextmanager
def using(handle):
    """Route every wrapper of this module through another build of the
    library (e.g. checked_library()) inside the block."""
    global lib
    saved = lib
    lib = handle
    try:
        yield handle
    finally:
        lib = saved


W4_OK, W4_ERR_INVALID_ARG, W4_ERR_UNSUPPORTED, W4_ERR_CUDA, W4_ERR_TIMEOUT, \
    W4_ERR_DEVICE_INPUT = range(6)
W4_ERR_SCRATCH_LIMIT = 6
W4_ERR_BOUNDS = 7
W4_STATIC_SCRATCH_BYTES = 16 * 1024 * 1024


class W4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib.w4_status_string(status).decode()} ({status})")


def header_functions() -> list:
    """Names of the functions declared in include/w4.h."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(\w+)\s*\(", text)) - {"defined", "if"})


def _check(status: int, what: str) -> None:
    if status != W4_OK:
        raise W4Error(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _cuda(t, dtype, name):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    return t


def device_status() -> int:
    """Synchronise the current stream and return/clear the device error word."""
    return lib.w4_device_status(_stream())


def selftest_wait_timeout() -> None:
    """Run the bounded-wait failure path once (see w4.h); device_status() then
    reports W4_ERR_TIMEOUT."""
    _check(lib.w4_selftest_wait_timeout(_stream()), "w4_selftest_wait_timeout")


# ----------------------------------------------------------------- INT4 RTN

def _quantize_int4(fn, name, W, G, g_idx):
    _cuda(W, torch.float32, "W")
    N, K = W.shape
    dev = W.device
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sc = torch.empty((N, K // G), dtype=torch.float16, device=dev)
    zr = torch.empty((N, K // G), dtype=torch.uint8, device=dev)
    if g_idx is not None:
        _cuda(g_idx, torch.int32, "g_idx")
    _check(fn(_ptr(W), N, K, G, _ptr(g_idx), _ptr(Wq), _ptr(sc), _ptr(zr), _stream()), name)
    return Wq, sc, zr


def quantize_rtn(W, G, g_idx=None):
    """fp32 W [N, K] -> (Wq uint8 [N, K/2], scales fp16 [N, K/G], zeros uint8 [N, K/G])."""
    return _quantize_int4(lib.w4_quantize_rtn, "w4_quantize_rtn", W, G, g_idx)


def quantize_sym(W, G, g_idx=None):
    """Symmetric INT4 (scale max|w|/7, zero point 8), same outputs as quantize_rtn."""
    return _quantize_int4(lib.w4_quantize_sym, "w4_quantize_sym", W, G, g_idx)


def awq_scale_weights(W, s, out=None):
    """fp32 W [N, K] * s [K] (per input channel) in fp32."""
    _cuda(W, torch.float32, "W")
    _cuda(s, torch.float32, "s")
    N, K = W.shape
    if out is None:
        out = torch.empty_like(W)
    _check(lib.w4_awq_scale_weights(_ptr(W), _ptr(s), N, K, _ptr(out), _stream()),
           "w4_awq_scale_weights")
    return out


def awq_scale_activations(X, s, out=None):
    """bf16 X [M, K] / s [K] per input channel, rounded to bf16."""
    _cuda(X, torch.bfloat16, "X")
    _cuda(s, torch.float32, "s")
    M, K = X.shape
    if out is None:
        out = torch.empty_like(X)
    _check(lib.w4_awq_scale_activations(_ptr(X), _ptr(s), M, K, _ptr(out), _stream()),
           "w4_awq_scale_activations")
    return out


def gptq_hessian(X):
    """H = 2 X^T X (fp32 [K, K]) for bf16 calibration activations X [n, K]."""
    _cuda(X, torch.bfloat16, "X")
    n, K = X.shape
    H = torch.empty((K, K), dtype=torch.float32, device=X.device)
    _check(lib.w4_gptq_hessian(_ptr(X), n, K, _ptr(H), _stream()), "w4_gptq_hessian")
    return H


def gptq_quantize(W, H, G, act_order=False, damp=0.01):
    """INT4 codes with GPTQ error compensation: (Wq, scales, zeros, g_idx)
    in the format of quantize_rtn (g_idx None without act-order)."""
    _cuda(W, torch.float32, "W")
    _cuda(H, torch.float32, "H")
    N, K = W.shape
    dev = W.device
    need = lib.w4_gptq_workspace_bytes(N, K, G)
    if need == 0:
        raise W4Error(W4_ERR_INVALID_ARG, "w4_gptq_workspace_bytes")
    ws = _ws_view(torch.empty(need + 256, dtype=torch.uint8, device=dev))
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sc = torch.empty((N, K // G), dtype=torch.float16, device=dev)
    zr = torch.empty((N, K // G), dtype=torch.uint8, device=dev)
    gi = torch.empty(K, dtype=torch.int32, device=dev) if act_order else None
    _check(lib.w4_gptq_quantize(_ptr(W), _ptr(H), N, K, G, int(bool(act_order)), float(damp),
                                _ptr(Wq), _ptr(sc), _ptr(zr), _ptr(gi), _ptr(ws), ws.numel(),
                                _stream()), "w4_gptq_quantize")
    return Wq, sc, zr, gi


def llm_int8_quantize_weights(W):
    """fp32 W [N, K] -> (q_w int8 [N, K], s_w fp32 [N]), one scale per output row."""
    _cuda(W, torch.float32, "W")
    N, K = W.shape
    qw = torch.empty((N, K), dtype=torch.int8, device=W.device)
    sw = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(lib.llm_int8_quantize_weights(_ptr(W), N, K, _ptr(qw), _ptr(sw), _stream()),
           "llm_int8_quantize_weights")
    return qw, sw


def llm_int8_gemm(X, qw, sw, threshold=6.0, out=None, workspace=None):
    """Y = X . W^T by the LLM.int8 mixed decomposition (outliers |x| > threshold)."""
    _cuda(X, torch.bfloat16, "X")
    M, K = X.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    need = lib.llm_int8_workspace_bytes(M, N, K)
    if need == 0:
        raise W4Error(W4_ERR_INVALID_ARG, "llm_int8_workspace_bytes")
    ws = _ws_view(workspace if workspace is not None else _WS_SCRATCH.get(need, X.device))
    _check(lib.llm_int8_gemm(_ptr(X), _ptr(qw), _ptr(sw), M, N, K, float(threshold), _ptr(out),
                             _ptr(ws), ws.numel(), _stream()), "llm_int8_gemm")
    return out


def dequant(Wq, scales, zeros, G, g_idx=None):
    N, K = Wq.shape[0], Wq.shape[1] * 2
    out = torch.empty((N, K), dtype=torch.bfloat16, device=Wq.device)
    _check(lib.w4_dequant(_ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(g_idx), N, K, G, _ptr(out),
                          _stream()), "w4_dequant")
    return out


def prepacked_bytes(N, K, G, act_order=False) -> int:
    return lib.w4_prepacked_bytes(N, K, G, int(bool(act_order)))


def prepack(Wq, scales, zeros, G, g_idx=None):
    N, K = Wq.shape[0], Wq.shape[1] * 2
    nbytes = prepacked_bytes(N, K, G, g_idx is not None)
    if nbytes == 0:
        raise W4Error(W4_ERR_INVALID_ARG, "w4_prepacked_bytes")
    Wp = torch.empty(nbytes, dtype=torch.uint8, device=Wq.device)
    _check(lib.w4_prepack(_ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(g_idx), N, K, G, _ptr(Wp),
                          _stream()), "w4_prepack")
    return Wp


def unprepack(Wp, N, K, G, act_order=False):
    dev = Wp.device
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sc = torch.empty((N, K // G), dtype=torch.float16, device=dev)
    zr = torch.empty((N, K // G), dtype=torch.uint8, device=dev)
    perm = torch.empty(K, dtype=torch.int32, device=dev) if act_order else None
    _check(lib.w4_unprepack(_ptr(Wp), N, K, G, int(bool(act_order)), _ptr(Wq), _ptr(sc),
                            _ptr(zr), _ptr(perm), _stream()), "w4_unprepack")
    return Wq, sc, zr, perm


class Workspace:
    """Per-device scratch buffer, zero-filled once when (re)allocated; the
    library leaves it zeroed after each call."""

    def __init__(self):
        self._buf = {}

    def get(self, nbytes: int, device) -> torch.Tensor:
        dev = torch.device(device)
        key = dev.index if dev.index is not None else torch.cuda.current_device()
        buf = self._buf.get(key)
        if buf is None or buf.numel() < nbytes:
            size = max(nbytes, 1 << 20)
            buf = torch.zeros(size + 256, dtype=torch.uint8, device=dev)
            self._buf[key] = buf
        return buf


_WS = Workspace()
# scratch whose contents the library does not keep zeroed (LLM.int8): never
# the zero-kept workspace of the W4A16 / NF4 GEMMs
_WS_SCRATCH = Workspace()


def _ws_view(buf):
    off = (-buf.data_ptr()) % 256
    return buf[off:]


def workspace_bytes(M, N, K, G, act_order=False) -> int:
    return lib.w4_workspace_bytes(M, N, K, G, int(bool(act_order)))


def w4a16_gemm(X, Wp, N, K, G, act_order=False, out=None, workspace=None):
    """Y[M, N] = X . dequant(W)^T for bf16 X [M, K] and prepacked Wp."""
    _cuda(X, torch.bfloat16, "X")
    M = X.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    need = workspace_bytes(M, N, K, G, act_order)
    ws = _ws_view(workspace if workspace is not None else _WS.get(need, X.device))
    _check(lib.w4a16_gemm(_ptr(X), _ptr(Wp), M, N, K, G, int(bool(act_order)), _ptr(out),
                          _ptr(ws), ws.numel(), _stream()), "w4a16_gemm")
    return out


def w4a16_gemm_static_scratch(X, Wp, N, K, G, act_order=False, out=None):
    """w4a16_gemm with the library's static device scratch as workspace (the
    call allocates nothing); shapes needing more than W4_STATIC_SCRATCH_BYTES
    raise W4Error with status W4_ERR_SCRATCH_LIMIT."""
    _cuda(X, torch.bfloat16, "X")
    M = X.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _check(lib.w4a16_gemm_static_scratch(_ptr(X), _ptr(Wp), M, N, K, G, int(bool(act_order)),
                                         _ptr(out), _stream()), "w4a16_gemm_static_scratch")
    return out


def awq_workspace_bytes(M, N, K, G, act_order=False) -> int:
    return lib.w4_awq_workspace_bytes(M, N, K, G, int(bool(act_order)))


def w4a16_awq_gemm(X, s, Wp, N, K, G, act_order=False, out=None, workspace=None):
    """Y[M, N] = (X / s) . dequant(W s)^T for bf16 X [M, K], the AWQ factor
    s [K] and prepacked Wp of weights quantized after awq_scale_weights."""
    _cuda(X, torch.bfloat16, "X")
    _cuda(s, torch.float32, "s")
    M = X.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    need = awq_workspace_bytes(M, N, K, G, act_order)
    ws = _ws_view(workspace if workspace is not None else _WS.get(need, X.device))
    _check(lib.w4a16_awq_gemm(_ptr(X), _ptr(s), _ptr(Wp), M, N, K, G, int(bool(act_order)),
                              _ptr(out), _ptr(ws), ws.numel(), _stream()), "w4a16_awq_gemm")
    return out


# ----------------------------------------------------------------- NF4

def _levels(fn):
    buf = (ctypes.c_float * 16)()
    fn(ctypes.cast(buf, ctypes.c_void_p))
    return list(buf)


def nf4_levels():
    return _levels(lib.nf4_levels)


def fp4_levels():
    return _levels(lib.fp4_levels)


def _blockwise_quantize(fn, name, W, blocksize, dq_group):
    _cuda(W, torch.float32, "W")
    N, K = W.shape
    dev = W.device
    nb = N * K // blocksize
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    aq = torch.empty(nb, dtype=torch.uint8, device=dev)
    s2 = torch.empty((nb + dq_group - 1) // dq_group, dtype=torch.float32, device=dev)
    _check(fn(_ptr(W), N, K, blocksize, dq_group, _ptr(Wq), _ptr(aq), _ptr(s2), _stream()), name)
    return Wq, aq, s2


def _blockwise_dequant(fn, name, Wq, absmax_q, s2, dq_group, blocksize):
    N, K = Wq.shape[0], Wq.shape[1] * 2
    out = torch.empty((N, K), dtype=torch.bfloat16, device=Wq.device)
    _check(fn(_ptr(Wq), _ptr(absmax_q), _ptr(s2), N, K, blocksize, dq_group, _ptr(out),
              _stream()), name)
    return out


def nf4_quantize(W, blocksize=64, dq_group=256):
    return _blockwise_quantize(lib.nf4_quantize, "nf4_quantize", W, blocksize, dq_group)


def nf4_dequant(Wq, absmax_q, s2, dq_group=256, blocksize=64):
    return _blockwise_dequant(lib.nf4_dequant, "nf4_dequant", Wq, absmax_q, s2, dq_group,
                              blocksize)


def nf4_quantize_meandq(W, blocksize=64, dq_group=256):
    """NF4 with mean-offset double quantization of the block constants:
    (Wq, absmax codes int8, run means fp32, s2 fp32)."""
    _cuda(W, torch.float32, "W")
    N, K = W.shape
    dev = W.device
    nb = N * K // blocksize
    runs = (nb + dq_group - 1) // dq_group
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    aq = torch.empty(nb, dtype=torch.int8, device=dev)
    mean = torch.empty(runs, dtype=torch.float32, device=dev)
    s2 = torch.empty(runs, dtype=torch.float32, device=dev)
    _check(lib.nf4_quantize_meandq(_ptr(W), N, K, blocksize, dq_group, _ptr(Wq), _ptr(aq),
                                   _ptr(mean), _ptr(s2), _stream()), "nf4_quantize_meandq")
    return Wq, aq, mean, s2


def nf4_dequant_meandq(Wq, absmax_q, mean, s2, dq_group=256, blocksize=64):
    N, K = Wq.shape[0], Wq.shape[1] * 2
    out = torch.empty((N, K), dtype=torch.bfloat16, device=Wq.device)
    _check(lib.nf4_dequant_meandq(_ptr(Wq), _ptr(absmax_q), _ptr(mean), _ptr(s2), N, K,
                                  blocksize, dq_group, _ptr(out), _stream()),
           "nf4_dequant_meandq")
    return out


def nf4_gemm_meandq(X, Wp, mean, s2, N, K, dq_group=256, out=None, workspace=None):
    """Y = X . w_hat^T for NF4 weights with mean-offset constants (Wp from
    nf4_prepack of the codes and the int8 constants)."""
    _cuda(X, torch.bfloat16, "X")
    M = X.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    need = nf4_workspace_bytes(M, N, K)
    ws = _ws_view(workspace if workspace is not None else _WS.get(need, X.device))
    _check(lib.nf4_gemm_meandq(_ptr(X), _ptr(Wp), _ptr(mean), _ptr(s2), M, N, K, dq_group,
                               _ptr(out), _ptr(ws), ws.numel(), _stream()), "nf4_gemm_meandq")
    return out


def fp4_quantize(W, blocksize=64, dq_group=256):
    """FP4 (E2M1 / 6) codes in the NF4 block-wise layout: (Wq, absmax codes, s2)."""
    return _blockwise_quantize(lib.fp4_quantize, "fp4_quantize", W, blocksize, dq_group)


def fp4_dequant(Wq, absmax_q, s2, dq_group=256, blocksize=64):
    return _blockwise_dequant(lib.fp4_dequant, "fp4_dequant", Wq, absmax_q, s2, dq_group,
                              blocksize)


def nf4_prepack(Wq, absmax_q):
    """Prepack NF4 or FP4 codes (the layout is shared)."""
    N, K = Wq.shape[0], Wq.shape[1] * 2
    nbytes = lib.nf4_prepacked_bytes(N, K)
    if nbytes == 0:
        raise W4Error(W4_ERR_INVALID_ARG, "nf4_prepacked_bytes")
    Wp = torch.empty(nbytes, dtype=torch.uint8, device=Wq.device)
    _check(lib.nf4_prepack(_ptr(Wq), _ptr(absmax_q), N, K, _ptr(Wp), _stream()), "nf4_prepack")
    return Wp


def nf4_workspace_bytes(M, N, K) -> int:
    return lib.nf4_workspace_bytes(M, N, K)


def _blockwise_gemm(fn, name, X, Wp, s2, N, K, dq_group, out, workspace):
    _cuda(X, torch.bfloat16, "X")
    M = X.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    need = nf4_workspace_bytes(M, N, K)
    ws = _ws_view(workspace if workspace is not None else _WS.get(need, X.device))
    _check(fn(_ptr(X), _ptr(Wp), _ptr(s2), M, N, K, dq_group, _ptr(out), _ptr(ws), ws.numel(),
              _stream()), name)
    return out


def nf4_gemm(X, Wp, s2, N, K, dq_group=256, out=None, workspace=None):
    return _blockwise_gemm(lib.nf4_gemm, "nf4_gemm", X, Wp, s2, N, K, dq_group, out, workspace)


def fp4_gemm(X, Wp, s2, N, K, dq_group=256, out=None, workspace=None):
    """Y = X . w_hat^T for FP4 weights prepacked with nf4_prepack."""
    return _blockwise_gemm(lib.fp4_gemm, "fp4_gemm", X, Wp, s2, N, K, dq_group, out, workspace)
