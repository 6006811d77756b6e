"""Python binding of libzq (ctypes; argument marshalling only).

Every function mirrors one entry point of ``include/zq.h``: it checks the
tensors' device, dtype, shape and contiguity, passes their device pointers
and the current CUDA stream to the C ABI, and raises ``ZQError`` on a
non-zero status.  All arithmetic happens in the CUDA kernels; there is no
CPU or PyTorch fallback, and importing this module without a built
``libzq.so`` raises immediately.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libzq.so")

ZQ_OK, ZQ_ERR_NULL, ZQ_ERR_SHAPE, ZQ_ERR_ALIGN, ZQ_ERR_UNSUPPORTED, ZQ_ERR_CUDA, ZQ_ERR_TIMEOUT = range(7)
OPT_GEMM_PATH, OPT_GEMM_BN, OPT_SPLIT_K, OPT_MAX_CTAS, OPT_CTA_PAIR = 1, 2, 3, 4, 5

EXPORTS = (
    "zq_status_str", "zq_abi_version", "zq_quantize_weights_groupwise", "zq_ln_quant",
    "zq_gemm_w8a8", "zq_gemm_w4a8", "zq_device_status", "zq_set_option", "zq_get_option",
    "zq_debug_wait_timeout", "zq_gemm_w8a8_noalloc", "zq_bias_act_quant", "zq_static_quant",
    "zq_gemm_w8a16", "zq_gemm_w4a16", "zq_launch_count", "zq_workspace_reserve",
    "zq_widen_int4_weights",
)


class ZQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} ({status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libzq.so is not built ({LIB_PATH}); run "
                          "`python -m int4_quantized_transformer_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sig = {
        "zq_status_str": ([I], ctypes.c_char_p),
        "zq_abi_version": ([], I),
        "zq_quantize_weights_groupwise": ([P, I, I, I, I, P, P, P], I),
        "zq_ln_quant": ([P, P, P, I, I, F, P, P, P, P], I),
        "zq_gemm_w8a8": ([P, P, P, P, I, P, I, I, I, P, P, P], I),
        "zq_gemm_w4a8": ([P, P, P, P, I, P, I, I, I, P, P, P], I),
        "zq_device_status": ([P, ctypes.POINTER(I)], I),
        "zq_set_option": ([I, I], I),
        "zq_get_option": ([I], I),
        "zq_debug_wait_timeout": ([P], I),
        "zq_gemm_w8a8_noalloc": ([P, P, P, P, I, P, I, I, I, P, P, P], I),
        "zq_bias_act_quant": ([P, P, I, I, I, P, P, P, P], I),
        "zq_static_quant": ([P, I, I, F, P, P, P], I),
        "zq_gemm_w8a16": ([P, P, P, I, P, I, I, I, P, P, P], I),
        "zq_gemm_w4a16": ([P, P, P, I, P, I, I, I, P, P, P], I),
        "zq_launch_count": ([], ctypes.c_ulonglong),
        "zq_workspace_reserve": ([ctypes.c_ulonglong], I),
        "zq_widen_int4_weights": ([P, I, I, P, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def lib():
    return _lib


def status_str(s: int) -> str:
    return _lib.zq_status_str(int(s)).decode()


def abi_version() -> int:
    return _lib.zq_abi_version()


def _check(rc: int, what: str):
    if rc != ZQ_OK:
        raise ZQError(rc, what)


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dev(t: torch.Tensor | None, dtype, shape, name: str):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def workspace_reserve(nbytes: int):
    """Grow the library workspace of the current device to nbytes now
    (zq_workspace_reserve)."""
    _check(_lib.zq_workspace_reserve(int(nbytes)), "zq_workspace_reserve")


def launch_count() -> int:
    """Kernel launches this library has issued in this process (zq_launch_count)."""
    return int(_lib.zq_launch_count())


def set_option(key: int, value: int):
    _check(_lib.zq_set_option(key, value), "zq_set_option")


def get_option(key: int) -> int:
    return _lib.zq_get_option(key)


class options:
    """Context manager that forces GEMM kernel variants (zq_set_option)."""

    def __init__(self, **kw):
        keys = {"path": OPT_GEMM_PATH, "bn": OPT_GEMM_BN, "split_k": OPT_SPLIT_K,
                "max_ctas": OPT_MAX_CTAS, "pair": OPT_CTA_PAIR}
        self.kw = {keys[k]: v for k, v in kw.items()}

    def __enter__(self):
        self.old = {k: get_option(k) for k in self.kw}
        for k, v in self.kw.items():
            set_option(k, v)
        return self

    def __exit__(self, *exc):
        for k, v in self.old.items():
            set_option(k, v)


def device_status(stream=None) -> tuple[int, int]:
    """Synchronize the stream; return (status, detail) of the device status word."""
    d = ctypes.c_int(0)
    rc = _lib.zq_device_status(_stream(stream), ctypes.byref(d))
    return rc, d.value


def quantize_weights_groupwise(W: torch.Tensor, g: int, bits: int, Wq=None, s_grp=None, stream=None):
    """Group-wise weight quantization (zq_quantize_weights_groupwise).
    Returns (Wq, s_grp): int8 [N,K] (bits 8) or uint8 [N,K/2] (bits 4), fp32 [g]."""
    N, K = W.shape
    if Wq is None:
        Wq = torch.empty((N, K) if bits == 8 else (N, K // 2),
                         dtype=torch.int8 if bits == 8 else torch.uint8, device=W.device)
    if s_grp is None:
        s_grp = torch.empty(g, dtype=torch.float32, device=W.device)
    wq_dtype = torch.int8 if bits == 8 else torch.uint8
    _check(_lib.zq_quantize_weights_groupwise(
        _dev(W, torch.float16, (N, K), "W"), N, K, g, bits,
        _dev(Wq, wq_dtype, (N, K) if bits == 8 else (N, K // 2), "Wq"),
        _dev(s_grp, torch.float32, (g,), "s_grp"), _stream(stream)), "zq_quantize_weights_groupwise")
    return Wq, s_grp


def ln_quant(X: torch.Tensor, gamma=None, beta=None, eps: float = 1e-5, Xq=None, s_tok=None,
             y_ln=None, stream=None):
    """Fused LayerNorm + token-wise INT8 quantization (zq_ln_quant); gamma=None
    is quant-only.  Returns (Xq int8 [T,K], s_tok fp32 [T])."""
    T, K = X.shape
    if Xq is None:
        Xq = torch.empty((T, K), dtype=torch.int8, device=X.device)
    if s_tok is None:
        s_tok = torch.empty(T, dtype=torch.float32, device=X.device)
    _check(_lib.zq_ln_quant(
        _dev(X, torch.float16, (T, K), "X"), _dev(gamma, torch.float16, (K,), "gamma"),
        _dev(beta, torch.float16, (K,), "beta"), T, K, float(eps),
        _dev(Xq, torch.int8, (T, K), "Xq"), _dev(s_tok, torch.float32, (T,), "s_tok"),
        _dev(y_ln, torch.float16, (T, K), "Y_ln"), _stream(stream)), "zq_ln_quant")
    return Xq, s_tok


ACT_NONE, ACT_GELU = 0, 1


def bias_act_quant(X: torch.Tensor, bias=None, act: int = ACT_NONE, Xq=None, s_tok=None, y=None,
                   stream=None):
    """Token-wise INT8 quantization fused into a bias-add (act=ACT_NONE) or a
    GeLU (act=ACT_GELU) (zq_bias_act_quant).  Returns (Xq int8 [T,K],
    s_tok fp32 [T]); y, if given, receives the fp16 activation."""
    T, K = X.shape
    if Xq is None:
        Xq = torch.empty((T, K), dtype=torch.int8, device=X.device)
    if s_tok is None:
        s_tok = torch.empty(T, dtype=torch.float32, device=X.device)
    _check(_lib.zq_bias_act_quant(
        _dev(X, torch.float16, (T, K), "X"), _dev(bias, torch.float16, (K,), "bias"), T, K,
        int(act), _dev(Xq, torch.int8, (T, K), "Xq"), _dev(s_tok, torch.float32, (T,), "s_tok"),
        _dev(y, torch.float16, (T, K), "Y_act"), _stream(stream)), "zq_bias_act_quant")
    return Xq, s_tok


def static_quant(X: torch.Tensor, amax: float, Xq=None, s_tok=None, stream=None):
    """Static (per-tensor) INT8 quantization with a calibrated range amax
    (zq_static_quant).  Returns (Xq int8 [T,K], s_tok fp32 [T] = amax/127)."""
    T, K = X.shape
    if Xq is None:
        Xq = torch.empty((T, K), dtype=torch.int8, device=X.device)
    if s_tok is None:
        s_tok = torch.empty(T, dtype=torch.float32, device=X.device)
    _check(_lib.zq_static_quant(
        _dev(X, torch.float16, (T, K), "X"), T, K, float(amax), _dev(Xq, torch.int8, (T, K), "Xq"),
        _dev(s_tok, torch.float32, (T,), "s_tok"), _stream(stream)), "zq_static_quant")
    return Xq, s_tok


def _gemm(fn, what, Xq, s_tok, Wq, s_grp, bias, N, Y, acc, stream, bits):
    T, K = Xq.shape
    g = s_grp.shape[0]
    if Y is None:
        Y = torch.empty((T, N), dtype=torch.float16, device=Xq.device)
    wshape = (N, K) if bits == 8 else (N, K // 2)
    _check(fn(
        _dev(Xq, torch.int8, (T, K), "Xq"), _dev(s_tok, torch.float32, (T,), "s_tok"),
        _dev(Wq, torch.int8 if bits == 8 else torch.uint8, wshape, "Wq"),
        _dev(s_grp, torch.float32, (g,), "s_grp"), g, _dev(bias, torch.float16, (N,), "bias"),
        T, N, K, _dev(Y, torch.float16, (T, N), "Y"), _dev(acc, torch.int32, (T, N), "acc_dbg"),
        _stream(stream)), what)
    return Y


def gemm_w8a8(Xq, s_tok, Wq, s_grp, bias=None, Y=None, acc_dbg=None, stream=None):
    """Y = fp16(((acc * s_tok) * s_grp[group]) + bias), acc = Xq Wq^T in int32."""
    return _gemm(_lib.zq_gemm_w8a8, "zq_gemm_w8a8", Xq, s_tok, Wq, s_grp, bias, Wq.shape[0], Y,
                 acc_dbg, stream, 8)


def gemm_w4a8(Xq, s_tok, Wq4, s_grp, bias=None, Y=None, acc_dbg=None, stream=None):
    """As gemm_w8a8 with packed INT4 weights uint8 [N, K/2]."""
    return _gemm(_lib.zq_gemm_w4a8, "zq_gemm_w4a8", Xq, s_tok, Wq4, s_grp, bias, Wq4.shape[0], Y,
                 acc_dbg, stream, 4)


def widen_int4_weights(Wq4, K: int, Wq8=None, stream=None):
    """Packed INT4 codes uint8 [N, K/2] -> int8 codes [N, K] (zq_widen_int4_weights)."""
    N = Wq4.shape[0]
    if Wq8 is None:
        Wq8 = torch.empty((N, K), dtype=torch.int8, device=Wq4.device)
    _check(_lib.zq_widen_int4_weights(
        _dev(Wq4, torch.uint8, (N, K // 2), "Wq4"), N, K, _dev(Wq8, torch.int8, (N, K), "Wq8"),
        _stream(stream)), "zq_widen_int4_weights")
    return Wq8


def gemm_w8a8_noalloc(Xq, s_tok, Wq, s_grp, bias=None, Y=None, acc_dbg=None, stream=None):
    """gemm_w8a8 without any device allocation by the library: the split-K
    scratch comes from a fixed array in device memory (zq_gemm_w8a8_noalloc)."""
    return _gemm(_lib.zq_gemm_w8a8_noalloc, "zq_gemm_w8a8_noalloc", Xq, s_tok, Wq, s_grp, bias,
                 Wq.shape[0], Y, acc_dbg, stream, 8)


def _gemm_a16(fn, what, X, Wq, s_grp, bias, N, Y, acc, stream, bits):
    T, K = X.shape
    g = s_grp.shape[0]
    if Y is None:
        Y = torch.empty((T, N), dtype=torch.float16, device=X.device)
    wshape = (N, K) if bits == 8 else (N, K // 2)
    _check(fn(
        _dev(X, torch.float16, (T, K), "X"),
        _dev(Wq, torch.int8 if bits == 8 else torch.uint8, wshape, "Wq"),
        _dev(s_grp, torch.float32, (g,), "s_grp"), g, _dev(bias, torch.float16, (N,), "bias"),
        T, N, K, _dev(Y, torch.float16, (T, N), "Y"), _dev(acc, torch.float32, (T, N), "acc_dbg"),
        _stream(stream)), what)
    return Y


def gemm_w8a16(X, Wq, s_grp, bias=None, Y=None, acc_dbg=None, stream=None):
    """FP16 activations, INT8 weights: Y = fp16(acc * s_grp[group] + bias),
    acc = X Wq^T accumulated in fp32 on the tensor cores."""
    return _gemm_a16(_lib.zq_gemm_w8a16, "zq_gemm_w8a16", X, Wq, s_grp, bias, Wq.shape[0], Y,
                     acc_dbg, stream, 8)


def gemm_w4a16(X, Wq4, s_grp, bias=None, Y=None, acc_dbg=None, stream=None):
    """As gemm_w8a16 with packed INT4 weights uint8 [N, K/2]."""
    return _gemm_a16(_lib.zq_gemm_w4a16, "zq_gemm_w4a16", X, Wq4, s_grp, bias, Wq4.shape[0], Y,
                     acc_dbg, stream, 4)


def debug_wait_timeout(stream=None):
    _check(_lib.zq_debug_wait_timeout(_stream(stream)), "zq_debug_wait_timeout")
