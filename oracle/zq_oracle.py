"""ctypes front end of the plain C oracle (``zq_oracle.c``).

TEST INFRASTRUCTURE ONLY: loaded by tests, the smoke check and the bench's
CPU-baseline leg, never by the product path.

Every function takes and returns NumPy arrays; fp16 tensors are
``numpy.float16`` arrays whose bit patterns cross into C as uint16.  Each
wrapper names the passage of "ZeroQuant: Efficient and Affordable
Post-Training Quantization for Large-Scale Transformers" (arXiv 2206.01861,
section-by-section summary page, Section 3.4) that the C function follows.

Parity note: every function here is pinned by a test in
``tests/test_oracle_pins.py`` against what the paper and the mathematics fix
(error bounds, exact round trips, brute force, library routines); the op
order and rounding choices listed in the C file header (R1..R9) are readings,
not pinned by the paper.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zq_oracle.c")
_LIB = os.path.join(_HERE, "libzq_oracle.so")

CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile ``zq_oracle.c`` into ``libzq_oracle.so`` next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        # ZQ_ORACLE_LIB loads another build of this same C source: the
        # mutation test plants a mistake in a copy of the oracle and checks
        # that the pins reject it.
        path = os.environ.get("ZQ_ORACLE_LIB")
        if not path:
            path = build()
        _lib = _bind(ctypes.CDLL(path))
    return _lib


def _bind(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.zqo_group_of.argtypes = [I, I, I]
    lib.zqo_group_of.restype = I
    lib.zqo_quantize_weights_groupwise.argtypes = [P, I, I, I, I, P, P]
    lib.zqo_pack_int4.argtypes = [P, I, I, P]
    lib.zqo_unpack_int4.argtypes = [P, I, I, P]
    lib.zqo_ln_row_stats.argtypes = [P, I, ctypes.c_float, P, P, P, P]
    lib.zqo_ln_row_stats.restype = None
    lib.zqo_layernorm.argtypes = [P, P, P, I, I, ctypes.c_float, P]
    lib.zqo_token_quant.argtypes = [P, I, I, P, P]
    lib.zqo_ln_quant.argtypes = [P, P, P, I, I, ctypes.c_float, P, P, P]
    lib.zqo_gemm_i32.argtypes = [P, P, I, I, I, P]
    lib.zqo_gelu.argtypes = [ctypes.c_double]
    lib.zqo_gelu.restype = ctypes.c_double
    lib.zqo_bias_act_quant.argtypes = [P, P, I, I, I, P, P, P]
    lib.zqo_static_calibrate.argtypes = [P, I, I, I, ctypes.c_float, P]
    lib.zqo_static_quant.argtypes = [P, I, I, ctypes.c_float, P, P]
    lib.zqo_dequant.argtypes = [P, P, P, I, P, I, I, P]
    lib.zqo_linear_q.argtypes = [P, P, P, P, I, P, I, I, I, P]
    lib.zqo_gemm_a16.argtypes = [P, P, P, I, P, I, I, I, P, P, P]
    lib.zqo_rounding_is_nearest.argtypes = []
    for f in ("zqo_quantize_weights_groupwise", "zqo_pack_int4", "zqo_unpack_int4",
              "zqo_layernorm", "zqo_token_quant", "zqo_ln_quant", "zqo_bias_act_quant",
              "zqo_static_calibrate", "zqo_static_quant", "zqo_gemm_i32",
              "zqo_dequant", "zqo_linear_q", "zqo_rounding_is_nearest"):
        getattr(lib, f).restype = I
    return lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _h(a, shape=None):
    a = np.ascontiguousarray(a, dtype=np.float16)
    if shape is not None:
        assert a.shape == tuple(shape), (a.shape, shape)
    return a


def _check(rc, what):
    if rc == -2:
        raise OverflowError(f"{what}: an accumulator does not fit int32")
    if rc != 0:
        raise ValueError(f"{what}: bad arguments (rc={rc})")


def group_of(o: int, N: int, g: int) -> int:
    """Group of output row ``o``: floor(o*g/N) (g contiguous row groups, Sec. 3.4
    "Group-wise Weight Quantization"; uneven groups when g does not divide N)."""
    return _L().zqo_group_of(o, N, g)


def group_index(N: int, g: int) -> np.ndarray:
    return np.array([group_of(o, N, g) for o in range(N)], dtype=np.int64)


def quantize_weights_groupwise(W, g: int, bits: int):
    """Sec. 3.4 "Group-wise Weight Quantization" with Eq. 2: one symmetric scale
    per group of contiguous output rows.  Returns (q int8 [N,K], s_grp fp32 [g])."""
    W = _h(W)
    N, K = W.shape
    q = np.empty((N, K), np.int8)
    s = np.empty(g, np.float32)
    _check(_L().zqo_quantize_weights_groupwise(_p(W), N, K, g, bits, _p(q), _p(s)), "wquant")
    return q, s


def pack_int4(q):
    """Two signed INT4 weights per byte: of each eight consecutive k, byte i
    holds k = i in its low nibble and k = 4 + i in its high nibble (reading of
    the paper's W4 storage, Sec. 3.4 "Which weights get INT4")."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    N, K = q.shape
    out = np.empty((N, K // 2), np.uint8)
    _check(_L().zqo_pack_int4(_p(q), N, K, _p(out)), "pack_int4")
    return out


def unpack_int4(packed, K: int):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    q = np.empty((N, K), np.int8)
    _check(_L().zqo_unpack_int4(_p(packed), N, K, _p(q)), "unpack_int4")
    return q


def ln_row_stats(x, eps: float = 1e-5):
    """(mean fp32, rstd fp32, mean, biased var) of one fp16 row (fp32 values)."""
    x = _h(x)
    m = ctypes.c_float()
    r = ctypes.c_float()
    md = ctypes.c_double()
    vd = ctypes.c_double()
    _L().zqo_ln_row_stats(_p(x), x.size, ctypes.c_float(eps), ctypes.byref(m), ctypes.byref(r),
                          ctypes.byref(md), ctypes.byref(vd))
    return np.float32(m.value), np.float32(r.value), md.value, vd.value


def layernorm(X, gamma=None, beta=None, eps: float = 1e-5):
    """Unfused LayerNorm to fp16 (Fig. 2 left, first box).  gamma=None is the
    quant-only mode: the row passes through unchanged."""
    X = _h(X)
    T, K = X.shape
    Y = np.empty((T, K), np.float16)
    g = None if gamma is None else _h(gamma, (K,))
    b = None if beta is None else _h(beta, (K,))
    _check(_L().zqo_layernorm(_p(X), _p(g), _p(b), T, K, ctypes.c_float(eps), _p(Y)), "layernorm")
    return Y


def token_quant(Y):
    """Sec. 3.4 "Token-wise Activation Quantization": one scale per token row.
    Returns (q int8 [T,K], s_tok fp32 [T])."""
    Y = _h(Y)
    T, K = Y.shape
    q = np.empty((T, K), np.int8)
    s = np.empty(T, np.float32)
    _check(_L().zqo_token_quant(_p(Y), T, K, _p(q), _p(s)), "token_quant")
    return q, s


def ln_quant(X, gamma=None, beta=None, eps: float = 1e-5, want_y: bool = False):
    """Fused LN + token quantization (Fig. 2 right, first box; Sec. 3.4
    "Kernel fusion for token-wise activation quantization").
    Returns (q, s_tok) or (q, s_tok, y_ln)."""
    X = _h(X)
    T, K = X.shape
    q = np.empty((T, K), np.int8)
    s = np.empty(T, np.float32)
    y = np.empty((T, K), np.float16) if want_y else None
    g = None if gamma is None else _h(gamma, (K,))
    b = None if beta is None else _h(beta, (K,))
    _check(_L().zqo_ln_quant(_p(X), _p(g), _p(b), T, K, ctypes.c_float(eps), _p(q), _p(s), _p(y)),
           "ln_quant")
    return (q, s, y) if want_y else (q, s)


ACT_NONE, ACT_GELU = 0, 1


def gelu(v: float) -> float:
    """GeLU, exact (erf) form, in double (reading R13)."""
    return float(_L().zqo_gelu(float(v)))


def bias_act_quant(X, bias=None, act: int = ACT_NONE, want_y: bool = False):
    """The token quantization fused into a bias-add (act = ACT_NONE) or a GeLU
    (act = ACT_GELU) (Sec. 3.4 "Kernel fusion for token-wise activation
    quantization"; readings R12 / R13).  Returns (q, s_tok) or (q, s_tok, y)."""
    X = _h(X)
    T, K = X.shape
    q = np.empty((T, K), np.int8)
    s = np.empty(T, np.float32)
    y = np.empty((T, K), np.float16) if want_y else None
    b = None if bias is None else _h(bias, (K,))
    _check(_L().zqo_bias_act_quant(_p(X), _p(b), T, K, int(act), _p(q), _p(s), _p(y)),
           "bias_act_quant")
    return (q, s, y) if want_y else (q, s)


def static_calibrate(batches, momentum: float = 0.95) -> float:
    """Static PTQ calibration (reading R14): moving averages of each batch's
    max and min; returns the range A = max(|x_max|, |x_min|).  batches is
    [nb, T, K] fp16."""
    Xb = np.ascontiguousarray(batches, dtype=np.float16)
    nb, T, K = Xb.shape
    A = np.empty(1, np.float32)
    _check(_L().zqo_static_calibrate(_p(Xb), nb, T, K, ctypes.c_float(momentum), _p(A)),
           "static_calibrate")
    return float(A[0])


def static_quant(X, A: float):
    """Static (per-tensor) quantization with range A (R14): every token uses
    s = A/127.  Returns (q int8 [T,K], s_tok fp32 [T])."""
    X = _h(X)
    T, K = X.shape
    q = np.empty((T, K), np.int8)
    s = np.empty(T, np.float32)
    _check(_L().zqo_static_quant(_p(X), T, K, ctypes.c_float(A), _p(q), _p(s)), "static_quant")
    return q, s


def gemm_i32(xq, wq):
    """INT8 x INT8 -> INT32 accumulator, acc[t,o] = sum_k xq[t,k]*wq[o,k]
    (Sec. 3.4 "Dequantization fused into the GEMM epilogue": the INT32 result)."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    T, K = xq.shape
    N, K2 = wq.shape
    assert K == K2
    acc = np.empty((T, N), np.int32)
    _check(_L().zqo_gemm_i32(_p(xq), _p(wq), T, N, K, _p(acc)), "gemm_i32")
    return acc


def dequant(acc, s_tok, s_grp, bias=None):
    """INT32 -> fp16 by token scale x group scale (+ bias), Sec. 3.4 epilogue."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    T, N = acc.shape
    s_tok = np.ascontiguousarray(s_tok, dtype=np.float32)
    s_grp = np.ascontiguousarray(s_grp, dtype=np.float32)
    b = None if bias is None else _h(bias, (N,))
    Y = np.empty((T, N), np.float16)
    _check(_L().zqo_dequant(_p(acc), _p(s_tok), _p(s_grp), s_grp.size, _p(b), T, N, _p(Y)), "dequant")
    return Y


def linear_q(xq, s_tok, wq, s_grp, bias=None):
    """GEMM + dequant without an INT32 buffer (Fig. 2 right, second box)."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    T, K = xq.shape
    N = wq.shape[0]
    s_tok = np.ascontiguousarray(s_tok, dtype=np.float32)
    s_grp = np.ascontiguousarray(s_grp, dtype=np.float32)
    b = None if bias is None else _h(bias, (N,))
    Y = np.empty((T, N), np.float16)
    _check(_L().zqo_linear_q(_p(xq), _p(s_tok), _p(wq), _p(s_grp), s_grp.size, _p(b), T, N, K, _p(Y)),
           "linear_q")
    return Y


def gemm_a16(X, q, s_grp, bias=None):
    """FP16 activations times group-wise quantized weights (R15; W8A16 and,
    with q = unpack_int4(packed), W4A16): X (q S)^T + b in double.  Returns
    (acc float64 [T,N], y float64 [T,N], Y fp16 [T,N] = fp16(y))."""
    X = _h(X)
    q = np.ascontiguousarray(q, dtype=np.int8)
    T, K = X.shape
    N, K2 = q.shape
    assert K == K2
    s_grp = np.ascontiguousarray(s_grp, dtype=np.float32)
    b = None if bias is None else _h(bias, (N,))
    acc = np.empty((T, N), np.float64)
    y = np.empty((T, N), np.float64)
    Y = np.empty((T, N), np.float16)
    _check(_L().zqo_gemm_a16(_p(X), _p(q), _p(s_grp), s_grp.size, _p(b), T, N, K, _p(acc), _p(y),
                             _p(Y)), "gemm_a16")
    return acc, y, Y


def rounding_is_nearest() -> bool:
    return bool(_L().zqo_rounding_is_nearest())


__all__ = [
    "build", "group_of", "group_index", "quantize_weights_groupwise", "pack_int4", "unpack_int4",
    "ln_row_stats", "layernorm", "token_quant", "ln_quant", "ACT_NONE", "ACT_GELU", "gelu",
    "bias_act_quant", "static_calibrate", "static_quant", "gemm_i32", "dequant", "linear_q",
    "gemm_a16", "rounding_is_nearest",
]
