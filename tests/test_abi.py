"""The C ABI library loads, exports every entry point include/zq.h declares,
and rejects bad arguments synchronously, before anything is launched (these
tests make no compute call and need no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zq.h")


@pytest.fixture(scope="module")
def zq():
    from int4_quantized_transformer_b200 import build

    build.build()
    from int4_quantized_transformer_b200 import zq as m

    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for f in ("zq_quantize_weights_groupwise", "zq_ln_quant", "zq_gemm_w8a8", "zq_gemm_w4a8"):
        assert f in names


def test_library_exports_every_declared_symbol(zq):
    lib = ctypes.CDLL(zq.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", zq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (zq_[a-z0-9_]+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported
    assert set(zq.EXPORTS) == set(declared_functions())


def test_status_strings_and_version(zq):
    assert zq.abi_version() == 105
    for s in range(7):
        assert zq.status_str(s).startswith("ZQ_")
    assert "unknown" in zq.status_str(99)


def test_options_validate(zq):
    L = zq.lib()
    assert L.zq_set_option(99, 1) == zq.ZQ_ERR_UNSUPPORTED
    assert L.zq_set_option(zq.OPT_GEMM_PATH, 5) == zq.ZQ_ERR_SHAPE
    assert L.zq_set_option(zq.OPT_CTA_PAIR, 3) == zq.ZQ_ERR_SHAPE
    assert L.zq_set_option(zq.OPT_GEMM_BN, 100) == zq.ZQ_ERR_SHAPE
    assert L.zq_set_option(zq.OPT_SPLIT_K, -1) == zq.ZQ_ERR_SHAPE
    with zq.options(path=2, split_k=5):
        assert zq.get_option(zq.OPT_GEMM_PATH) == 2 and zq.get_option(zq.OPT_SPLIT_K) == 5
    assert zq.get_option(zq.OPT_GEMM_PATH) == 0 and zq.get_option(zq.OPT_SPLIT_K) == 0


FAKE = 1 << 40  # an aligned address that is never dereferenced: every call below fails validation


@pytest.mark.parametrize("args,expect", [
    # (W, N, K, g, bits, Wq, s_grp)
    ((FAKE, 256, 64, 4, 3, FAKE, FAKE), "UNSUPPORTED"),
    ((FAKE, 256, 64, 0, 8, FAKE, FAKE), "SHAPE"),
    ((FAKE, 256, 64, 257, 8, FAKE, FAKE), "SHAPE"),
    ((FAKE, 256, 40, 4, 8, FAKE, FAKE), "SHAPE"),
    ((FAKE, 256, 48, 4, 4, FAKE, FAKE), "SHAPE"),
    ((None, 256, 64, 4, 8, FAKE, FAKE), "NULL"),
    ((FAKE + 2, 256, 64, 4, 8, FAKE, FAKE), "ALIGN"),
])
def test_wquant_rejects(zq, args, expect):
    rc = zq.lib().zq_quantize_weights_groupwise(*args, None)
    assert rc == getattr(zq, "ZQ_ERR_" + expect)


@pytest.mark.parametrize("args,expect", [
    # (X, gamma, beta, T, K, eps, Xq, s_tok, Y_ln)
    ((FAKE, None, None, 4, 40, 1e-5, FAKE, FAKE, None), "SHAPE"),
    ((FAKE, None, None, 4, 0, 1e-5, FAKE, FAKE, None), "SHAPE"),
    ((FAKE, None, None, 4, 65536, 1e-5, FAKE, FAKE, None), "SHAPE"),
    ((FAKE, None, None, -1, 64, 1e-5, FAKE, FAKE, None), "SHAPE"),
    ((None, None, None, 4, 64, 1e-5, FAKE, FAKE, None), "NULL"),
    ((FAKE, None, None, 4, 64, 1e-5, FAKE, None, None), "NULL"),
    ((FAKE, FAKE + 8, None, 4, 64, 1e-5, FAKE, FAKE, None), "ALIGN"),
    ((FAKE, None, None, 4, 64, 1e-5, FAKE + 1, FAKE, None), "ALIGN"),
])
def test_ln_quant_rejects(zq, args, expect):
    rc = zq.lib().zq_ln_quant(*args, None)
    assert rc == getattr(zq, "ZQ_ERR_" + expect)


@pytest.mark.parametrize("args,expect", [
    # (X, bias, T, K, act, Xq, s_tok, Y_act)
    ((FAKE, None, 4, 64, 2, FAKE, FAKE, None), "UNSUPPORTED"),
    ((FAKE, None, 4, 64, -1, FAKE, FAKE, None), "UNSUPPORTED"),
    ((FAKE, None, 4, 40, 1, FAKE, FAKE, None), "SHAPE"),
    ((FAKE, None, 4, 65536, 0, FAKE, FAKE, None), "SHAPE"),
    ((FAKE, None, -1, 64, 0, FAKE, FAKE, None), "SHAPE"),
    ((None, None, 4, 64, 1, FAKE, FAKE, None), "NULL"),
    ((FAKE, None, 4, 64, 1, FAKE, None, None), "NULL"),
    ((FAKE, FAKE + 8, 4, 64, 0, FAKE, FAKE, None), "ALIGN"),
    ((FAKE, None, 4, 64, 1, FAKE, FAKE, FAKE + 2), "ALIGN"),
])
def test_bias_act_quant_rejects(zq, args, expect):
    rc = zq.lib().zq_bias_act_quant(*args, None)
    assert rc == getattr(zq, "ZQ_ERR_" + expect)


@pytest.mark.parametrize("args,expect", [
    # (X, T, K, amax, Xq, s_tok)
    ((FAKE, 4, 64, -1.0, FAKE, FAKE), "SHAPE"),
    ((FAKE, 4, 64, float("nan"), FAKE, FAKE), "SHAPE"),
    ((FAKE, 4, 64, 1e6, FAKE, FAKE), "SHAPE"),
    ((FAKE, 4, 40, 1.0, FAKE, FAKE), "SHAPE"),
    ((None, 4, 64, 1.0, FAKE, FAKE), "NULL"),
    ((FAKE, 4, 64, 1.0, FAKE, None), "NULL"),
    ((FAKE + 2, 4, 64, 1.0, FAKE, FAKE), "ALIGN"),
])
def test_static_quant_rejects(zq, args, expect):
    rc = zq.lib().zq_static_quant(*args, None)
    assert rc == getattr(zq, "ZQ_ERR_" + expect)


@pytest.mark.parametrize("args,expect", [
    # (Wq4, N, K, Wq8)
    ((FAKE, 0, 64, FAKE), "SHAPE"),
    ((FAKE, 16, 48, FAKE), "SHAPE"),
    ((FAKE, 16, 16, FAKE), "SHAPE"),
    ((None, 16, 64, FAKE), "NULL"),
    ((FAKE, 16, 64, None), "NULL"),
    ((FAKE + 8, 16, 64, FAKE), "ALIGN"),
])
def test_widen_int4_rejects(zq, args, expect):
    rc = zq.lib().zq_widen_int4_weights(*args, None)
    assert rc == getattr(zq, "ZQ_ERR_" + expect)


def test_zero_tokens_is_a_no_op(zq):
    assert zq.lib().zq_bias_act_quant(None, None, 0, 64, 1, None, None, None, None) == zq.ZQ_OK
    assert zq.lib().zq_ln_quant(None, None, None, 0, 64, 1e-5, None, None, None, None) == zq.ZQ_OK
    for fn in ("zq_gemm_w8a8", "zq_gemm_w4a8"):
        assert getattr(zq.lib(), fn)(None, None, None, None, 4, None, 0, 256, 64, None, None,
                                     None) == zq.ZQ_OK


@pytest.mark.parametrize("fn", ["zq_gemm_w8a8", "zq_gemm_w4a8"])
@pytest.mark.parametrize("args,expect", [
    # (Xq, s_tok, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg)
    ((FAKE, FAKE, FAKE, FAKE, 4, None, 16, 250, 64, FAKE, None), "SHAPE"),     # N % 8
    ((FAKE, FAKE, FAKE, FAKE, 4, None, 16, 0, 64, FAKE, None), "SHAPE"),
    ((FAKE, FAKE, FAKE, FAKE, 4, None, 16, 256, 72, FAKE, None), "SHAPE"),     # K % 16
    ((FAKE, FAKE, FAKE, FAKE, 4, None, 16, 256, 133152, FAKE, None), "SHAPE"),  # int32 bound
    ((FAKE, FAKE, FAKE, FAKE, 0, None, 16, 256, 64, FAKE, None), "SHAPE"),
    ((FAKE, FAKE, FAKE, FAKE, 300, None, 16, 256, 64, FAKE, None), "SHAPE"),
    ((FAKE, FAKE, FAKE, FAKE, 4, None, -2, 256, 64, FAKE, None), "SHAPE"),
    ((None, FAKE, FAKE, FAKE, 4, None, 16, 256, 64, FAKE, None), "NULL"),
    ((FAKE, FAKE, FAKE, None, 4, None, 16, 256, 64, FAKE, None), "NULL"),
    ((FAKE, FAKE, FAKE, FAKE, 4, None, 16, 256, 64, None, None), "NULL"),
    ((FAKE, FAKE, FAKE + 4, FAKE, 4, None, 16, 256, 64, FAKE, None), "ALIGN"),
    ((FAKE, FAKE, FAKE, FAKE, 4, FAKE + 2, 16, 256, 64, FAKE, None), "ALIGN"),
    ((FAKE, FAKE, FAKE, FAKE, 4, None, 16, 256, 64, FAKE, FAKE + 4), "ALIGN"),
])
def test_gemm_rejects(zq, fn, args, expect):
    rc = getattr(zq.lib(), fn)(*args, None)
    assert rc == getattr(zq, "ZQ_ERR_" + expect)


@pytest.mark.parametrize("fn", ["zq_gemm_w8a16", "zq_gemm_w4a16"])
@pytest.mark.parametrize("args,expect", [
    # (X, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg)
    ((FAKE, FAKE, FAKE, 4, None, 16, 250, 64, FAKE, None), "SHAPE"),      # N % 8
    ((FAKE, FAKE, FAKE, 4, None, 16, 0, 64, FAKE, None), "SHAPE"),
    ((FAKE, FAKE, FAKE, 4, None, 16, 256, 72, FAKE, None), "SHAPE"),      # K % 16
    ((FAKE, FAKE, FAKE, 4, None, 16, 256, (1 << 20) + 64, FAKE, None), "SHAPE"),
    ((FAKE, FAKE, FAKE, 0, None, 16, 256, 64, FAKE, None), "SHAPE"),
    ((FAKE, FAKE, FAKE, 257, None, 16, 256, 64, FAKE, None), "SHAPE"),
    ((FAKE, FAKE, FAKE, 4, None, -1, 256, 64, FAKE, None), "SHAPE"),
    ((None, FAKE, FAKE, 4, None, 16, 256, 64, FAKE, None), "NULL"),
    ((FAKE, None, FAKE, 4, None, 16, 256, 64, FAKE, None), "NULL"),
    ((FAKE, FAKE, None, 4, None, 16, 256, 64, FAKE, None), "NULL"),
    ((FAKE, FAKE, FAKE, 4, None, 16, 256, 64, None, None), "NULL"),
    ((FAKE + 2, FAKE, FAKE, 4, None, 16, 256, 64, FAKE, None), "ALIGN"),
    ((FAKE, FAKE + 8, FAKE, 4, None, 16, 256, 64, FAKE, None), "ALIGN"),
    ((FAKE, FAKE, FAKE, 4, FAKE + 2, 16, 256, 64, FAKE, None), "ALIGN"),
    ((FAKE, FAKE, FAKE, 4, None, 16, 256, 64, FAKE, FAKE + 4), "ALIGN"),
])
def test_gemm_a16_rejects(zq, fn, args, expect):
    rc = getattr(zq.lib(), fn)(*args, None)
    assert rc == getattr(zq, "ZQ_ERR_" + expect)


def test_gemm_a16_argument_rules(zq):
    L = zq.lib()
    # INT4 weights need K % 32 == 0
    assert L.zq_gemm_w4a16(FAKE, FAKE, FAKE, 4, None, 16, 256, 48, FAKE, None, None) == zq.ZQ_ERR_SHAPE
    # no tokens: nothing to check, nothing launched
    assert L.zq_gemm_w8a16(None, None, None, 4, None, 0, 256, 64, None, None, None) == zq.ZQ_OK
    # the matrix-vector path takes at most four tokens
    with zq.options(path=3):
        assert L.zq_gemm_w8a16(FAKE, FAKE, FAKE, 4, None, 5, 256, 64, FAKE, None,
                               None) == zq.ZQ_ERR_UNSUPPORTED
    # only the 128- and 256-wide tiles exist for FP16 activations
    with zq.options(bn=192):
        assert L.zq_gemm_w8a16(FAKE, FAKE, FAKE, 4, None, 16, 256, 64, FAKE, None,
                               None) == zq.ZQ_ERR_UNSUPPORTED
        # (a T <= 4 call takes the matrix-vector path, where the tile width
        # does not apply: it is not checked here because it would launch)


def test_w4a8_needs_k_multiple_of_32(zq):
    rc = zq.lib().zq_gemm_w4a8(FAKE, FAKE, FAKE, FAKE, 4, None, 16, 256, 48, FAKE, None, None)
    assert rc == zq.ZQ_ERR_SHAPE


def test_binding_refuses_cpu_tensors(zq):
    import torch

    x = torch.zeros(4, 64, dtype=torch.float16)
    with pytest.raises(TypeError):
        zq.ln_quant(x)
