"""The allocation-free GEMM entry point (zq_gemm_w8a8_noalloc).

Callers such as a serving runtime that owns the whole device memory pool, or
a process with a fixed memory budget, cannot let the library call cudaMalloc.
This entry point serves them from a fixed scratch array in device memory.
Its results must equal those of zq_gemm_w8a8, call after call, because the
scratch array keeps whatever the previous call left in it.

This file is collected last so that a run stopping at the first failure has
already run every other test; it passes on its own in a fresh process too.
"""
import numpy as np
import pytest
import torch

from int4_quantized_transformer_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zq():
    from int4_quantized_transformer_b200 import zq as m

    return m


def _operands(zq, T, N, K, g, seed):
    X = synth.activations(T, K, seed=seed, n_outliers=6, outlier_scale=20.0).cuda()
    W = synth.weights(N, K, 0.02, seed=seed + 1).cuda()
    b = synth.bias(N, seed + 2).cuda()
    Wq, sg = zq.quantize_weights_groupwise(W, g, 8)
    Xq, st = zq.ln_quant(X)
    return Xq, st, Wq, sg, b


def _call(zq, fn_name, Xq, st, Wq, sg, b):
    """One call through the C ABI; returns (Y, acc) as host arrays."""
    T, K = Xq.shape
    N = Wq.shape[0]
    Y = torch.full((T, N), float("nan"), dtype=torch.float16, device="cuda")
    acc = torch.zeros((T, N), dtype=torch.int32, device="cuda")
    rc = getattr(zq.lib(), fn_name)(Xq.data_ptr(), st.data_ptr(), Wq.data_ptr(), sg.data_ptr(),
                                    sg.numel(), b.data_ptr(), T, N, K, Y.data_ptr(),
                                    acc.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == zq.ZQ_OK, zq.status_str(rc)
    torch.cuda.synchronize()
    return Y.cpu().numpy(), acc.cpu().numpy()


def _ulp16(v):
    v = np.abs(np.asarray(v, np.float64))
    return 2.0 ** (np.floor(np.log2(np.maximum(v, 2.0 ** -14))) - 10)


def _assert_same(y, acc, y_ref, acc_ref):
    assert np.array_equal(acc, acc_ref)
    r = y_ref.astype(np.float64)
    assert np.all(np.abs(y.astype(np.float64) - r) <= np.maximum(1e-3 * np.abs(r), 2 * _ulp16(r)))
    assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16))


@pytest.mark.parametrize("T,N,K,g", [(8, 1024, 4096, 16), (1, 4096, 4096, 128), (64, 512, 2048, 8)])
def test_noalloc_matches_allocating_entry_point_twice(zq, T, N, K, g):
    # two calls in a row, with different inputs, so a result left in the
    # shared scratch array by the first call cannot pass for the second
    for call, seed in enumerate((T + N, T + N + 50)):
        ops = _operands(zq, T, N, K, g, seed)
        y_ref, acc_ref = _call(zq, "zq_gemm_w8a8", *ops)
        y, acc = _call(zq, "zq_gemm_w8a8_noalloc", *ops)
        _assert_same(y, acc, y_ref, acc_ref)
    assert zq.device_status()[0] == zq.ZQ_OK


def test_noalloc_forced_splits_and_oversize_rejected(zq):
    ops = _operands(zq, 16, 2048, 3072, 32, 7)
    with zq.options(path=2, split_k=6):
        y_ref, acc_ref = _call(zq, "zq_gemm_w8a8", *ops)
        for _ in range(2):
            y, acc = _call(zq, "zq_gemm_w8a8_noalloc", *ops)
            _assert_same(y, acc, y_ref, acc_ref)
    # 2 splits x 256 tokens x 8192 outputs of int32 partial sums exceed the
    # fixed 8 MiB: rejected before anything is launched
    T, N, K = 256, 8192, 1024
    Xq = torch.zeros((T, K), dtype=torch.int8, device="cuda")
    st = torch.zeros(T, dtype=torch.float32, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    sg = torch.zeros(4, dtype=torch.float32, device="cuda")
    Y = torch.zeros((T, N), dtype=torch.float16, device="cuda")
    with zq.options(path=2, split_k=2):
        rc = zq.lib().zq_gemm_w8a8_noalloc(Xq.data_ptr(), st.data_ptr(), Wq.data_ptr(),
                                           sg.data_ptr(), 4, None, T, N, K, Y.data_ptr(), None,
                                           torch.cuda.current_stream().cuda_stream)
    assert rc == zq.ZQ_ERR_SHAPE
    assert zq.device_status()[0] == zq.ZQ_OK
