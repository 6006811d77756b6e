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


def test_noalloc_replans_splits_that_do_not_fit(zq):
    # The automatic plan for 256 tokens x 4096 outputs x K = 16384 splits K
    # four ways (16 MiB of partial sums); the allocation-free call plans again
    # with as many splits as its fixed array holds and gives the same result.
    ops = _operands(zq, 256, 4096, 16384, 64, 11)
    y_ref, acc_ref = _call(zq, "zq_gemm_w8a8", *ops)
    for _ in range(2):
        y, acc = _call(zq, "zq_gemm_w8a8_noalloc", *ops)
        _assert_same(y, acc, y_ref, acc_ref)
    assert zq.device_status()[0] == zq.ZQ_OK


_FRESH = r"""
import sys, torch
sys.path.insert(0, {root!r})
from int4_quantized_transformer_b200 import zq
T, N, K, g = 64, 4096, 8192, 64
Xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, device="cuda")
st = torch.rand(T, device="cuda")
Wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda")
sg = torch.rand(g, device="cuda")
outs = [torch.empty((T, N), dtype=torch.float16, device="cuda") for _ in range(3)]
s = torch.cuda.current_stream().cuda_stream

def call(name, Y):
    rc = getattr(zq.lib(), name)(Xq.data_ptr(), st.data_ptr(), Wq.data_ptr(), sg.data_ptr(), g,
                                 None, T, N, K, Y.data_ptr(), None, s)
    assert rc == zq.ZQ_OK, zq.status_str(rc)
    torch.cuda.synchronize()

torch.cuda.synchronize()
# The library links its own CUDA runtime, which loads the library's device
# code (the fixed scratch array included) at its first call: make that call
# (a status query, no GEMM and no allocation) before measuring.
assert zq.device_status()[0] == zq.ZQ_OK
with zq.options(path=2, split_k=4):  # 4 x 64 x 4096 int32 partial sums = 4 MiB
    free0 = torch.cuda.mem_get_info()[0]
    call("zq_gemm_w8a8_noalloc", outs[0])
    call("zq_gemm_w8a8_noalloc", outs[1])
    free1 = torch.cuda.mem_get_info()[0]
    call("zq_gemm_w8a8", outs[2])  # the allocating entry point: its workspace shows
    free2 = torch.cuda.mem_get_info()[0]
assert torch.equal(outs[0], outs[2]) and torch.equal(outs[1], outs[2])
print(free0, free1, free2)
"""


def test_noalloc_first_call_in_a_fresh_process_allocates_nothing():
    """In a fresh process whose kernels are all loaded up front (after one
    status query), the first GEMM call of the library is an allocation-free
    call at a split-K shape:
    the device's free memory is the same before and after it (and after a
    second one), while the allocating entry point's split-K workspace, 4 MiB
    here, does show up afterwards."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, CUDA_MODULE_LOADING="EAGER")
    out = subprocess.run([sys.executable, "-c", _FRESH.format(root=root)], env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-3000:]
    free0, free1, free2 = (int(v) for v in out.stdout.split()[-3:])
    assert free1 == free0, (free0, free1)
    assert free2 <= free1 - 4 * 1024 * 1024, (free1, free2)
