"""The library workspace and CUDA graphs.

A split-K GEMM call keeps its int32 partial sums in the library workspace, a
device buffer the library grows when a call needs more than it holds.  A
graph recorded with that buffer must stay valid when a later call grows the
workspace (the old buffer stays allocated), and a call that would grow it
while its stream is being captured must refuse (ZQ_ERR_UNSUPPORTED) without
breaking the capture.  Run in a fresh process, so that the workspace starts
empty whatever other tests did before.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

_SCRIPT = r"""
import sys, torch
sys.path.insert(0, {root!r})
from int4_quantized_transformer_b200 import zq
gen = torch.Generator().manual_seed(5)
T, N, K, g = 16, 4096, 8192, 64
Xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, generator=gen).cuda()
st = torch.rand(T, generator=gen).cuda()
Wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, generator=gen).cuda()
sg = torch.rand(g, generator=gen).cuda()
b = torch.randn(N, generator=gen).half().cuda()
Y = torch.full((T, N), float("nan"), dtype=torch.float16, device="cuda")
# the library's own CUDA runtime starts up at its first call: make that call
# (a status query) outside any capture
assert zq.device_status()[0] == zq.ZQ_OK
with zq.options(path=2, split_k=4):  # 4 x 16 x 4096 int32 partial sums
    # 1. the first call that needs the workspace is made inside a capture
    refused = None
    g1 = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g1):
            zq.gemm_w8a8(Xq, st, Wq, sg, b, Y=Y)
    except zq.ZQError as e:
        refused = e.status
    assert refused == zq.ZQ_ERR_UNSUPPORTED, refused
    torch.cuda.synchronize()
    assert torch.isnan(Y.float()).all()  # nothing was launched
    # 2. an eager call sizes the workspace; the same call records into a graph
    zq.gemm_w8a8(Xq, st, Wq, sg, b, Y=Y)
    torch.cuda.synchronize()
    ref = Y.clone()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2):
        zq.gemm_w8a8(Xq, st, Wq, sg, b, Y=Y)
    # 3. the workspace grows; the graph still replays into the same result
    zq.workspace_reserve(64 << 20)
    for _ in range(2):
        Y.fill_(float("nan"))
        g2.replay()
        torch.cuda.synchronize()
        assert torch.equal(Y, ref)
    Y.fill_(float("nan"))
    zq.gemm_w8a8(Xq, st, Wq, sg, b, Y=Y)  # eager, on the grown workspace
    torch.cuda.synchronize()
    assert torch.equal(Y, ref)
assert zq.device_status()[0] == zq.ZQ_OK
print("ok")
"""


def test_graph_survives_workspace_growth_and_capture_refuses_growth():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", _SCRIPT.format(root=root)],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-3000:]
    assert out.stdout.split()[-1] == "ok"
