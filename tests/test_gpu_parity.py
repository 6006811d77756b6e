"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Integer outputs (int8 codes, packed int4 bytes, int32 accumulators) and the
fp32 scales must match bit for bit.  fp16 outputs must agree within the
stated tolerance |y - ref| <= max(1e-3 |ref|, 2 ulp16(ref)); both sides run
the same IEEE op sequence, so exact equality is expected and asserted too.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_quantized_transformer_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zq():
    from int4_quantized_transformer_b200 import zq as m

    yield m
    rc, detail = m.device_status()
    assert rc == m.ZQ_OK, f"device status {rc} detail {detail}"


@pytest.fixture(autouse=True)
def _device_status_clean(zq):
    """Every test leaves the device status word clean: a bounded wait that
    ran out anywhere (a drain at kernel exit included) fails the test that
    launched it, even when its outputs were right."""
    yield
    rc, detail = zq.device_status()
    assert rc == zq.ZQ_OK, f"device status {rc} ({zq.status_str(rc)}), wait site {detail}"


def dev(t):
    return t.cuda()


def host(t):
    return t.cpu().numpy()


def ulp16(v):
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -14)))
    return 2.0 ** (e - 10)


def assert_fp16_close(y, ref):
    y64, r64 = y.astype(np.float64), ref.astype(np.float64)
    tol = np.maximum(1e-3 * np.abs(r64), 2 * ulp16(r64))
    bad = np.abs(y64 - r64) > tol
    assert not bad.any(), f"{bad.sum()} fp16 outputs outside tolerance"
    assert np.array_equal(y.view(np.uint16), ref.view(np.uint16)), \
        f"{(y.view(np.uint16) != ref.view(np.uint16)).sum()} fp16 outputs differ in the last bits"


def assert_bits_equal(a, b):
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    assert a.shape == b.shape
    av, bv = a.view(np.uint8), b.view(np.uint8)
    assert np.array_equal(av, bv), f"{(av != bv).sum()} bytes differ"


# ------------------------------------------------------------ weights

@pytest.mark.parametrize("N,K,g,bits", [(256, 64, 4, 8), (1024, 1024, 48, 8), (768, 3072, 48, 8),
                                        (1024, 4096, 64, 4), (96, 64, 7, 4), (64, 32, 64, 4),
                                        (4096, 4096, 128, 8), (2000, 160, 1, 8)])
def test_wquant_bit_exact(zq, N, K, g, bits):
    W = synth.weights(N, K, 0.02, seed=N + K + g)
    W[: N // 10] *= 8  # unequal group ranges
    if g > 2:
        W[N // 2: N // 2 + (N // g)] = 0  # an all-zero stretch of rows
    qd, sd = zq.quantize_weights_groupwise(dev(W), g, bits)
    q, s = oracle.quantize_weights_groupwise(W.numpy(), g, bits)
    if bits == 4:
        q = oracle.pack_int4(q)
    assert_bits_equal(host(sd), s)
    assert_bits_equal(host(qd), q)


# ------------------------------------------------------------ ln_quant

@pytest.mark.parametrize("K", [64, 768, 1024, 3072, 4096, 6144, 16384, 24576])
@pytest.mark.parametrize("mode", ["ln", "ln_no_beta", "quant_only"])
def test_ln_quant_bit_exact(zq, K, mode):
    T = 37
    X = synth.activations(T, K, seed=K, n_outliers=max(1, K // 1000), outlier_scale=30.0)
    gamma, beta = synth.ln_params(K, K + 1)
    if mode == "quant_only":
        gamma = beta = None
    elif mode == "ln_no_beta":
        beta = None
    Xd = dev(X)
    yd = torch.empty_like(Xd)
    qd, sd = zq.ln_quant(Xd, None if gamma is None else dev(gamma),
                         None if beta is None else dev(beta), 1e-5, y_ln=yd)
    q, s, y = oracle.ln_quant(X.numpy(), None if gamma is None else gamma.numpy(),
                              None if beta is None else beta.numpy(), 1e-5, want_y=True)
    assert_bits_equal(host(yd), y)
    assert_bits_equal(host(sd), s)
    assert_bits_equal(host(qd), q)


@pytest.mark.parametrize("kind", ["zero_rows", "constant_rows", "max_values", "tiny_values"])
@pytest.mark.parametrize("with_ln", [True, False])
def test_ln_quant_edge_rows(zq, kind, with_ln):
    T, K = 29, 768
    X = synth.edge_activations(kind, T, K)
    gamma, beta = synth.ln_params(K, 3) if with_ln else (None, None)
    qd, sd = zq.ln_quant(dev(X), None if gamma is None else dev(gamma),
                         None if beta is None else dev(beta), 1e-5)
    q, s = oracle.ln_quant(X.numpy(), None if gamma is None else gamma.numpy(),
                           None if beta is None else beta.numpy(), 1e-5)
    assert_bits_equal(host(sd), s)
    assert_bits_equal(host(qd), q)


@pytest.mark.parametrize("T", [1, 2, 9, 1000])
def test_ln_quant_token_counts(zq, T):
    K = 1024
    X = synth.activations(T, K, seed=T, n_outliers=6, outlier_scale=20.0)
    gamma, beta = synth.ln_params(K, 5)
    qd, sd = zq.ln_quant(dev(X), dev(gamma), dev(beta), 1e-5)
    q, s = oracle.ln_quant(X.numpy(), gamma.numpy(), beta.numpy(), 1e-5)
    assert_bits_equal(host(sd), s)
    assert_bits_equal(host(qd), q)


# ------------------------------------------------------------ GEMM

def _quant_operands(T, N, K, g, bits, seed):
    X = synth.activations(T, K, seed=seed, n_outliers=6, outlier_scale=20.0)
    W = synth.weights(N, K, 0.02, seed=seed + 1)
    b = synth.bias(N, seed + 2)
    xq, st = oracle.ln_quant(X.numpy())
    wq, sg = oracle.quantize_weights_groupwise(W.numpy(), g, bits)
    return xq, st, wq, sg, b.numpy()


def _run_gemm(zq, xq, st, wq, sg, b, bits, **opts):
    T, K = xq.shape
    N = wq.shape[0]
    wdev = torch.from_numpy(oracle.pack_int4(wq) if bits == 4 else wq).cuda()
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    fn = zq.gemm_w4a8 if bits == 4 else zq.gemm_w8a8
    with zq.options(**opts):
        Y = fn(torch.from_numpy(xq).cuda(), torch.from_numpy(st).cuda(), wdev,
               torch.from_numpy(sg).cuda(), None if b is None else torch.from_numpy(b).cuda(),
               acc_dbg=acc)
    return host(Y), host(acc)


def _check_gemm(zq, T, N, K, g, bits, seed=0, bias=True, **opts):
    xq, st, wq, sg, b = _quant_operands(T, N, K, g, bits, seed)
    if not bias:
        b = None
    Y, acc = _run_gemm(zq, xq, st, wq, sg, b, bits, **opts)
    acc_ref = oracle.gemm_i32(xq, wq)
    assert_bits_equal(acc, acc_ref)
    assert_fp16_close(Y, oracle.dequant(acc_ref, st, sg, b))


GEMM_SHAPES = [
    # T, N, K, g
    (16, 256, 64, 4),      # the single-layer configuration
    (1, 256, 64, 4),
    (7, 768, 768, 48),
    (129, 1024, 768, 48),  # ragged token tile
    (300, 768, 784, 48),   # K not a multiple of 128
    (256, 2304, 768, 48),
    (513, 1000, 256, 3),   # N not a multiple of the tile, N % g != 0
]


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("T,N,K,g", GEMM_SHAPES)
def test_gemm_auto(zq, bits, T, N, K, g):
    if bits == 4 and K % 32:
        pytest.skip("int4 needs K % 32 == 0")
    _check_gemm(zq, T, N, K, g, bits, seed=T + N + K)


@pytest.mark.parametrize("T,N,K,g", [(1100, 640, 2048, 5), (130, 512, 2048, 8), (128, 384, 4096, 3),
                                     (2048, 256, 3072, 4), (1024, 1024, 1024, 16),
                                     (511, 768, 1024, 6), (512, 768, 1024, 6)])
def test_gemm_w4_tiling_choices(zq, T, N, K, g):
    """INT4 weights choose weight-row tiles (widened weights in TMEM) up to
    T = 128, token-row tiles below 512 tokens and the widening pass with the
    INT8 GEMM from there; both sides of each boundary, and the forced
    weight-row alternative, match the oracle."""
    _check_gemm(zq, T, N, K, g, 4, seed=T + K)
    _check_gemm(zq, T, N, K, g, 4, seed=T + K + 1, path=2)


@pytest.mark.parametrize("T,N,K,g", [(1, 256, 64, 4), (7, 768, 768, 48), (300, 1000, 512, 3),
                                     (1100, 640, 2048, 5), (2048, 256, 3072, 4),
                                     (513, 2304, 800, 48), (1024, 1024, 1024, 16)])
@pytest.mark.parametrize("pair", [1, 2])
def test_gemm_w4_widened_then_int8(zq, T, N, K, g, pair):
    """INT4 weights widened once into the library workspace (an HBM-bound
    pass), then the INT8 GEMM on the widened codes, single CTAs or CTA pairs;
    automatic from 512 tokens, forced here at every size."""
    _check_gemm(zq, T, N, K, g, 4, seed=T + N + pair, path=4, pair=pair)


@pytest.mark.parametrize("N,K", [(256, 64), (1000, 4160), (24576, 6144), (3, 32)])
def test_widen_int4_weights_bit_exact(zq, N, K):
    """The INT4 unpack step on its own: every widened code equals the oracle's
    unpacking of the packed bytes, and a W8A8 GEMM on the widened codes equals
    the W4A8 GEMM on the packed ones."""
    W = synth.weights(N, K, 0.02, seed=N + K)
    q, _ = oracle.quantize_weights_groupwise(W.numpy(), max(1, N // 64), 4)
    packed = torch.from_numpy(oracle.pack_int4(q)).cuda()
    wide = zq.widen_int4_weights(packed, K)
    assert_bits_equal(host(wide), oracle.unpack_int4(oracle.pack_int4(q), K))
    assert_bits_equal(host(wide), q)
    if N * K <= 1 << 22 and N % 8 == 0:
        xq, st, _, sg, b = _quant_operands(40, N, K, max(1, N // 64), 4, N)
        X, S, B = (torch.from_numpy(a).cuda() for a in (xq, st, b))
        sgd = torch.from_numpy(np.ones(max(1, N // 64), np.float32)).cuda()
        y8 = zq.gemm_w8a8(X, S, wide, sgd, B)
        y4 = zq.gemm_w4a8(X, S, packed, sgd, B)
        assert torch.equal(y8, y4)


def test_gemm_w4_widened_after_a_larger_call_and_reserve(zq):
    """The workspace holds the widened codes of the largest call so far; a
    smaller call after it, and calls after an explicit reservation, still
    match the oracle."""
    zq.workspace_reserve(8 << 20)
    _check_gemm(zq, 1024, 2048, 2048, 8, 4, seed=91)
    _check_gemm(zq, 1030, 520, 1056, 8, 4, seed=92)
    _check_gemm(zq, 8, 1024, 2048, 8, 8, seed=93, path=2, split_k=4)
    _check_gemm(zq, 1024, 2048, 2048, 8, 4, seed=94)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("bn", [128, 192, 256])
@pytest.mark.parametrize("T,N,K", [(16, 256, 64), (300, 1000, 512), (1024, 768, 1024)])
def test_gemm_token_rows_tiles(zq, bits, bn, T, N, K):
    _check_gemm(zq, T, N, K, 8, bits, seed=bn, path=1, bn=bn, pair=1)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("bn", [128, 192, 256])
@pytest.mark.parametrize("T,N,K", [(16, 256, 64), (300, 1000, 512), (1024, 768, 1024),
                                   (513, 2304, 768)])
def test_gemm_cta_pair_tiles(zq, bits, bn, T, N, K):
    """256-row tiles shared by a CTA pair (tcgen05 cta_group::2): each CTA
    loads 128 token rows and half of the weight rows (INT4: and unpacks its
    half); ragged token counts leave the second CTA's rows partly or wholly
    past T."""
    _check_gemm(zq, T, N, K, 8, bits, seed=bn + 1, path=1, bn=bn, pair=2)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("T,N,K,pair", [(2560, 2048, 1024, 2), (2048, 2560, 2048, 1),
                                        (2600, 2056, 1056, 2)])
def test_gemm_last_wave_split(zq, bits, T, N, K, pair):
    """A partial last wave whose tiles are split along K (forced here; automatic
    for long rows), their int32 partial sums added and dequantized by the
    finalize kernel (80 pair units over 74 pair slots, 160 single-CTA units
    over 148 SMs; ragged T, N and K)."""
    _check_gemm(zq, T, N, K, 8, bits, seed=T + K + pair, pair=pair, bn=256, split_k=3)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("split", [1, 2, 3, 7])
@pytest.mark.parametrize("T,N,K", [(1, 512, 1024), (8, 1024, 896), (64, 384, 2048),
                                   (200, 256, 1024), (300, 256, 512)])
def test_gemm_weight_rows_split_k(zq, bits, split, T, N, K):
    _check_gemm(zq, T, N, K, 16, bits, seed=split, path=2, split_k=split)


def test_gemm_persistent_loop_with_few_ctas(zq):
    # fewer CTAs than work units: every CTA walks several units through both
    # TMEM accumulator buffers
    _check_gemm(zq, 640, 1024, 512, 8, 8, seed=3, path=1, bn=128, max_ctas=5, pair=1)
    _check_gemm(zq, 640, 1024, 512, 8, 4, seed=4, path=1, bn=256, max_ctas=3)
    _check_gemm(zq, 1280, 1024, 512, 8, 8, seed=6, path=1, bn=128, max_ctas=4, pair=2)
    _check_gemm(zq, 1000, 2048, 384, 8, 8, seed=7, path=1, bn=256, max_ctas=6, pair=2)
    _check_gemm(zq, 1000, 2048, 384, 8, 4, seed=8, path=1, bn=256, max_ctas=6, pair=2)
    _check_gemm(zq, 16, 2048, 1024, 8, 8, seed=5, path=2, split_k=4, max_ctas=7)


def test_gemm_no_bias_and_extremes(zq):
    # saturated operands: every product is +-127*127 (int8) and accumulators
    # reach +-127*127*K
    T, N, K, g = 64, 256, 4096, 2
    xq = np.full((T, K), 127, np.int8)
    xq[1::2] = -127
    wq = np.full((N, K), 127, np.int8)
    wq[::3] = -127
    st = np.linspace(1e-3, 1e-2, T).astype(np.float32)
    sg = np.array([1e-4, 2e-4], np.float32)
    for bits in (8, 4):
        w = wq if bits == 8 else np.sign(wq).astype(np.int8) * 7
        Y, acc = _run_gemm(zq, xq, st, w, sg, None, bits)
        acc_ref = oracle.gemm_i32(xq, w)
        assert_bits_equal(acc, acc_ref)
        assert_fp16_close(Y, oracle.dequant(acc_ref, st, sg, None))


def test_gemm_zero_scales_give_bias(zq):
    T, N, K, g = 5, 64, 128, 4
    xq, st, wq, sg, b = _quant_operands(T, N, K, g, 8, 11)
    st[:] = 0
    Y, _ = _run_gemm(zq, xq, st, wq, sg, b, 8)
    assert_bits_equal(Y, np.broadcast_to(b, (T, N)))


# ------------------------------------------------------------ bias-add / GeLU + quant

ACT_SHAPES = [(5, 16), (37, 768), (64, 3072), (9, 4096), (3, 16384), (130, 1040)]


def _run_act(zq, X, b, act):
    T, K = X.shape
    y = torch.empty((T, K), dtype=torch.float16, device="cuda")
    xq, st = zq.bias_act_quant(dev(torch.from_numpy(X)), None if b is None else dev(torch.from_numpy(b)),
                               act, y=y)
    return host(xq), host(st), host(y)


@pytest.mark.parametrize("T,K", ACT_SHAPES)
@pytest.mark.parametrize("with_bias", [False, True])
def test_bias_quant_bit_exact(zq, T, K, with_bias):
    """Token quantization fused into a bias-add: every output bit equals the
    oracle's (one fp32 add, fp16 rounding, Eq. 2)."""
    rng = np.random.default_rng(T * 31 + K)
    X = synth.activations(T, K, seed=T + K, n_outliers=6, outlier_scale=20.0).numpy()
    X[0, :8] = np.array([-0.0, 0.0, 65504, -65504, 6e-8, -6e-8, 1.0, -1.0], np.float16)
    b = None
    if with_bias:
        b = (rng.standard_normal(K) * 2).astype(np.float16)
        b[2:4] = 0  # keep x + b finite next to +-65504
    q, s, y = _run_act(zq, X, b, zq.ACT_NONE)
    q_ref, s_ref, y_ref = oracle.bias_act_quant(X, b, oracle.ACT_NONE, want_y=True)
    assert_bits_equal(y, y_ref)
    assert_bits_equal(q, q_ref)
    assert_bits_equal(s, s_ref)


@pytest.mark.parametrize("T,K", ACT_SHAPES)
@pytest.mark.parametrize("with_bias", [False, True])
def test_gelu_quant_matches_oracle(zq, T, K, with_bias):
    """Token quantization fused into a GeLU: y (CUDA's erfcf in fp32) is
    within one fp16 ulp of the oracle's y (fp64, rounded once), and the codes
    and scales are exactly the token quantization of the kernel's own y."""
    rng = np.random.default_rng(T * 17 + K)
    X = (rng.standard_normal((T, K)) * 3).astype(np.float16)
    X[0, :6] = np.array([-0.0, 0.0, -12.0, 12.0, -3.0, 3.0], np.float16)
    b = (rng.standard_normal(K) * 0.5).astype(np.float16) if with_bias else None
    q, s, y = _run_act(zq, X, b, zq.ACT_GELU)
    _, _, y_ref = oracle.bias_act_quant(X, b, oracle.ACT_GELU, want_y=True)
    d = np.abs(y.astype(np.float64) - y_ref.astype(np.float64))
    assert np.all(d <= ulp16(y_ref)), f"max |dy| {d.max()}"
    assert np.mean(y.view(np.uint16) == y_ref.view(np.uint16)) > 0.99
    q_own, s_own = oracle.token_quant(y)
    assert_bits_equal(q, q_own)
    assert_bits_equal(s, s_own)


@pytest.mark.parametrize("T,K", [(5, 16), (64, 768), (33, 3072), (7, 16384)])
@pytest.mark.parametrize("amax", [0.0, 0.75, 3.0, 40.0])
def test_static_quant_bit_exact(zq, T, K, amax):
    """Static per-tensor quantization: one calibrated range for every token,
    codes beyond it clamped; bit-exact against the oracle."""
    X = synth.activations(T, K, seed=T + K, n_outliers=4, outlier_scale=20.0)
    xq, st = zq.static_quant(dev(X), amax)
    q_ref, s_ref = oracle.static_quant(X.numpy(), amax)
    assert_bits_equal(host(xq), q_ref)
    assert_bits_equal(host(st), s_ref)


# ------------------------------------------------------------ matrix-vector path (T <= 4)

@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K,g", [(256, 64, 4), (1000, 4160, 5), (8, 96, 1), (4104, 3072, 24)])
def test_gemv_path(zq, bits, T, N, K, g):
    """The CUDA-core matrix-vector path: weight rows go in pairs per warp
    (the pairs do not fill the last round of warps), K is not a multiple of
    one round of 32 lanes x 3 chunks, a single group, and T = 3 runs in the
    four-token kernel."""
    if bits == 4 and K % 32:
        pytest.skip("int4 needs K % 32 == 0")
    _check_gemm(zq, T, N, K, g, bits, seed=T * 7 + N + K, path=3)


def test_gemv_persistent_rows_and_extremes(zq):
    # fewer CTAs than row pairs: every warp walks several pairs
    _check_gemm(zq, 3, 2048, 1024, 8, 8, seed=21, path=3, max_ctas=3)
    _check_gemm(zq, 4, 2048, 1024, 8, 4, seed=22, path=3, max_ctas=2)
    # saturated operands: accumulators reach +-127*127*K (int8) and the INT4
    # widening multiplies them by 16 before the exact division
    T, N, K = 4, 64, 8192
    xq = np.full((T, K), 127, np.int8)
    xq[1::2] = -127
    st = np.linspace(1e-3, 1e-2, T).astype(np.float32)
    sg = np.array([1e-4, 2e-4], np.float32)
    for bits in (8, 4):
        w = np.full((N, K), 127 if bits == 8 else 7, np.int8)
        w[::3] = -127 if bits == 8 else -8
        Y, acc = _run_gemm(zq, xq, st, w, sg, None, bits, path=3)
        acc_ref = oracle.gemm_i32(xq, w)
        assert_bits_equal(acc, acc_ref)
        assert_fp16_close(Y, oracle.dequant(acc_ref, st, sg, None))


def test_gemv_path_rejects_more_tokens(zq):
    xq, st, wq, sg, b = _quant_operands(5, 64, 64, 2, 8, 1)
    with pytest.raises(zq.ZQError) as e:
        _run_gemm(zq, xq, st, wq, sg, b, 8, path=3)
    assert e.value.status == zq.ZQ_ERR_UNSUPPORTED


def test_repeated_split_k_calls_leave_workspace_clean(zq):
    # the split-K workspace must return to zero after every call
    for i in range(3):
        _check_gemm(zq, 8, 1024, 2048, 8, 8, seed=100 + i, path=2, split_k=8)


# ------------------------------------------------------------ full-size configurations

def _sample_rows(T, n=6):
    """Token rows at every tiling edge of the plans the GEMMs choose, plus
    random ones: the first and last row of 16- to 256-row token tiles around
    the start, of the last 128-row tile and of both 128-row halves of the
    last 256-row CTA-pair tile, and T - 1."""
    edges = {0, T - 1}
    for b in (16, 32, 64, 128, 256, 512):
        edges |= {b - 1, b}
    for tile in (128, 256):
        last = (T - 1) // tile * tile
        edges |= {last - 1, last, min(last + 127, T - 1), last + 128}
    rnd = np.random.default_rng(T).integers(0, T, n)
    return np.array(sorted(r for r in edges | set(int(v) for v in rnd) if 0 <= r < T))


FULL = [(layer, gi, T) for layer in ("bert_base", "gpt350m", "gptj6b", "neox20b")
        for gi in range(4) for T in synth.LAYERS[layer].tokens]


@pytest.mark.parametrize("layer,gi,T", FULL)
def test_full_size_sampled_rows(zq, layer, gi, T):
    """Every GEMM of every layer configuration at its full size, in the launch
    configuration the benchmark uses; the oracle recomputes sampled token
    rows (each row depends only on its own activations and all weights)."""
    inp = synth.gemm_inputs(layer, gi, T)
    s = inp.spec
    Xd, Wd, bd = dev(inp.X), dev(inp.W), dev(inp.b)
    gd = None if inp.gamma is None else dev(inp.gamma)
    betad = None if inp.beta is None else dev(inp.beta)
    wq_d, sg_d = zq.quantize_weights_groupwise(Wd, s.g, s.bits)
    xq_d, st_d = zq.ln_quant(Xd, gd, betad, 1e-5)
    acc_d = torch.empty((T, s.N), dtype=torch.int32, device="cuda")
    fn = zq.gemm_w4a8 if s.bits == 4 else zq.gemm_w8a8
    Y_d = fn(xq_d, st_d, wq_d, sg_d, bd, acc_dbg=acc_d)

    wq, sg = oracle.quantize_weights_groupwise(inp.W.numpy(), s.g, s.bits)
    assert_bits_equal(host(sg_d), sg)
    assert_bits_equal(host(wq_d), oracle.pack_int4(wq) if s.bits == 4 else wq)
    rows = _sample_rows(T)
    Xs = inp.X.numpy()[rows]
    xq, st = oracle.ln_quant(Xs, None if inp.gamma is None else inp.gamma.numpy(),
                             None if inp.beta is None else inp.beta.numpy(), 1e-5)
    assert_bits_equal(host(xq_d)[rows], xq)
    assert_bits_equal(host(st_d)[rows], st)
    acc = oracle.gemm_i32(xq, wq)
    assert_bits_equal(host(acc_d)[rows], acc)
    assert_fp16_close(host(Y_d)[rows], oracle.dequant(acc, st, sg, inp.b.numpy()))
    if layer == "neox20b" and T == 4096 and s.bits == 4:
        # INT4 weights at prefill size: every token of the first and the last
        # 128-row weight tile (one output stripe each), against the oracle
        xq_all, st_all = oracle.ln_quant(inp.X.numpy(),
                                         None if inp.gamma is None else inp.gamma.numpy(),
                                         None if inp.beta is None else inp.beta.numpy(), 1e-5)
        assert_bits_equal(host(xq_d), xq_all)
        for c0 in (0, s.N - 128):
            cols = slice(c0, c0 + 128)
            acc_s = oracle.gemm_i32(xq_all, wq[cols])
            assert_bits_equal(host(acc_d)[:, cols], acc_s)
            sg_cols = sg[oracle.group_index(s.N, s.g)[cols]]
            ref = oracle.dequant(acc_s, st_all, sg_cols, inp.b.numpy()[cols])
            assert_fp16_close(host(Y_d)[:, cols], ref)


# ------------------------------------------------------------ FP16 activations (W8A16 / W4A16)
#
# The tensor cores sum fp16 x code products in fp32 in their own order, so the
# GPU accumulator is compared with the oracle's double sum within the bound of
# fp32 summation in any order, |acc - acc64| <= 2 K 2^-24 sum_k |x q| (the
# factor 2 also covers adders that truncate), and Y within that bound times
# the group scale, plus the two fp32 roundings of the epilogue and half an
# fp16 ulp for the final rounding.

def _assert_a16_close(X, q, sg, acc, Y, acc_ref, y_ref, Y_ref, min_equal=0.8):
    T, K = X.shape
    N = q.shape[0]
    mag = np.abs(X.astype(np.float64)) @ np.abs(q.astype(np.float64)).T
    e_acc = 2.0 * K * 2.0 ** -24 * mag
    bad = np.abs(acc.astype(np.float64) - acc_ref) > e_acc
    assert not bad.any(), f"{bad.sum()} accumulators outside the fp32 summation bound"
    s = sg.astype(np.float64)[np.arange(N) * sg.size // N][None, :]
    y = Y.astype(np.float64)
    tol = (e_acc * s + 2.0 ** -23 * (np.abs(acc_ref * s) + np.abs(y_ref))
           + 0.5 * ulp16(np.maximum(np.abs(y), np.abs(y_ref))))
    bad = np.abs(y - y_ref) > tol
    assert not bad.any(), f"{bad.sum()} fp16 outputs outside the tolerance"
    equal = np.mean(Y.view(np.uint16) == Y_ref.view(np.uint16))
    assert equal >= min_equal, f"only {equal:.3f} of the outputs equal the correctly rounded value"


def _check_a16(zq, T, N, K, g, bits, seed=0, bias=True, **opts):
    X = synth.activations(T, K, seed=seed, n_outliers=6, outlier_scale=20.0)
    W = synth.weights(N, K, 0.02, seed=seed + 1)
    b = synth.bias(N, seed + 2) if bias else None
    wq, sg = oracle.quantize_weights_groupwise(W.numpy(), g, bits)
    wdev = torch.from_numpy(oracle.pack_int4(wq) if bits == 4 else wq).cuda()
    acc_d = torch.empty((T, N), dtype=torch.float32, device="cuda")
    fn = zq.gemm_w4a16 if bits == 4 else zq.gemm_w8a16
    with zq.options(**opts):
        Y = fn(dev(X), wdev, torch.from_numpy(sg).cuda(), None if b is None else dev(b),
               acc_dbg=acc_d)
    acc_ref, y_ref, Y_ref = oracle.gemm_a16(X.numpy(), wq, sg, None if b is None else b.numpy())
    _assert_a16_close(X.numpy(), wq, sg, host(acc_d), host(Y), acc_ref, y_ref, Y_ref)


A16_SHAPES = [
    # T, N, K, g
    (16, 256, 64, 4),
    (1, 256, 64, 4),
    (7, 768, 768, 48),
    (129, 1024, 768, 48),  # ragged token tile
    (300, 768, 784, 48),   # K not a multiple of the 64-element slice
    (513, 1000, 256, 3),   # N not a multiple of the tile, N % g != 0
    (64, 72, 48, 2),       # a single, partial K slice
    (200, 520, 96, 8),
]


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("T,N,K,g", A16_SHAPES)
def test_gemm_a16_matches_oracle(zq, bits, T, N, K, g):
    if bits == 4 and K % 32:
        pytest.skip("int4 needs K % 32 == 0")
    _check_a16(zq, T, N, K, g, bits, seed=T + N + K)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("T,N,K", [(16, 256, 64), (300, 1000, 512), (1024, 768, 1024)])
def test_gemm_a16_tiles(zq, bits, bn, T, N, K):
    _check_a16(zq, T, N, K, 8, bits, seed=bn + T, bn=bn)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K,g", [(256, 64, 4), (1000, 4160, 5), (8, 96, 1), (4104, 3072, 24)])
def test_gemm_a16_gemv_path(zq, bits, T, N, K, g):
    """T <= 4 runs on the CUDA-core matrix-vector kernel (automatic and forced)."""
    if bits == 4 and K % 32:
        pytest.skip("int4 needs K % 32 == 0")
    _check_a16(zq, T, N, K, g, bits, seed=T * 7 + N)
    _check_a16(zq, T, N, K, g, bits, seed=T * 7 + N + 1, bias=False, path=3, max_ctas=5)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("pair", [1, 2])
@pytest.mark.parametrize("T,N,K", [(16, 256, 64), (513, 1000, 256), (1024, 768, 1024),
                                   (700, 2304, 448), (1100, 520, 2112)])
def test_gemm_a16_widened_weights(zq, bits, pair, T, N, K):
    """Codes widened once into fp16 rows in the workspace, then the fp16 GEMM
    with TMA-fed weight tiles (automatic from 1024 tokens, forced here), on
    single CTAs and CTA pairs."""
    _check_a16(zq, T, N, K, 8, bits, seed=T + N + pair, path=4, pair=pair)


def test_gemm_a16_small_t_on_tensor_cores(zq):
    """The tensor-core path forced for a few tokens (one partial 128-row tile)."""
    _check_a16(zq, 3, 520, 256, 8, 8, seed=41, path=1)
    _check_a16(zq, 1, 520, 256, 8, 4, seed=42, path=1)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("T,N,K", [(16, 256, 64), (513, 1000, 256), (1024, 768, 1024), (700, 2304, 448)])
def test_gemm_a16_cta_pairs(zq, bits, bn, T, N, K):
    """256-row units shared by a CTA pair (cta_group::2): each CTA widens
    half of the weight tile and keeps its 128 rows of the accumulators."""
    _check_a16(zq, T, N, K, 8, bits, seed=bn + T + 3, bn=bn, pair=2)


def test_gemm_a16_pairs_persistent(zq):
    """Two pairs walk many units (both weight widths, with and without bias)."""
    _check_a16(zq, 1500, 1536, 640, 12, 8, seed=8, bias=False, pair=2, max_ctas=4)
    _check_a16(zq, 1500, 1536, 640, 12, 4, seed=9, pair=2, max_ctas=4)


def test_gemm_a16_persistent_loop_and_no_bias(zq):
    """Three CTAs walk 36 tiles (two TMEM buffers and every pipeline slot
    reused many times); no bias."""
    _check_a16(zq, 600, 1536, 640, 12, 8, seed=5, bias=False, max_ctas=3)
    _check_a16(zq, 600, 1536, 640, 12, 4, seed=6, bias=False, max_ctas=3)


def test_gemm_a16_zero_scales_give_bias(zq):
    T, N, K, g = 40, 256, 128, 4
    X = synth.activations(T, K, seed=31)
    b = synth.bias(N, 32)
    q = np.zeros((N, K), np.int8)
    sg = np.zeros(g, np.float32)
    for bits, fn in ((8, zq.gemm_w8a16), (4, zq.gemm_w4a16)):
        wdev = torch.from_numpy(oracle.pack_int4(q) if bits == 4 else q).cuda()
        Y = fn(dev(X), wdev, torch.from_numpy(sg).cuda(), dev(b))
        assert np.array_equal(host(Y).view(np.uint16),
                              np.broadcast_to(b.numpy(), (T, N)).view(np.uint16))


def test_gemm_a16_zero_tokens_is_a_no_op(zq):
    X = torch.empty((0, 64), dtype=torch.float16, device="cuda")
    q = torch.zeros((256, 64), dtype=torch.int8, device="cuda")
    Y = zq.gemm_w8a16(X, q, torch.ones(4, device="cuda"))
    assert Y.shape == (0, 256)


A16_FULL = [("neox20b", 0, 4096, 8), ("neox20b", 0, 16, 8), ("neox20b", 2, 1, 4), ("gptj6b", 0, 4, 8),
            ("gpt350m", 2, 16384, 4),
            ("gptj6b", 3, 512, 4)]


@pytest.mark.parametrize("layer,gi,T,bits", A16_FULL)
def test_gemm_a16_full_size_sampled_rows(zq, layer, gi, T, bits):
    """Full-size layers with FP16 activations (GPT-NeoX's attention input, the
    W4/8A16 FFN weights); the oracle recomputes sampled token rows."""
    inp = synth.gemm_inputs(layer, gi, T)
    s = inp.spec
    wq, sg = oracle.quantize_weights_groupwise(inp.W.numpy(), s.g, bits)
    wdev = torch.from_numpy(oracle.pack_int4(wq) if bits == 4 else wq).cuda()
    acc_d = torch.empty((T, s.N), dtype=torch.float32, device="cuda")
    fn = zq.gemm_w4a16 if bits == 4 else zq.gemm_w8a16
    Y = fn(dev(inp.X), wdev, torch.from_numpy(sg).cuda(), dev(inp.b), acc_dbg=acc_d)
    rows = _sample_rows(T, n=2)
    Xs = inp.X.numpy()[rows]
    acc_ref, y_ref, Y_ref = oracle.gemm_a16(Xs, wq, sg, inp.b.numpy())
    _assert_a16_close(Xs, wq, sg, host(acc_d)[rows], host(Y)[rows], acc_ref, y_ref, Y_ref)


# ------------------------------------------------------------ errors on the device

def test_bounded_wait_reports_timeout(zq):
    rc, _ = zq.device_status()
    assert rc == zq.ZQ_OK
    zq.debug_wait_timeout()
    rc, detail = zq.device_status()
    assert rc == zq.ZQ_ERR_TIMEOUT and detail > 0
    # the context is still usable and the status word was cleared
    _check_gemm(zq, 16, 256, 64, 4, 8)
    # so are the arrival counters of the in-kernel split-K reduction
    _check_gemm(zq, 8, 1024, 2048, 8, 8, seed=9, path=2, split_k=4)
    assert zq.device_status()[0] == zq.ZQ_OK


def test_misaligned_device_pointer_rejected(zq):
    X = torch.zeros(4 * 64 + 8, dtype=torch.float16, device="cuda")
    Xq = torch.zeros(4 * 64, dtype=torch.int8, device="cuda")
    s = torch.zeros(4, dtype=torch.float32, device="cuda")
    rc = zq.lib().zq_ln_quant(X.data_ptr() + 2, None, None, 4, 64, 1e-5, Xq.data_ptr(),
                              s.data_ptr(), None, None)
    assert rc == zq.ZQ_ERR_ALIGN


def test_cuda_graph_replay_matches_eager(zq):
    """The hot path can be recorded once as a CUDA graph and replayed (the
    paper uses CUDA Graphs for small models); replay gives identical bits."""
    T, K, N, g = 512, 768, 768, 48
    X = synth.activations(T, K, seed=21, n_outliers=6, outlier_scale=20.0).cuda()
    gamma, beta = (t.cuda() for t in synth.ln_params(K, 22))
    W = synth.weights(N, K, 0.02, seed=23).cuda()
    b = synth.bias(N, 24).cuda()
    outs = {}
    for bits in (8, 4):
        Wq, sg = zq.quantize_weights_groupwise(W, g, bits)
        Xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
        st = torch.empty(T, dtype=torch.float32, device="cuda")
        Y = torch.empty((T, N), dtype=torch.float16, device="cuda")
        fn = zq.gemm_w4a8 if bits == 4 else zq.gemm_w8a8

        def step():
            zq.ln_quant(X, gamma, beta, 1e-5, Xq=Xq, s_tok=st)
            fn(Xq, st, Wq, sg, b, Y=Y)

        step()
        torch.cuda.synchronize()
        ref = Y.clone()
        Y.zero_()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        graph.replay()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(Y, ref)
        outs[bits] = ref
    assert zq.device_status()[0] == zq.ZQ_OK


def test_back_to_back_kernels_keep_stream_order(zq):
    """Kernels may be scheduled while the previous one finishes; each waits for
    it before touching memory.  Reusing one set of buffers for several
    LN -> GEMM passes in a row (read-after-write and write-after-read on the
    same buffers) must give exactly the results of separate passes."""
    T, K, N, g = 1024, 768, 2304, 48
    gamma, beta = (t.cuda() for t in synth.ln_params(K, 31))
    W = synth.weights(N, K, 0.02, seed=32).cuda()
    b = synth.bias(N, 33).cuda()
    Wq, sg = zq.quantize_weights_groupwise(W, g, 8)
    Xs = [synth.activations(T, K, seed=40 + i, n_outliers=6, outlier_scale=20.0).cuda()
          for i in range(4)]
    refs = []
    for X in Xs:  # separate passes, synchronised after each
        Xq, st = zq.ln_quant(X, gamma, beta, 1e-5)
        refs.append(zq.gemm_w8a8(Xq, st, Wq, sg, b))
        torch.cuda.synchronize()
    Xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
    st = torch.empty(T, dtype=torch.float32, device="cuda")
    Y = torch.empty((T, N), dtype=torch.float16, device="cuda")
    outs = []
    for X in Xs:  # one buffer set, no synchronisation in between
        zq.ln_quant(X, gamma, beta, 1e-5, Xq=Xq, s_tok=st)
        zq.gemm_w8a8(Xq, st, Wq, sg, b, Y=Y)
        outs.append(Y.clone())
    torch.cuda.synchronize()
    for o, r in zip(outs, refs):
        assert torch.equal(o, r)
