"""Seeded synthetic inputs shaped like the paper's BERT / GPT layers.

This module only draws random tensors and names shapes; it holds none of the
quantization arithmetic.  Both the CUDA path and the CPU oracle are fed from
it (tensors are created on the CPU with a seeded ``torch.Generator`` and then
copied where they are needed), so the two sides always see identical inputs.

Shapes follow "ZeroQuant" (arXiv 2206.01861), Section 5 (BERT-base, GPT-3
350M, GPT-J 6B, GPT-NeoX 20B) and the group counts of Section 3.4
"Group-wise Weight Quantization"; W4/8 puts the FFN weights in INT4 and the
attention weights in INT8 (Sec. 3.4 "Which weights get INT4").  The trained
weights and real activations are not available, so:

* X ~ N(0, 1) fp16 with a seeded set of outlier channels scaled up (standing
  in for the per-token range spread of Fig. 1),
* W ~ N(0, sigma) fp16, bias ~ N(0, 0.01) fp16,
* LayerNorm gamma = 1 + 0.1 N(0,1), beta = 0.1 N(0,1) (fp16).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Gemm:
    """One quantized linear layer: Y[T,N] = X[T,K] W[N,K]^T + b."""

    name: str
    K: int
    N: int
    g: int
    bits: int  # 8 = W8A8, 4 = W4A8
    ln: bool  # input produced by the fused LayerNorm + quant (else quant only)


@dataclass(frozen=True)
class Layer:
    name: str
    hidden: int
    gemms: tuple
    tokens: tuple  # token counts (batch * seq) this layer is run at
    sigma_w: float
    outlier_frac: float | None = None  # fraction of channels ...
    outlier_count: int | None = None  # ... or a fixed count
    outlier_scale: float = 20.0
    seed_base: int = 0
    notes: str = ""

    def n_outliers(self, K: int) -> int:
        if self.outlier_count is not None:
            return min(self.outlier_count, K)
        if self.outlier_frac:
            return max(1, round(self.outlier_frac * K))
        return 0


def _g(name, K, N, g, bits, ln):
    return Gemm(name, K, N, g, bits, ln)


LAYERS = {
    # Single W8A8 linear layer, 16 tokens x 64 hidden, 256 outputs in 4 groups.
    "tiny": Layer("tiny", 64, (_g("linear", 64, 256, 4, 8, False),), (16,), 0.02,
                  seed_base=0, notes="seed 0; no outliers"),
    # BERT-base encoder layer, batch 32 x seq 128, g = 48.
    "bert_base": Layer("bert_base", 768,
                       (_g("qkv", 768, 2304, 48, 8, True), _g("attn_out", 768, 768, 48, 8, False),
                        _g("ffn1", 768, 3072, 48, 8, True), _g("ffn2", 3072, 768, 48, 8, False)),
                       (4096,), 0.02, outlier_count=6, outlier_scale=20.0, seed_base=100),
    # GPT-3-350M-style decoder layer, W4/8A8: FFN INT4 (g=64), attention INT8 (g=48).
    "gpt350m": Layer("gpt350m", 1024,
                     (_g("qkv", 1024, 3072, 48, 8, True), _g("attn_out", 1024, 1024, 48, 8, False),
                      _g("ffn1", 1024, 4096, 64, 4, True), _g("ffn2", 4096, 1024, 64, 4, False)),
                     (16384, 8), 0.02, outlier_count=6, outlier_scale=20.0, seed_base=200),
    # GPT-J-6B layer, W8A8, g = 128.
    "gptj6b": Layer("gptj6b", 4096,
                    (_g("qkv", 4096, 12288, 128, 8, True), _g("attn_out", 4096, 4096, 128, 8, False),
                     _g("ffn1", 4096, 16384, 128, 8, True), _g("ffn2", 16384, 4096, 128, 8, False)),
                    (1, 8, 64, 512, 2048), 0.015, outlier_frac=0.001, outlier_scale=30.0,
                    seed_base=300),
    # GPT-NeoX-20B layer, W4/8A8: FFN INT4, attention INT8, g = 192.
    "neox20b": Layer("neox20b", 6144,
                     (_g("qkv", 6144, 18432, 192, 8, True), _g("attn_out", 6144, 6144, 192, 8, False),
                      _g("ffn1", 6144, 24576, 192, 4, True), _g("ffn2", 24576, 6144, 192, 4, False)),
                     (1, 16, 4096), 0.01, outlier_frac=0.001, outlier_scale=30.0, seed_base=400),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def activations(T: int, K: int, seed: int, n_outliers: int = 0, outlier_scale: float = 20.0,
                std: float = 1.0) -> torch.Tensor:
    """fp16 [T, K] ~ N(0, std) with ``n_outliers`` seeded channels scaled."""
    gen = _gen(seed)
    x = torch.randn(T, K, generator=gen, dtype=torch.float32) * std
    if n_outliers:
        idx = torch.randperm(K, generator=gen)[:n_outliers]
        x[:, idx] *= outlier_scale
    return x.to(torch.float16)


def weights(N: int, K: int, sigma: float, seed: int) -> torch.Tensor:
    gen = _gen(seed)
    return (torch.randn(N, K, generator=gen, dtype=torch.float32) * sigma).to(torch.float16)


def bias(N: int, seed: int, std: float = 0.01) -> torch.Tensor:
    gen = _gen(seed)
    return (torch.randn(N, generator=gen, dtype=torch.float32) * std).to(torch.float16)


def ln_params(K: int, seed: int):
    gen = _gen(seed)
    gamma = (1.0 + 0.1 * torch.randn(K, generator=gen)).to(torch.float16)
    beta = (0.1 * torch.randn(K, generator=gen)).to(torch.float16)
    return gamma, beta


@dataclass
class GemmInputs:
    spec: Gemm
    T: int
    X: torch.Tensor  # fp16 [T, K] (pre-LN hidden state when spec.ln)
    W: torch.Tensor  # fp16 [N, K]
    b: torch.Tensor  # fp16 [N]
    gamma: torch.Tensor | None = None
    beta: torch.Tensor | None = None
    extra: dict = field(default_factory=dict)


def gemm_activations(layer: str, gemm_index: int, T: int) -> torch.Tensor:
    """The seeded fp16 input rows [T, K] of one GEMM of one layer: the X of
    gemm_inputs, without drawing the weights."""
    L = LAYERS[layer]
    s = L.gemms[gemm_index]
    if layer == "tiny":
        return activations(T, s.K, 0)
    base = L.seed_base + 10 * gemm_index
    return activations(T, s.K, base + 1, L.n_outliers(s.K), L.outlier_scale)


def gemm_inputs(layer: str, gemm_index: int, T: int) -> GemmInputs:
    """Seeded inputs of one GEMM of one layer (sub-seed = base + 10*index + tensor)."""
    L = LAYERS[layer]
    s = L.gemms[gemm_index]
    base = L.seed_base + 10 * gemm_index
    if layer == "tiny":  # seed 0 throughout, as the configuration states
        X = activations(T, s.K, 0)
        W = weights(s.N, s.K, L.sigma_w, 1)
        b = bias(s.N, 2)
        return GemmInputs(s, T, X, W, b)
    X = gemm_activations(layer, gemm_index, T)
    W = weights(s.N, s.K, L.sigma_w, base + 2)
    b = bias(s.N, base + 3)
    gamma = beta = None
    if s.ln:
        gamma, beta = ln_params(s.K, base + 4)
    return GemmInputs(s, T, X, W, b, gamma, beta)


def edge_activations(kind: str, T: int, K: int, seed: int = 7) -> torch.Tensor:
    """Degenerate activation rows used by the edge-case tests."""
    x = activations(T, K, seed)
    if kind == "zero_rows":
        x[::3] = 0
    elif kind == "constant_rows":
        x[:] = x[:, :1]
    elif kind == "max_values":
        x[::2, ::5] = 65504.0
        x[1::2, ::7] = -65504.0
    elif kind == "tiny_values":
        x = (x.float() * 2.0 ** -20).to(torch.float16)  # subnormal fp16
    elif kind != "normal":
        raise ValueError(kind)
    return x
