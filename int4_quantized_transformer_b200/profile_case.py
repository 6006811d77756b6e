"""Run one kernel of the hot path on one layer shape, for ncu captures.

    python -m int4_quantized_transformer_b200.profile_case --kind gemm --layer bert_base --gemm 0
    python -m int4_quantized_transformer_b200.profile_case --kind ln --layer bert_base --gemm 0
    python -m int4_quantized_transformer_b200.profile_case --kind act --act gelu --layer bert_base --gemm 3
    python -m int4_quantized_transformer_b200.profile_case --kind a16 --bits 8 --layer neox20b --gemm 0

Quantizes the weights, runs `--warmup` untimed launches and then `--reps`
launches of the chosen kernel (the fused LN+quant of that GEMM's input, the
GEMM itself, or with --kind a16 the FP16-activation GEMM of that shape)
recorded in one CUDA graph, printing the mean device time per launch
measured with CUDA events around the graph replay.  With --flush every
launch follows an L2 flush, and the time of a graph of the flushes alone is
subtracted.  Options force a GEMM variant (see zq_set_option).

--kind cublas times the library references on the same shape: cuBLAS's
INT8 GEMM through torch._int_mm (int32 output, no scales) and torch.matmul
in fp16.  They are context for the roofline numbers, not part of the path.
"""
from __future__ import annotations

import argparse
import json

import torch

from int4_quantized_transformer_b200 import synth, zq


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kind", choices=["gemm", "a16", "ln", "act", "static", "wquant", "cublas"],
                    default="gemm")
    ap.add_argument("--bits", type=int, default=0, choices=[0, 4, 8],
                    help="weight bits for --kind a16 (default: the layer GEMM's)")
    ap.add_argument("--act", choices=["gelu", "none"], default="gelu",
                    help="--kind act: GeLU + quant, or bias-add + quant (with a bias)")
    ap.add_argument("--layer", default="bert_base", choices=sorted(synth.LAYERS))
    ap.add_argument("--gemm", type=int, default=0, help="index of the layer's GEMM (0..3)")
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--path", type=int, default=0)
    ap.add_argument("--bn", type=int, default=0)
    ap.add_argument("--split-k", type=int, default=0)
    ap.add_argument("--pair", type=int, default=0, help="1 = single-CTA tiles, 2 = CTA pairs")
    ap.add_argument("--eager", action="store_true",
                    help="eager launches instead of a graph (for ncu captures: the printed time then "
                         "includes host launch latency)")
    ap.add_argument("--flush", action="store_true",
                    help="flush the L2 before every launch (512 MB write + 256 MB read, as in bench.py)")
    a = ap.parse_args()

    T = a.tokens or synth.LAYERS[a.layer].tokens[0]
    gi = synth.gemm_inputs(a.layer, a.gemm, T)
    s = gi.spec
    W = gi.W.cuda()
    Wq, sg = zq.quantize_weights_groupwise(W, s.g, s.bits)
    X = gi.X.cuda()
    gamma = None if gi.gamma is None else gi.gamma.cuda()
    beta = None if gi.beta is None else gi.beta.cuda()
    Xq, st = zq.ln_quant(X, gamma, beta)
    b = gi.b.cuda()
    # the bias of the bias-add + quant form: the GEMM's input width
    act_bias = None if a.act == "gelu" else gi.X[0].cuda() * 0.25
    Y = torch.empty((T, s.N), dtype=torch.float16, device="cuda")
    gemm = zq.gemm_w4a8 if s.bits == 4 else zq.gemm_w8a8
    bits = a.bits or s.bits
    if a.kind == "a16":
        Wq16, sg16 = zq.quantize_weights_groupwise(W, s.g, bits)
        gemm16 = zq.gemm_w4a16 if bits == 4 else zq.gemm_w8a16
    if a.kind == "cublas":
        x8 = torch.randint(-127, 128, (T, s.K), dtype=torch.int8, device="cuda")
        w8 = torch.randint(-127, 128, (s.N, s.K), dtype=torch.int8, device="cuda")
        w16 = W

    # L2 flush: write 512 MB, then read 256 MB, so the L2 is cold and clean
    flush = None
    if a.flush:
        flush = (torch.zeros(128 * 1024 * 1024, dtype=torch.float32, device="cuda"),
                 torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda"),
                 torch.empty((), dtype=torch.float32, device="cuda"))

    def do_flush():
        flush[0].add_(1)
        torch.sum(flush[1], dim=0, out=flush[2])

    def run():
        if a.kind == "gemm":
            gemm(Xq, st, Wq, sg, b, Y=Y)
        elif a.kind == "ln":
            zq.ln_quant(X, gamma, beta, Xq=Xq, s_tok=st)
        elif a.kind == "static":
            zq.static_quant(X, 8.0, Xq=Xq, s_tok=st)
        elif a.kind == "act":
            zq.bias_act_quant(X, act_bias, zq.ACT_GELU if a.act == "gelu" else zq.ACT_NONE,
                              Xq=Xq, s_tok=st)
        elif a.kind == "a16":
            gemm16(X, Wq16, sg16, b, Y=Y)
        else:
            zq.quantize_weights_groupwise(W, s.g, s.bits, Wq=Wq, s_grp=sg)

    def timed(body):
        """Mean device time of one body() over --reps, in microseconds."""
        graph = None
        if not a.eager:
            # back-to-back launches recorded in a CUDA graph: device time
            # rather than host launch overhead
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(a.reps):
                    body()
            graph.replay()
            torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if graph is not None:
            graph.replay()
        else:
            for _ in range(a.reps):
                body()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) * 1e3 / a.reps

    def measure(op):
        for _ in range(a.warmup):
            op()
        torch.cuda.synchronize()
        if flush is None:
            return timed(op)
        both = timed(lambda: (do_flush(), op()))
        return max(both - timed(do_flush), 0.0)

    extra = {}
    with zq.options(path=a.path, bn=a.bn, split_k=a.split_k, pair=a.pair):
        if a.kind == "cublas":
            # torch._int_mm takes more than 16 rows only
            us = measure(lambda: torch._int_mm(x8, w8.t())) if T > 16 else float("nan")
            extra["fp16_us"] = round(measure(lambda: torch.matmul(X, w16.t())), 2)
        else:
            us = measure(run)
    rc, detail = zq.device_status()
    if rc != zq.ZQ_OK:
        raise SystemExit(f"device status {rc} ({detail})")
    ops = 2.0 * T * s.N * s.K
    res = {"kind": a.kind, "layer": a.layer, "gemm": s.name, "T": T, "N": s.N, "K": s.K,
           "bits": bits if a.kind == "a16" else s.bits, "flush": flush is not None,
           "us": round(us, 2), **extra}
    if a.kind in ("ln", "act", "static"):  # fp16 in, int8 + one fp32 scale per row out
        res["gbs"] = round((3 * T * s.K + 4 * T) / us / 1e3, 1)
    elif a.kind == "a16":  # fp16 tensor work; the weight stream bounds small T
        res["tflops"] = round(ops / us / 1e6, 1)
        res["weight_gbs"] = round(s.N * s.K * bits / 8 / us / 1e3, 1)
    else:
        res["tops"] = round(ops / us / 1e6, 1)
        if "fp16_us" in res:
            res["fp16_tflops"] = round(ops / res["fp16_us"] / 1e6, 1)
    print(json.dumps(res))


if __name__ == "__main__":
    main()
