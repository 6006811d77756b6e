"""Run one kernel of the hot path on one layer shape, for ncu captures.

    python -m int4_quantized_transformer_b200.profile_case --kind gemm --layer bert_base --gemm 0
    python -m int4_quantized_transformer_b200.profile_case --kind ln --layer bert_base --gemm 0
    python -m int4_quantized_transformer_b200.profile_case --kind act --act gelu --layer bert_base --gemm 3

Quantizes the weights, runs `--warmup` untimed launches and then `--reps`
launches of the chosen kernel (the fused LN+quant of that GEMM's input, or
the GEMM itself) recorded in one CUDA graph, printing the mean device time
per launch measured with CUDA events around the graph replay (with --flush,
the L2 flush before each launch is included in that time).  Options force a
GEMM variant (see zq_set_option).
"""
from __future__ import annotations

import argparse
import json

import torch

from int4_quantized_transformer_b200 import synth, zq


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kind", choices=["gemm", "ln", "act", "static", "wquant"], default="gemm")
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
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of a graph")
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

    # L2 flush: write 512 MB, then read 256 MB, so the L2 is cold and clean
    flush = None
    if a.flush:
        flush = (torch.zeros(128 * 1024 * 1024, dtype=torch.float32, device="cuda"),
                 torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda"),
                 torch.empty((), dtype=torch.float32, device="cuda"))

    def run():
        if flush is not None:
            flush[0].add_(1)
            torch.sum(flush[1], dim=0, out=flush[2])
        if a.kind == "gemm":
            gemm(Xq, st, Wq, sg, b, Y=Y)
        elif a.kind == "ln":
            zq.ln_quant(X, gamma, beta, Xq=Xq, s_tok=st)
        elif a.kind == "static":
            zq.static_quant(X, 8.0, Xq=Xq, s_tok=st)
        elif a.kind == "act":
            zq.bias_act_quant(X, act_bias, zq.ACT_GELU if a.act == "gelu" else zq.ACT_NONE,
                              Xq=Xq, s_tok=st)
        else:
            zq.quantize_weights_groupwise(W, s.g, s.bits, Wq=Wq, s_grp=sg)

    with zq.options(path=a.path, bn=a.bn, split_k=a.split_k, pair=a.pair):
        for _ in range(a.warmup):
            run()
        torch.cuda.synchronize()
        # Back-to-back launches recorded in a CUDA graph, so the timing is
        # device time rather than host launch overhead.
        graph = None
        if not a.eager:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(a.reps):
                    run()
            graph.replay()
            torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if graph is not None:
            graph.replay()
        else:
            for _ in range(a.reps):
                run()
        e1.record()
        e1.synchronize()
    rc, detail = zq.device_status()
    if rc != zq.ZQ_OK:
        raise SystemExit(f"device status {rc} ({detail})")
    us = e0.elapsed_time(e1) * 1e3 / a.reps
    ops = 2.0 * T * s.N * s.K
    res = {"kind": a.kind, "layer": a.layer, "gemm": s.name, "T": T, "N": s.N, "K": s.K,
           "bits": s.bits, "us": round(us, 2)}
    if a.kind in ("ln", "act", "static"):  # fp16 in, int8 + one fp32 scale per row out
        res["gbs"] = round((3 * T * s.K + 4 * T) / us / 1e3, 1)
    else:
        res["tops"] = round(ops / us / 1e6, 1)
    print(json.dumps(res))


if __name__ == "__main__":
    main()
