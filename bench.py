"""Benchmark of the fused quantized linear layer (ZeroQuant hot path) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--layer bert_base] [--tokens T]
    python bench.py --impl reference ...      # the CPU oracle on the host cores

One step = one pass of the hot path of a transformer layer over one batch of
synthetic tokens: for each of the layer's four quantized linear layers (QKV,
attention-out, FFN1, FFN2), the fused LayerNorm + token quantization (quant
only where no LayerNorm precedes the GEMM) followed by the W8A8 / W4A8 GEMM
with its fused dequant epilogue.  Weights are quantized once before timing
(offline, as in the paper) and that time is reported separately.

Prints ONE JSON line (rank 0).  `value` is int8 TOPS of the whole step
(2*T*N*K summed over the four GEMMs / step time) with inputs resident in HBM;
`e2e` is the same through the C ABI with the step's fp16 inputs copied from
pinned host memory and its fp16 outputs copied back inside the timed region.
The L2 is flushed before every timed step: a 512 MB write, then a 256 MB
read, so that the timed region starts with a cold L2 holding no dirty lines
of the flush itself (their write-back would otherwise land inside it).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from int4_quantized_transformer_b200 import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0  # nominal dense int8 / bf16 tensor ratio on B200 (4.5 / 2.25 PFLOP/s)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of the dominant GEMM with a cold L2, keyed by
# (layer, gemm name, T); valid only for the GEMM source it was taken with
# (sha256 prefix of csrc/gemm_i8.cu, recorded in profiles/).
NCU_TRAFFIC = {
    # profiles/gemm_i8_dram_traffic.md, bert_base ffn1 row (the fp16 output
    # is still in L2 when the kernel ends, so DRAM writes read 0)
    ("ffn1", 768, 3072, 4096): {"bytes": 5572608 + 6912, "source": "df86abc2f23b"},
}


def _gemm_source_hash():
    import hashlib

    p = os.path.join(ROOT, "int4_quantized_transformer_b200", "csrc", "gemm_i8.cu")
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:12]


def traffic_for(spec, T):
    entry = NCU_TRAFFIC.get((spec.name, spec.K, spec.N, T))
    if entry is None or entry["source"] != _gemm_source_hash():
        return None
    return entry["bytes"]


def layer_workload(layer: str, T: int):
    L = synth.LAYERS[layer]
    return [synth.gemm_inputs(layer, i, T) for i in range(len(L.gemms))]


def gemm_ops(specs, T):
    return sum(2.0 * T * s.N * s.K for s in specs)


def weight_bytes(specs):
    return sum(s.N * s.K * s.bits // 8 for s in specs)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ GPU arm

class LayerStep:
    """Device-resident operands and the kernel sequence of one step."""

    def __init__(self, zq, inputs, device):
        self.zq = zq
        self.items = []
        for gi in inputs:
            s = gi.spec
            W = gi.W.to(device)
            Wq, sg = zq.quantize_weights_groupwise(W, s.g, s.bits)
            it = {
                "W16": W,  # the fp16 weights, for the fp16 cuBLAS comparison only
                "spec": s,
                "X": gi.X.to(device),
                "gamma": None if gi.gamma is None else gi.gamma.to(device),
                "beta": None if gi.beta is None else gi.beta.to(device),
                "Wq": Wq, "s_grp": sg, "b": gi.b.to(device),
                "Xq": torch.empty((gi.T, s.K), dtype=torch.int8, device=device),
                "s_tok": torch.empty(gi.T, dtype=torch.float32, device=device),
                "Y": torch.empty((gi.T, s.N), dtype=torch.float16, device=device),
                "T": gi.T,
            }
            self.items.append(it)
        self.launches_per_step = 2 * len(self.items)

    def run_ln(self, it, stream=None):
        self.zq.ln_quant(it["X"], it["gamma"], it["beta"], 1e-5, Xq=it["Xq"], s_tok=it["s_tok"],
                         stream=stream)

    def run_gemm(self, it, stream=None):
        fn = self.zq.gemm_w4a8 if it["spec"].bits == 4 else self.zq.gemm_w8a8
        fn(it["Xq"], it["s_tok"], it["Wq"], it["s_grp"], it["b"], Y=it["Y"], stream=stream)

    def run(self, stream=None):
        for it in self.items:
            self.run_ln(it, stream)
            self.run_gemm(it, stream)


def make_flush_buffers(device):
    """A 512 MB buffer that the flush writes and a 256 MB one that it reads
    (both larger than the 126 MB L2), plus the read's scalar result."""
    w = torch.zeros(512 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    r = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    return w, r, torch.empty((), dtype=torch.float32, device=device)


def flush_l2(buf):
    """Evict the L2: write a buffer larger than it, then read another one so
    that the lines left behind are clean."""
    w, r, out = buf
    w.add_(1)
    torch.sum(r, dim=0, out=out)


def barrier(dist_on, cuda=True):
    if dist_on:
        torch.distributed.barrier()
    if cuda:
        torch.cuda.synchronize()


def max_over_ranks(x: float, dist_on: bool, device="cuda") -> float:
    """The slowest rank's time: every rank contributes x, all receive the max."""
    if not dist_on:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tops(ops_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank runs the same work (replicas), timed
    as the max over ranks."""
    return world * ops_per_rank / (ms_max * 1e-3) / 1e12


def time_steps(fn, steps, flush_buf, stream):
    """Per-step device time (ms) with CUDA events on `stream`, L2 flushed
    before each step (outside the events)."""
    total = 0.0
    per = []
    for _ in range(steps):
        flush_l2(flush_buf)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        e1.synchronize()
        ms = e0.elapsed_time(e1)
        per.append(ms)
        total += ms
    return total, per


def gpu_arm(args, dist_on, rank, world):
    from int4_quantized_transformer_b200 import zq

    device = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    layer = args.layer
    T = args.tokens or synth.LAYERS[layer].tokens[0]
    inputs = layer_workload(layer, T)
    specs = [gi.spec for gi in inputs]
    ops = gemm_ops(specs, T)
    wbytes = weight_bytes(specs)
    stream = torch.cuda.current_stream()

    # offline weight quantization (timed once, reported separately)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    step = LayerStep(zq, inputs, device)
    torch.cuda.synchronize()
    wquant_s = time.perf_counter() - t0
    flush_buf = make_flush_buffers(device)

    for _ in range(args.warmup):
        step.run()
    rc, detail = zq.device_status()
    if rc != zq.ZQ_OK:
        raise RuntimeError(f"device status {rc} ({detail}) after warm-up")

    # The step's kernel sequence is recorded once as a CUDA graph and replayed
    # (the paper's remedy for launch overhead on small models, Appendix D).
    graph = None
    graph_error = None
    if not args.eager:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step.run()
            for _ in range(args.warmup):
                graph.replay()
        except Exception as exc:  # capture refused: report it and time eager launches
            graph, graph_error = None, f"{type(exc).__name__}: {exc}"
            torch.cuda.synchronize()
    run_step = graph.replay if graph is not None else step.run

    # ---- timed region: K steps, inputs resident in HBM
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(dist_on)
        total_ms, per_step = time_steps(run_step, args.steps, flush_buf, stream)
        barrier(dist_on)
    total_ms = max_over_ranks(total_ms, dist_on)
    ms_per_step = total_ms / args.steps
    eager_ms, _ = time_steps(step.run, max(3, args.steps // 2), flush_buf, stream)
    eager_ms /= max(3, args.steps // 2)

    # ---- per-kernel device times for the roofline: a CUDA graph of R x
    # [L2 flush, kernel] minus a graph of R x [L2 flush], divided by R, both
    # timed with CUDA events on the launching stream.  (Events between the
    # launches of an eager step would also count each kernel's launch
    # latency, which the step's graph with programmatic dependent launch
    # hides.)
    reps = max(3, min(args.steps, 20))

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                flush_l2(flush_buf)
                if fn is not None:
                    fn()
        return g

    def time_graph(g):
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1)

    kern = {}
    try:
        base_ms = time_graph(graph_of(None))
        for it in step.items:
            s = it["spec"]
            for kind in ("ln", "gemm"):
                fn = (lambda it=it: step.run_ln(it)) if kind == "ln" else (lambda it=it: step.run_gemm(it))
                kern[(s.name, kind)] = max(time_graph(graph_of(fn)) - base_ms, 1e-6) / reps
        kern_method = f"CUDA graph of {reps} x [L2 flush, kernel] minus {reps} x [L2 flush]"
    except Exception as exc:  # graphs refused: eager launches after a flush
        torch.cuda.synchronize()
        for it in step.items:
            s = it["spec"]
            for kind in ("ln", "gemm"):
                fn = (lambda it=it: step.run_ln(it)) if kind == "ln" else (lambda it=it: step.run_gemm(it))
                tot, _ = time_steps(fn, reps, flush_buf, stream)
                kern[(s.name, kind)] = tot / reps
        kern_method = f"eager launches after an L2 flush ({type(exc).__name__})"
    gemm_ms = sum(v for (n, k), v in kern.items() if k == "gemm")
    ln_ms = sum(v for (n, k), v in kern.items() if k == "ln")
    peak_tops = INT8_PER_BF16 * float(peaks["bf16_tflops"])
    # the dominant kernel: the GEMM launch with the largest device time
    dom = max((it for it in step.items), key=lambda it: kern[(it["spec"].name, "gemm")])
    dom_spec = dom["spec"]
    dom_ms = kern[(dom_spec.name, "gemm")]
    dom_ops = 2.0 * T * dom_spec.N * dom_spec.K
    achieved_tops = dom_ops / (dom_ms * 1e-3) / 1e12
    all_gemm_tops = ops / (gemm_ms * 1e-3) / 1e12

    # ---- end to end through the C ABI: pinned host inputs in, outputs out
    h_in = [it["X"].cpu().pin_memory() for it in step.items]
    h_out = [torch.empty(it["Y"].shape, dtype=torch.float16).pin_memory() for it in step.items]
    h2d = sum(x.numel() * 2 for x in h_in)
    d2h = sum(y.numel() * 2 for y in h_out)

    def e2e_step():
        for it, hx, hy in zip(step.items, h_in, h_out):
            it["X"].copy_(hx, non_blocking=True)
        run_step()
        for it, hx, hy in zip(step.items, h_in, h_out):
            hy.copy_(it["Y"], non_blocking=True)

    for _ in range(2):
        e2e_step()
    barrier(dist_on)
    e2e_ms, _ = time_steps(e2e_step, args.steps, flush_buf, stream)
    barrier(dist_on)
    e2e_ms = max_over_ranks(e2e_ms, dist_on) / args.steps
    rc, detail = zq.device_status()
    if rc != zq.ZQ_OK:
        raise RuntimeError(f"device status {rc} ({detail}) after timing")

    # ---- library references, measured last so that nothing above runs after
    # cuBLAS work or its graph captures: the same shapes in fp16 through cuBLAS
    # (torch.addmm: X W^T + b), per GEMM and as a graph of the four GEMMs, and
    # cuBLAS's own INT8 GEMM (torch._int_mm, int32 out, no scales) on the
    # dominant shape, timed like the kernels above
    ref16, ref16_step_ms, ref_i8, ref16_error = {}, None, None, None
    try:
        fns16 = [lambda it=it: torch.addmm(it["b"], it["X"], it["W16"].t()) for it in step.items]
        for fn16 in fns16:
            fn16()  # cuBLAS sets up its handle and workspace outside any capture
        torch.cuda.synchronize()
        for it, fn16 in zip(step.items, fns16):
            ref16[it["spec"].name] = max(time_graph(graph_of(fn16)) - base_ms, 1e-6) / reps
        # the fp16 layer: LayerNorm before the GEMMs that have one, then the GEMM
        def fp16_layer():
            for it in step.items:
                x = it["X"]
                if it["gamma"] is not None:
                    x = torch.nn.functional.layer_norm(x, (x.shape[1],), it["gamma"], it["beta"], 1e-5)
                torch.addmm(it["b"], x, it["W16"].t())

        fp16_layer()
        torch.cuda.synchronize()
        ref16_step_ms = max(time_graph(graph_of(fp16_layer)) - base_ms, 1e-6) / reps
        if T > 16:
            x8 = torch.randint(-127, 128, (T, dom_spec.K), dtype=torch.int8, device=device)
            w8 = torch.randint(-127, 128, (dom_spec.N, dom_spec.K), dtype=torch.int8, device=device)
            torch._int_mm(x8, w8.t())
            torch.cuda.synchronize()
            ref_i8 = max(time_graph(graph_of(lambda: torch._int_mm(x8, w8.t()))) - base_ms,
                         1e-6) / reps
    except Exception as exc:
        torch.cuda.synchronize()
        ref16_error = f"{type(exc).__name__}: {exc}"

    res = {
        "metric": "int8 TOPS of the fused quantized linear layers (LN+quant and W8A8/W4A8 GEMM "
                  "with dequant epilogue) per layer step",
        "value": round(whole_job_tops(ops, world, ms_per_step), 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "ms_per_step_median": round(statistics.median(per_step), 5),
        "ms_per_step_best": round(min(per_step), 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic (seeded N(0,1) activations with outlier channels, N(0,sigma) weights)",
        "config": {
            "workload": f"{layer} layer, T={T} tokens, 4 quantized linears "
                        + ", ".join(f"{s.name} {s.K}->{s.N} W{s.bits}A8 g={s.g}" for s in specs),
            "tokens": T,
            "l2": "flushed before every timed step (512 MB write, then 256 MB read)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "launch": "cuda graph replay of the step" if graph is not None else "eager launches",
        },
        "eager_ms_per_step": round(eager_ms, 5),
        "graph_error": graph_error,
        "weight_gbs": round(world * wbytes / (ms_per_step * 1e-3) / 1e9, 1),
        "roofline": {
            "bound": "tensor",
            "kernel": f"gemm_i8_kernel (tcgen05 kind::i8), {dom_spec.name} {dom_spec.K}->{dom_spec.N} "
                      f"T={T}",
            "achieved": round(achieved_tops, 1),
            "peak": round(peak_tops, 1),
            "unit": "TOPS",
            "frac": round(achieved_tops / peak_tops, 4),
            "peak_source": f"{peak_src}: 2 x bf16 dense {'burst' if peak_src == 'measured' else 'fallback'} "
                           f"({peaks['bf16_tflops']} TFLOP/s), nominal int8/bf16 ratio 2",
            "traffic": traffic_for(dom_spec, T),
            "all_gemms_tops": round(all_gemm_tops, 1),
            "kernel_time_method": kern_method,
        },
        "kernels_us": {f"{n}.{k}": round(v * 1e3, 2) for (n, k), v in kern.items()},
        "fp16_cublas": {"error": ref16_error} if not ref16 else {
            "what": "torch.addmm(bias, X, W^T) in fp16 (cuBLAS) on each GEMM shape of the step, "
                    "timed as the kernels above; step = a graph of the fp16 layer (torch layer_norm "
                    "before the GEMMs that have a LayerNorm, then the four GEMMs), L2 flushed before it",
            "gemm_us": {n: round(v * 1e3, 2) for n, v in ref16.items()},
            "step_us": None if ref16_step_ms is None else round(ref16_step_ms * 1e3, 2),
            "gemm_speedup": round(sum(ref16.values()) / gemm_ms, 3),
            "step_speedup": None if ref16_step_ms is None else round(ref16_step_ms / ms_per_step, 3),
            "dominant_fp16_tflops": round(dom_ops / (ref16[dom_spec.name] * 1e-3) / 1e12, 1),
            "dominant_cublas_int8_us": None if ref_i8 is None else round(ref_i8 * 1e3, 2),
        },
        "ln_quant_gbs": round(sum(3 * it["T"] * it["spec"].K for it in step.items) / (ln_ms * 1e-3) / 1e9, 1),
        "offline_wquant_ms": round(wquant_s * 1e3, 2),
        "e2e": {"value": round(whole_job_tops(ops, world, e2e_ms), 2), "unit": "TOPS",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(layer, T, args.cpu_tokens)
    return res


# ------------------------------------------------------------------ CPU oracle arm

def oracle_step(inputs, rows):
    """The oracle's hot path on a token subset: ln_quant + exact GEMM + dequant."""
    import oracle

    for gi in inputs:
        s = gi.spec
        X = gi.X.numpy()[:rows]
        xq, st = oracle.ln_quant(X, None if gi.gamma is None else gi.gamma.numpy(),
                                 None if gi.beta is None else gi.beta.numpy(), 1e-5)
        wq, sg = gi.extra["wq"], gi.extra["sg"]
        oracle.linear_q(xq, st, wq, sg, gi.b.numpy())


def prepare_oracle(layer, T):
    import oracle

    inputs = layer_workload(layer, T)
    for gi in inputs:
        wq, sg = oracle.quantize_weights_groupwise(gi.W.numpy(), gi.spec.g, gi.spec.bits)
        gi.extra["wq"], gi.extra["sg"] = wq, sg
    return inputs


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(layer, T, rows):
    rows = min(rows, T)
    inputs = prepare_oracle(layer, T)
    t0 = time.perf_counter()
    oracle_step(inputs, rows)
    dt = time.perf_counter() - t0
    ops = gemm_ops([gi.spec for gi in inputs], rows)
    return {"value": round(ops / dt / 1e12, 6), "unit": "TOPS", "cores": 1, "kind": "oracle",
            "host_cpu_model": host_cpu_model(),
            "sample": f"{rows} of {T} tokens of every GEMM of the step (LN+quant, exact int GEMM, "
                      f"dequant), single-threaded plain C, {dt:.1f} s",
            "host_cpus": os.cpu_count()}


def reference_arm(args, rank, world):
    layer = args.layer
    T = args.tokens or synth.LAYERS[layer].tokens[0]
    rows = min(args.ref_tokens, T)
    inputs = prepare_oracle(layer, T)
    specs = [gi.spec for gi in inputs]
    for _ in range(args.warmup):
        oracle_step(inputs, rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(inputs, rows)
    dt = (time.perf_counter() - t0) / args.steps
    ops = gemm_ops(specs, rows)
    val = round(ops / dt / 1e12, 6)
    sample = (f"{rows} of {T} tokens of every GEMM of the {layer} step per timed step "
              f"(oracle: LN+quant, exact int GEMM, dequant), single-threaded plain C")
    return {
        "impl": "reference",
        "metric": "int8 TOPS of the fused quantized linear layers (LN+quant and W8A8/W4A8 GEMM "
                  "with dequant epilogue) per layer step",
        "value": val, "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": f"{layer} layer, T={T} tokens (oracle timed on a {rows}-token sample)",
                   "tokens": T},
        "cpu_baseline": {"value": val, "unit": "TOPS", "cores": 1, "kind": "oracle", "sample": sample,
                         "host_cpu_model": host_cpu_model(), "host_cpus": os.cpu_count()},
        "e2e": {"value": val, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="zq", choices=["zq", "reference"])
    ap.add_argument("--layer", default="bert_base", choices=sorted(synth.LAYERS))
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--cpu-tokens", type=int, default=2048)
    ap.add_argument("--ref-tokens", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch kernels one by one (no CUDA graph)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args, rank, world)), flush=True)
        return

    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        res = gpu_arm(args, dist_on, rank, world)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if dist_on:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
