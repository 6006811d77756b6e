"""Benchmark of the fused quantized linear layer (ZeroQuant hot path) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--layer neox20b] [--tokens 4096]
    python bench.py --impl reference ...      # the CPU oracle on the host cores

One step = one pass of the hot path of a transformer layer over one batch of
synthetic tokens: for each of the layer's four quantized linear layers (QKV,
attention-out, FFN1, FFN2), the fused LayerNorm + token quantization (quant
only where no LayerNorm precedes the GEMM) followed by the W8A8 / W4A8 GEMM
with its fused dequant epilogue.  Weights are quantized once before timing
(offline, as in the paper) and that time is reported separately.

The headline workload is the GPT-NeoX-20B layer with INT4 FFN weights and
INT8 attention weights (g = 192) at 4096 tokens: the largest layer
configuration, tensor-bound.  The same JSON line carries the weight-streaming
(decode) steps of GPT-NeoX-20B at 1 and 16 tokens and GPT-J-6B at 8 and 64
tokens, each with its weight GB/s and an HBM roofline, and the BERT-base step.

Prints ONE JSON line (rank 0).  `value` is int8 TOPS of the headline step
(2*T*N*K summed over the four GEMMs / step time) with inputs resident in HBM;
`e2e` is the same through the C ABI with the step's fp16 inputs copied from
pinned host memory and its fp16 outputs copied back inside the timed region.
The L2 is flushed before every timed step: a 512 MB write, then a 256 MB
read, so that the timed region starts with a cold L2 holding no dirty lines
of the flush itself (their write-back would otherwise land inside it).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from int4_quantized_transformer_b200 import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0  # nominal dense int8 / bf16 tensor ratio on B200 (4.5 / 2.25 PFLOP/s)

HEADLINE = ("neox20b", 4096)
DECODE_CASES = (("neox20b", 1), ("neox20b", 16), ("gptj6b", 8), ("gptj6b", 64))
EXTRA_PREFILL = (("bert_base", 4096),)

METRIC = ("int8 TOPS of the fused quantized linear layers (LN+quant and W8A8/W4A8 GEMM with "
          "dequant epilogue) per layer step")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes per GEMM call (dram__bytes_read.sum + dram__bytes_write.sum,
# summed over the call's kernels) from one ncu capture with a cold L2, keyed
# by (layer, gemm, T); valid only for the GEMM source it was taken with
# (sha256 prefix of the .cu file named in "file").
NCU_TRAFFIC: dict = {
    # zq_gemm_w4a8, GPT-NeoX FFN2 24576->6144 at T=4096: widen_w4_kernel
    # (76935936 read + 93059072 written), gemm_i8_kernel (746100736 +
    # 44510464), tail_finalize_kernel (18382848 + 0)
    ("neox20b", "ffn2", 4096): {"file": "gemm_i8.cu", "source": "a0ad5c1ac28c",
                                "bytes": 978989056},
}


def _source_hash(name: str) -> str:
    import hashlib

    p = os.path.join(ROOT, "int4_quantized_transformer_b200", "csrc", name)
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:12]


def traffic_for(layer, spec, T):
    entry = NCU_TRAFFIC.get((layer, spec.name, T))
    if entry is None or entry["source"] != _source_hash(entry["file"]):
        return None
    return entry["bytes"]


def gemm_ops(specs, T):
    return sum(2.0 * T * s.N * s.K for s in specs)


def weight_bytes(specs):
    return sum(s.N * s.K * s.bits // 8 for s in specs)


def gemm_bytes(spec, T):
    """Algorithmic bytes of one quantized GEMM: weights (packed for INT4),
    int8 activations, fp16 output, fp32 scales, fp16 bias."""
    return (spec.N * spec.K * spec.bits // 8 + T * spec.K + 2 * T * spec.N
            + 4 * (T + spec.g) + 2 * spec.N)


def ln_bytes(spec, T):
    """Algorithmic bytes of one LN+quant (or quant-only) launch: fp16 rows in,
    int8 rows and one fp32 scale per row out, gamma/beta once."""
    return 3 * T * spec.K + 4 * T + (4 * spec.K if spec.ln else 0)


def workload_name(layer, T, specs):
    return (f"{layer} layer, T={T} tokens, 4 quantized linears "
            + ", ".join(f"{s.name} {s.K}->{s.N} W{s.bits}A8 g={s.g}" for s in specs))


def default_tokens(args):
    """--tokens, else the layer's largest (prefill) token count."""
    return args.tokens or max(synth.LAYERS[args.layer].tokens)


def bench_config(layer, T, world):
    specs = synth.LAYERS[layer].gemms
    cfg = {
        "workload": workload_name(layer, T, specs),
        "layer": layer,
        "tokens": T,
        "l2": "flushed before every timed step (512 MB write, then 256 MB read)",
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
    }
    if any(s.bits == 4 for s in specs) and T >= LayerStep.WIDEN_AHEAD_MIN_TOKENS:
        cfg["int4_widening"] = ("zq_widen_int4_weights on a second stream forked at the start of "
                                "the step (concurrent with the attention GEMMs), then zq_gemm_w8a8 "
                                "on the widened codes")
    return cfg


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

class LayerWeights:
    """One layer's weights on the device: fp16 (for the cuBLAS reference
    only), quantized codes and group scales, bias and LayerNorm parameters.
    The synthetic weights depend on the layer and GEMM, not on T, so every
    token count of a layer shares them."""

    def __init__(self, zq, layer, device, keep_fp16=True):
        self.layer = layer
        self.items = []
        # device time of the weight quantization alone (the synthetic fp16
        # weights are drawn on the host and copied in outside the events)
        self.wquant_ms = 0.0
        z = torch.zeros((8, 64), dtype=torch.float16, device=device)
        for bits in (8, 4):  # the first launch of each kernel loads it: keep that out of the events
            zq.quantize_weights_groupwise(z, 1, bits)
        for i, s in enumerate(synth.LAYERS[layer].gemms):
            gi = synth.gemm_inputs(layer, i, 1)
            W = gi.W.to(device)
            # outputs allocated before the events: only the kernel is timed
            Wq = torch.empty((s.N, s.K) if s.bits == 8 else (s.N, s.K // 2),
                             dtype=torch.int8 if s.bits == 8 else torch.uint8, device=device)
            sg = torch.empty(s.g, dtype=torch.float32, device=device)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            zq.quantize_weights_groupwise(W, s.g, s.bits, Wq=Wq, s_grp=sg)
            e1.record()
            e1.synchronize()
            self.wquant_ms += e0.elapsed_time(e1)
            self.items.append({
                "spec": s, "W16": W if keep_fp16 else None, "Wq": Wq, "s_grp": sg,
                "b": gi.b.to(device),
                "gamma": None if gi.gamma is None else gi.gamma.to(device),
                "beta": None if gi.beta is None else gi.beta.to(device),
            })
            del W


class LayerStep:
    """Device-resident operands of one layer at T tokens and the kernel
    sequence of one step.

    From 512 tokens (where the INT4 GEMM widens its codes before the INT8
    GEMM) the step widens the INT4 weights itself, with zq_widen_int4_weights
    on a second stream forked at the start of the step, so that this
    HBM-bound pass runs while the tensor-bound attention GEMMs do; the FFN
    GEMMs then run as zq_gemm_w8a8 on the widened codes (the same results as
    zq_gemm_w4a8, which tests check).  The per-GEMM timings still time the
    single zq_gemm_w4a8 call."""

    WIDEN_AHEAD_MIN_TOKENS = 512

    def __init__(self, zq, weights: LayerWeights, T, device, inputs=None):
        self.zq = zq
        self.layer = weights.layer
        self.T = T
        self.items = []
        for i, w in enumerate(weights.items):
            s = w["spec"]
            X = inputs[i].X if inputs is not None else synth.gemm_activations(self.layer, i, T)
            self.items.append(dict(w, X=X.to(device),
                                   Xq=torch.empty((T, s.K), dtype=torch.int8, device=device),
                                   s_tok=torch.empty(T, dtype=torch.float32, device=device),
                                   Y=torch.empty((T, s.N), dtype=torch.float16, device=device)))
        self.specs = [it["spec"] for it in self.items]
        self.widen_ahead = T >= self.WIDEN_AHEAD_MIN_TOKENS and any(s.bits == 4 for s in self.specs)
        if self.widen_ahead:
            self.side = torch.cuda.Stream(device=device)
            for it in self.items:
                if it["spec"].bits == 4:
                    it["W8"] = torch.empty((it["spec"].N, it["spec"].K), dtype=torch.int8,
                                           device=device)

    def run_ln(self, it, stream=None):
        self.zq.ln_quant(it["X"], it["gamma"], it["beta"], 1e-5, Xq=it["Xq"], s_tok=it["s_tok"],
                         stream=stream)

    def run_gemm(self, it, stream=None):
        fn = self.zq.gemm_w4a8 if it["spec"].bits == 4 else self.zq.gemm_w8a8
        fn(it["Xq"], it["s_tok"], it["Wq"], it["s_grp"], it["b"], Y=it["Y"], stream=stream)

    def run(self, stream=None):
        if not self.widen_ahead:
            for it in self.items:
                self.run_ln(it, stream)
                self.run_gemm(it, stream)
            return
        main = torch.cuda.current_stream() if stream is None else stream
        fork, join = torch.cuda.Event(), torch.cuda.Event()
        fork.record(main)
        self.side.wait_event(fork)
        for it in self.items:
            if it["spec"].bits == 4:
                self.zq.widen_int4_weights(it["Wq"], it["spec"].K, Wq8=it["W8"], stream=self.side)
        join.record(self.side)
        joined = False
        for it in self.items:
            self.run_ln(it, stream)
            if it["spec"].bits == 4:
                if not joined:
                    main.wait_event(join)
                    joined = True
                self.zq.gemm_w8a8(it["Xq"], it["s_tok"], it["W8"], it["s_grp"], it["b"], Y=it["Y"],
                                  stream=stream)
            else:
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


class KernelTimer:
    """Device time of one launch sequence: a CUDA graph of R x [L2 flush,
    body] minus a graph of R x [L2 flush], divided by R, timed with CUDA
    events on the launching stream.  (Events between the launches of an
    eager step would add each kernel's launch latency, which the step's
    graph with programmatic dependent launch hides.)"""

    def __init__(self, flush_buf, stream, reps):
        self.flush_buf = flush_buf
        self.stream = stream
        self.reps = reps
        self.base = self._graph(None)

    def _graph(self, fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(self.reps):
                flush_l2(self.flush_buf)
                if fn is not None:
                    fn()
        return g

    def _time(self, g):
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        g.replay()
        e1.record(self.stream)
        e1.synchronize()
        return e0.elapsed_time(e1)

    def ms(self, fn):
        """The flush-only graph is timed next to the kernel's graph, three
        times each in alternation, and the smallest of each is used, so a
        drift of the flush's own time (clocks under the power cap) does not
        land on the kernel."""
        fn()  # once outside capture: workspaces and launch settings exist first
        torch.cuda.synchronize()
        g = self._graph(fn)
        tk, tb = [], []
        for _ in range(3):
            tb.append(self._time(self.base))
            tk.append(self._time(g))
        del g
        return max(min(tk) - min(tb), 1e-6) / self.reps


def record_step(step, warmup):
    """Warm the step up, then record it once as a CUDA graph (the paper's
    remedy for launch overhead on small models).  Returns (graph or None,
    error, kernel launches of one step)."""
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    n0 = step.zq.launch_count()
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step.run()
        launches = step.zq.launch_count() - n0
        for _ in range(warmup):
            graph.replay()
        torch.cuda.synchronize()
        return graph, None, launches
    except Exception as exc:  # capture refused: report it and time eager launches
        torch.cuda.synchronize()
        n0 = step.zq.launch_count()
        step.run()
        torch.cuda.synchronize()
        return None, f"{type(exc).__name__}: {exc}", step.zq.launch_count() - n0


def kernel_times(step, timer):
    kern = {}
    for it in step.items:
        s = it["spec"]
        kern[(s.name, "ln")] = timer.ms(lambda it=it: step.run_ln(it))
        kern[(s.name, "gemm")] = timer.ms(lambda it=it: step.run_gemm(it))
    return kern


def gemm_kernel_name(spec, T):
    if spec.bits == 4:
        return "gemm_i8_kernel / gemv_i8_kernel (W4A8: INT4 widened to int8 before the MMA)"
    return "gemm_i8_kernel / gemv_i8_kernel (W8A8, tcgen05 kind::i8 or dp4a)"


def roofline_entry(layer, spec, T, ms, peaks, peak_src, peak_tops, int8_cublas):
    """Roofline of one GEMM launch: tensor-bound when its arithmetic intensity
    is above the ridge point (peak ops / HBM bandwidth), else HBM-bound."""
    ops = 2.0 * T * spec.N * spec.K
    nbytes = gemm_bytes(spec, T)
    hbm = float(peaks["hbm_gbs"])
    ridge = peak_tops * 1e12 / (hbm * 1e9)
    tensor = ops / nbytes > ridge
    base = {"kernel": f"{gemm_kernel_name(spec, T)}, {layer} {spec.name} {spec.K}->{spec.N} "
                      f"W{spec.bits}A8 T={T}",
            "time_us": round(ms * 1e3, 2),
            "traffic": traffic_for(layer, spec, T),
            "algorithmic_bytes": nbytes, "ops": ops}
    if tensor:
        achieved = ops / (ms * 1e-3) / 1e12
        r = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak_tops, 1),
             "unit": "TOPS", "frac": round(achieved / peak_tops, 4),
             "peak_source": f"{peak_src}: 2 x bf16 dense "
                            f"{'burst' if peak_src == 'measured' else 'fallback'} "
                            f"({peaks['bf16_tflops']} TFLOP/s), nominal int8/bf16 ratio 2"}
        if int8_cublas:
            r["frac_of_cublas_int8"] = round(achieved / int8_cublas, 4)
        r["hbm_gbs_achieved"] = round(nbytes / (ms * 1e-3) / 1e9, 1)
    else:
        achieved = nbytes / (ms * 1e-3) / 1e9
        r = {"bound": "hbm", "achieved": round(achieved, 1), "peak": round(hbm, 1), "unit": "GB/s",
             "frac": round(achieved / hbm, 4),
             "peak_source": f"{peak_src}: copy bandwidth (hbm_gbs)",
             "weight_gbs": round(spec.N * spec.K * spec.bits / 8 / (ms * 1e-3) / 1e9, 1),
             "tops": round(ops / (ms * 1e-3) / 1e12, 2)}
    r.update(base)
    return r


def measure_int8_peak(device, stream):
    """cuBLAS's dense INT8 GEMM (torch._int_mm) at 8192^3, best of 10 with
    CUDA events: a measured INT8 tensor rate on this GPU, reported next to
    the 2 x bf16 denominator.  Returns TOPS or None."""
    try:
        n = 8192
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device)
        bt = b.t()
        for _ in range(3):
            torch._int_mm(a, bt)
        torch.cuda.synchronize()
        best = None
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            torch._int_mm(a, bt)
            e1.record(stream)
            e1.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        del a, b, bt
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except Exception:
        torch.cuda.synchronize()
        return None


def step_summary(step, kern, ms_steps, launches):
    ops = gemm_ops(step.specs, step.T)
    ms = sum(ms_steps) / len(ms_steps)
    return {
        "workload": workload_name(step.layer, step.T, step.specs),
        "ms_per_step": round(ms, 5),
        "ms_per_step_median": round(statistics.median(ms_steps), 5),
        "ms_per_step_best": round(min(ms_steps), 5),
        "tops": round(ops / (ms * 1e-3) / 1e12, 2),
        "weight_gbs": round(weight_bytes(step.specs) / (ms * 1e-3) / 1e9, 1),
        "gpu_launches_per_step": launches,
        "kernels_us": {f"{n}.{k}": round(v * 1e3, 2) for (n, k), v in kern.items()},
        "ln_quant_gbs": round(sum(ln_bytes(s, step.T) for s in step.specs)
                              / (sum(v for (n, k), v in kern.items() if k == "ln") * 1e-3) / 1e9, 1),
    }


def dominant_gemm(step, kern):
    it = max(step.items, key=lambda it: kern[(it["spec"].name, "gemm")])
    return it["spec"], kern[(it["spec"].name, "gemm")]


def fp16_reference(step, timer, with_int8=False):
    """Library references, measured after this library's kernels: the same
    GEMM shapes in fp16 through cuBLAS (torch.addmm: X W^T + b), per GEMM and
    as a graph of the fp16 layer (torch layer_norm before the GEMMs that have
    a LayerNorm), and cuBLAS's INT8 GEMM (torch._int_mm, int32 out, no
    scales) on the dominant shape.  Context, not part of the path."""
    out = {}
    try:
        fns = [lambda it=it: torch.addmm(it["b"], it["X"], it["W16"].t()) for it in step.items]
        for fn in fns:
            fn()  # cuBLAS sets up its handle and workspace outside any capture
        torch.cuda.synchronize()
        per = {it["spec"].name: timer.ms(fn) for it, fn in zip(step.items, fns)}

        def fp16_layer():
            for it in step.items:
                x = it["X"]
                if it["gamma"] is not None:
                    x = torch.nn.functional.layer_norm(x, (x.shape[1],), it["gamma"], it["beta"],
                                                       1e-5)
                torch.addmm(it["b"], x, it["W16"].t())

        fp16_layer()
        torch.cuda.synchronize()
        out = {"gemm_us": {n: round(v * 1e3, 2) for n, v in per.items()},
               "step_us": round(timer.ms(fp16_layer) * 1e3, 2)}
        if with_int8 and step.T > 16:
            it = max(step.items, key=lambda it: it["spec"].N * it["spec"].K)
            s = it["spec"]
            x8 = torch.randint(-127, 128, (step.T, s.K), dtype=torch.int8, device=it["X"].device)
            w8 = torch.randint(-127, 128, (s.N, s.K), dtype=torch.int8, device=it["X"].device)
            torch._int_mm(x8, w8.t())
            torch.cuda.synchronize()
            out["cublas_int8_us"] = {s.name: round(timer.ms(lambda: torch._int_mm(x8, w8.t())) * 1e3,
                                                   2)}
    except Exception as exc:
        torch.cuda.synchronize()
        out = {"error": f"{type(exc).__name__}: {exc}"}
    return out


def l2_bytes(device) -> int:
    try:
        return int(torch.cuda.get_device_properties(device).L2_cache_size)
    except Exception:
        return 126 * 1024 * 1024


def time_graph_after_flush(g, flush_buf, stream, tries=3):
    """Smallest device time (ms) of one replay of graph g, the L2 flushed
    before each replay (outside the events)."""
    best = None
    for _ in range(tries):
        flush_l2(flush_buf)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        e1.synchronize()
        ms = e0.elapsed_time(e1)
        best = ms if best is None else min(best, ms)
    return best


def rotated_decode(zq, step, flush_buf, stream, peaks, peak_src, peak_tops, int8_cublas):
    """Weight streaming as a model's decode pass sees it: consecutive launches
    read different weights.  Each GEMM is replayed back to back over R copies
    of its quantized weights whose total exceeds twice the L2 (so every launch
    streams its weights from HBM; the L2 is also flushed before the replay),
    and the layer step is replayed over L copies of the layer's weights (L
    layers in a row).  Times are per launch and per layer."""
    need = 2 * l2_bytes(step.items[0]["Wq"].device)
    copies = {}
    for it in step.items:
        nb = it["Wq"].numel() * it["Wq"].element_size()
        r = max(2, min(16, -(-need // nb)))
        copies[it["spec"].name] = [it["Wq"]] + [it["Wq"].clone() for _ in range(r - 1)]
    torch.cuda.synchronize()

    def gemm_on(it, Wq):
        fn = zq.gemm_w4a8 if it["spec"].bits == 4 else zq.gemm_w8a8
        fn(it["Xq"], it["s_tok"], Wq, it["s_grp"], it["b"], Y=it["Y"])

    gemm_ms = {}
    for it in step.items:
        ws = copies[it["spec"].name]
        for w in ws:  # warm: the workspace and the launch settings exist before capture
            gemm_on(it, w)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for w in ws:
                gemm_on(it, w)
        gemm_ms[it["spec"].name] = time_graph_after_flush(g, flush_buf, stream) / len(ws)
        del g
    layers = min(len(v) for v in copies.values())

    def layer_steps():
        for l in range(layers):
            for it in step.items:
                step.run_ln(it)
                gemm_on(it, copies[it["spec"].name][l])

    layer_steps()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer_steps()
    layer_ms = time_graph_after_flush(g, flush_buf, stream) / layers
    del g
    wb = weight_bytes(step.specs)
    dom = max(step.items, key=lambda it: gemm_ms[it["spec"].name])
    out = {
        "method": f"each GEMM replayed back to back over 2-16 copies of its weights (more than 2x the "
                  f"L2 in total), and {layers} layers' steps in a row, L2 flushed before each replay",
        "layers": layers,
        "ms_per_layer": round(layer_ms, 5),
        "weight_gbs": round(wb / (layer_ms * 1e-3) / 1e9, 1),
        "frac_of_hbm": round(wb / (layer_ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]), 4),
        "gemm_us": {n: round(v * 1e3, 2) for n, v in gemm_ms.items()},
        "gemm_copies": {n: len(v) for n, v in copies.items()},
        "roofline": roofline_entry(step.layer, dom["spec"], step.T, gemm_ms[dom["spec"].name], peaks,
                                   peak_src, peak_tops, int8_cublas),
        "gemms": {it["spec"].name: roofline_entry(step.layer, it["spec"], step.T,
                                                  gemm_ms[it["spec"].name], peaks, peak_src,
                                                  peak_tops, int8_cublas) for it in step.items},
    }
    del copies
    torch.cuda.empty_cache()
    return out


def measure_step(zq, weights, T, args, timer, flush_buf, stream, dist_on, inputs=None):
    """Build one layer step at T tokens, record it as a graph, time K steps
    (L2 flushed before each) and every kernel on its own."""
    step = LayerStep(zq, weights, T, torch.device("cuda", torch.cuda.current_device()), inputs)
    # The per-kernel timings call zq_gemm_w4a8 on its own, which needs more
    # library workspace than the step (its INT4 widening goes there): size it
    # for those calls first, so that the step's graph records the final buffer.
    for it in step.items:
        step.run_gemm(it)
    graph, graph_error, launches = record_step(step, args.warmup)
    run_step = graph.replay if graph is not None else step.run
    barrier(dist_on)
    total_ms, per_step = time_steps(run_step, args.steps, flush_buf, stream)
    barrier(dist_on)
    total_ms = max_over_ranks(total_ms, dist_on)
    kern = kernel_times(step, timer)
    return step, graph, graph_error, launches, total_ms / args.steps, per_step, kern


def gpu_arm(args, dist_on, rank, world):
    from int4_quantized_transformer_b200 import zq

    device = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    peak_tops = INT8_PER_BF16 * float(peaks["bf16_tflops"])
    layer, T = args.layer, default_tokens(args)
    stream = torch.cuda.current_stream()
    flush_buf = make_flush_buffers(device)
    timer = KernelTimer(flush_buf, stream, max(3, min(args.steps, 20)))

    # ---- the headline step: inputs resident in HBM, K steps timed
    cpu_inputs = [synth.gemm_inputs(layer, i, T) for i in range(len(synth.LAYERS[layer].gemms))]
    weights = LayerWeights(zq, layer, device)
    with ClockSampler(torch.cuda.current_device()) as clk:
        step, graph, graph_error, launches, ms_per_step, per_step, kern = measure_step(
            zq, weights, T, args, timer, flush_buf, stream, dist_on, inputs=cpu_inputs)
    rc, detail = zq.device_status()
    if rc != zq.ZQ_OK:
        raise RuntimeError(f"device status {rc} ({detail}) after timing")
    run_step = graph.replay if graph is not None else step.run
    specs = step.specs
    ops = gemm_ops(specs, T)
    eager_ms, _ = time_steps(step.run, max(3, args.steps // 2), flush_buf, stream)
    eager_ms /= max(3, args.steps // 2)
    int8_cublas = measure_int8_peak(device, stream)

    dom_spec, dom_ms = dominant_gemm(step, kern)
    gemm_ms = sum(v for (n, k), v in kern.items() if k == "gemm")
    roof = roofline_entry(layer, dom_spec, T, dom_ms, peaks, peak_src, peak_tops, int8_cublas)
    roof["all_gemms_tops"] = round(ops / (gemm_ms * 1e-3) / 1e12, 1)
    roof["kernel_time_method"] = (f"CUDA graph of {timer.reps} x [L2 flush, kernel] minus "
                                  f"{timer.reps} x [L2 flush]")
    roof["int8_cublas_8192_tops"] = None if int8_cublas is None else round(int8_cublas, 1)
    per_gemm = {s.name: roofline_entry(layer, s, T, kern[(s.name, "gemm")], peaks, peak_src,
                                       peak_tops, int8_cublas) for s in specs}

    # ---- end to end through the C ABI: pinned host inputs in, outputs out
    h_in = [it["X"].cpu().pin_memory() for it in step.items]
    h_out = [torch.empty(it["Y"].shape, dtype=torch.float16).pin_memory() for it in step.items]
    h2d = sum(x.numel() * 2 for x in h_in)
    d2h = sum(y.numel() * 2 for y in h_out)

    def e2e_step():
        for it, hx in zip(step.items, h_in):
            it["X"].copy_(hx, non_blocking=True)
        run_step()
        for it, hy in zip(step.items, h_out):
            hy.copy_(it["Y"], non_blocking=True)

    for _ in range(2):
        e2e_step()
    barrier(dist_on)
    e2e_ms, _ = time_steps(e2e_step, args.steps, flush_buf, stream)
    barrier(dist_on)
    e2e_ms = max_over_ranks(e2e_ms, dist_on) / args.steps
    del h_in, h_out

    fp16 = fp16_reference(step, timer, with_int8=True)
    if "gemm_us" in fp16:
        fp16["gemm_speedup"] = round(sum(fp16["gemm_us"].values()) / (gemm_ms * 1e3), 3)
        fp16["step_speedup"] = round(fp16["step_us"] / (ms_per_step * 1e3), 3)
    wquant_ms = weights.wquant_ms
    summary = step_summary(step, kern, per_step, launches)
    del graph, step

    # ---- weight-streaming (decode) steps and the smaller prefill layer:
    # every GEMM gets its roofline (HBM at these token counts)
    decode = {}
    extra = {}
    if not args.no_decode:
        for dl, dT in DECODE_CASES:
            if weights.layer != dl:
                del weights
                torch.cuda.empty_cache()
                weights = LayerWeights(zq, dl, device)
            st, g, _, la, ms, per, kn = measure_step(zq, weights, dT, args, timer, flush_buf,
                                                     stream, dist_on)
            d = step_summary(st, kn, per, la)
            ds, dms = dominant_gemm(st, kn)
            d["roofline"] = roofline_entry(dl, ds, dT, dms, peaks, peak_src, peak_tops, int8_cublas)
            d["gemms"] = {s.name: roofline_entry(dl, s, dT, kn[(s.name, "gemm")], peaks, peak_src,
                                                 peak_tops, int8_cublas) for s in st.specs}
            d["fp16_cublas"] = fp16_reference(st, timer)
            d["rotated"] = rotated_decode(zq, st, flush_buf, stream, peaks, peak_src, peak_tops,
                                          int8_cublas)
            decode[f"{dl}_T{dT}"] = d
            del st, g
        for el, eT in EXTRA_PREFILL:
            del weights
            torch.cuda.empty_cache()
            weights = LayerWeights(zq, el, device)
            st, g, _, la, ms, per, kn = measure_step(zq, weights, eT, args, timer, flush_buf, stream,
                                                     dist_on)
            d = step_summary(st, kn, per, la)
            ds, dms = dominant_gemm(st, kn)
            d["roofline"] = roofline_entry(el, ds, eT, dms, peaks, peak_src, peak_tops, int8_cublas)
            d["fp16_cublas"] = fp16_reference(st, timer)
            extra[f"{el}_T{eT}"] = d
            del st, g
    rc, detail = zq.device_status()
    if rc != zq.ZQ_OK:
        raise RuntimeError(f"device status {rc} ({detail}) after the decode steps")

    cfg = bench_config(layer, T, world)
    cfg["launch"] = "cuda graph replay of the step" if graph_error is None else "eager launches"
    res = {
        "metric": METRIC,
        "value": round(whole_job_tops(ops, world, ms_per_step), 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "ms_per_step_median": summary["ms_per_step_median"],
        "ms_per_step_best": summary["ms_per_step_best"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic (seeded N(0,1) activations with outlier channels, N(0,sigma) weights)",
        "config": cfg,
        "eager_ms_per_step": round(eager_ms, 5),
        "graph_error": graph_error,
        "weight_gbs": round(world * weight_bytes(specs) / (ms_per_step * 1e-3) / 1e9, 1),
        "roofline": roof,
        "gemms": per_gemm,
        "kernels_us": summary["kernels_us"],
        "ln_quant_gbs": summary["ln_quant_gbs"],
        "fp16_cublas": fp16,
        "decode": decode,
        "extra_prefill": extra,
        "offline_wquant_ms": round(wquant_ms, 2),
        "e2e": {"value": round(whole_job_tops(ops, world, e2e_ms), 2), "unit": "TOPS",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(layer, T, args.cpu_tokens, args.cpu_tokens_1,
                                           cpu_inputs)
    return res


# ------------------------------------------------------------------ CPU oracle arm

def prepare_oracle(layer, T, inputs=None):
    import oracle

    inputs = inputs or [synth.gemm_inputs(layer, i, T)
                        for i in range(len(synth.LAYERS[layer].gemms))]
    ready = []
    for gi in inputs:
        wq, sg = oracle.quantize_weights_groupwise(gi.W.numpy(), gi.spec.g, gi.spec.bits)
        ready.append({"spec": gi.spec, "X": gi.X.numpy(), "wq": wq, "sg": sg, "b": gi.b.numpy(),
                      "gamma": None if gi.gamma is None else gi.gamma.numpy(),
                      "beta": None if gi.beta is None else gi.beta.numpy()})
    return ready


def _oracle_rows(g, r0, r1):
    import oracle

    xq, st = oracle.ln_quant(g["X"][r0:r1], g["gamma"], g["beta"], 1e-5)
    oracle.linear_q(xq, st, g["wq"], g["sg"], g["b"])


def oracle_step(ready, rows, pool=None, threads=1):
    """The oracle's hot path on the first `rows` tokens: LN+quant, exact int
    GEMM, dequant, for every GEMM of the layer.  With a thread pool the rows
    are split into `threads` contiguous chunks (the C oracle runs without the
    interpreter lock, so the chunks run on separate cores)."""
    for g in ready:
        if pool is None:
            _oracle_rows(g, 0, rows)
            continue
        cuts = [rows * i // threads for i in range(threads + 1)]
        list(pool.map(lambda ab: _oracle_rows(g, *ab),
                      [(a, b) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]))


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(layer, T, rows_all, rows_one, inputs=None):
    """The oracle as it stands on the host cores: all cores (threads over
    token-row chunks) and one core, each on a bounded token sample."""
    ready = prepare_oracle(layer, T, inputs)
    specs = [g["spec"] for g in ready]
    threads = _host_threads()
    rows_all = min(rows_all, T)
    rows_one = min(rows_one, T)
    with cf.ThreadPoolExecutor(max_workers=threads) as pool:
        t0 = time.perf_counter()
        oracle_step(ready, rows_all, pool, threads)
        dt_all = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle_step(ready, rows_one)
    dt_one = time.perf_counter() - t0
    v_all = gemm_ops(specs, rows_all) / dt_all / 1e12
    v_one = gemm_ops(specs, rows_one) / dt_one / 1e12
    return {"value": round(v_all, 6), "unit": "TOPS", "cores": threads, "kind": "oracle",
            "sample": f"{rows_all} of {T} tokens of every GEMM of the {layer} step (LN+quant, exact "
                      f"int GEMM, dequant), plain C on {threads} threads over token-row chunks, "
                      f"{dt_all:.1f} s",
            "single_core": {"value": round(v_one, 6), "unit": "TOPS", "cores": 1,
                            "sample": f"{rows_one} of {T} tokens of every GEMM, single-threaded, "
                                      f"{dt_one:.1f} s"},
            "host_cpu_model": host_cpu_model(), "host_cpus": os.cpu_count()}


def reference_arm(args, rank, world):
    layer, T = args.layer, default_tokens(args)
    rows = min(args.ref_tokens, T)
    ready = prepare_oracle(layer, T)
    specs = [g["spec"] for g in ready]
    threads = _host_threads()
    with cf.ThreadPoolExecutor(max_workers=threads) as pool:
        for _ in range(args.warmup):
            oracle_step(ready, rows, pool, threads)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle_step(ready, rows, pool, threads)
        dt = (time.perf_counter() - t0) / args.steps
    val = round(gemm_ops(specs, rows) / dt / 1e12, 6)
    sample = (f"{rows} of {T} tokens of every GEMM of the {layer} step per timed step (oracle: "
              f"LN+quant, exact int GEMM, dequant), plain C on {threads} threads over token-row "
              f"chunks")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": val, "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": bench_config(layer, T, world),
        "cpu_baseline": {"value": val, "unit": "TOPS", "cores": threads, "kind": "oracle",
                         "sample": sample, "host_cpu_model": host_cpu_model(),
                         "host_cpus": os.cpu_count()},
        "e2e": {"value": val, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="zq", choices=["zq", "reference"])
    ap.add_argument("--layer", default=HEADLINE[0], choices=sorted(synth.LAYERS))
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--cpu-tokens", type=int, default=256,
                    help="token sample of the all-core CPU baseline")
    ap.add_argument("--cpu-tokens-1", type=int, default=32,
                    help="token sample of the single-core CPU baseline")
    ap.add_argument("--ref-tokens", type=int, default=32,
                    help="token sample per step of the reference (oracle) arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode steps and the extra prefill layer")
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
