#!/usr/bin/env python
"""Forward throughput of the top-k gated MoE FFN layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl moe|reference]

A step is one moe_layer_forward (gate GEMM + normalisation/top-k, permutation
with capacity, both grouped expert GEMMs, combine) over one batch of
synthetic tokens already resident in HBM; by default it is replayed from a
CUDA graph.  The headline workload is the Mixtral-8x7B-shaped dropless layer
(T 16384, d 4096, 8 SwiGLU experts of 14336, top-2), the largest that fits
one GPU; the FastMoE Transformer-XL layer is timed the same way and reported
under "extra".  Between timed steps a 512 MiB memset flushes the 126 MB L2, and
each step is bracketed by its own CUDA events (the flush is outside them).
Under torchrun each rank runs an independent replica on its own token shard
(weak scaling; no collective on the data path) and the reported time is the
maximum over ranks.

One JSON line is printed by rank 0.  ``--impl reference`` times the float64
CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import moe_workloads as mw  # noqa: E402

METRIC = "MoE layer fwd tokens/s at 1 B200; % bf16 tensor peak (GEMM), % HBM BW (permute)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "mixture_experts_layer_logit_b200", "csrc")
# source files of each expert kernel (the DRAM traffic ncu measured is only
# reported while they are unchanged)
KERNEL_SOURCES = {
    "tc_expert_mlp": ["gemm_mlp.cu", "gemm_common.cuh", "tc_ptx.cuh"],
    "tc_grouped_gemm_pair": ["gemm_tc2.cu", "gemm_common.cuh", "tc_ptx.cuh"],
    "tc_grouped_gemm": ["gemm_tc.cu", "gemm_common.cuh", "tc_ptx.cuh"],
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=mw.BENCH_WORKLOAD, choices=sorted(mw.WORKLOADS))
    ap.add_argument("--extra", default=",".join(mw.BENCH_EXTRA_WORKLOADS),
                    help="comma-separated workloads also timed on the device (1 GPU only); '' for none")
    ap.add_argument("--hidden", default="f16", choices=["f16", "bf16"],
                    help="element type of the expert hidden activation and W2 on the bf16 path")
    ap.add_argument("--impl", default="moe", choices=["moe", "reference"])
    ap.add_argument("--no-graph", action="store_true", help="launch the C ABI call directly instead of a graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip timing the layer's backward")
    ap.add_argument("--no-fp8", action="store_true", help="skip timing the FP8-weight decode layer")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle time budget for cpu_baseline")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def graph_kernel_nodes(graph) -> int:
    """Kernel nodes of a captured CUDA graph (kept un-instantiated by keep_graph)."""
    from cuda.bindings import runtime as rt
    g = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
    err, _, n = rt.cudaGraphGetNodes(g, 0)
    assert err == rt.cudaError_t.cudaSuccess, err
    err, nodes, n = rt.cudaGraphGetNodes(g, n)
    assert err == rt.cudaError_t.cudaSuccess, err
    kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
    return sum(1 for nd in nodes[:n] if rt.cudaGraphNodeGetType(nd)[1] == kernel)


def workload_config(w: mw.Workload, n_gpus: int, graph: bool, hidden: str = "f16"):
    return {"workload": w.name, "tokens_per_gpu": w.T, "global_batch": w.T * n_gpus, "d_model": w.d,
            "experts": w.E, "ffn_hidden": w.F, "top_k": w.k, "activation": w.act,
            "capacity_factor": w.capacity_factor if w.capacity_factor > 0 else "dropless",
            "lambda": w.lam, "gate_bias": "zipf1.2" if w.zipf_bias else None,
            "hidden_dtype": hidden if w.dtype == mw.BF16 else "f32",
            "precision": ("x, W_gate, W1 bf16; h and W2 " + hidden + "; fp32 accumulation; out fp32")
            if w.dtype == mw.BF16 else "fp32 throughout", "out_dtype": "f32",
            "parallelism": "replicas" if n_gpus == 1 else f"dp{n_gpus} replicas",
            "l2": "flushed between steps (512 MiB memset outside the timed events)",
            "cuda_graph": graph}


# ------------------------------------------------------------ CPU oracle
def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        return int(n[0]) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_forward_fn(w: mw.Workload, inp: mw.Inputs, T_sample: int):
    import oracle
    from oracle import moe_oracle as om
    cfg = oracle.LayerConfig.from_workload(w, T_sample)
    x = mw.to_f64(inp.x[:T_sample])
    wg = mw.to_f64(inp.wg)
    w1, w2 = mw.F64Experts(inp.w1), mw.F64Experts(inp.w2)
    return lambda: om.forward(x, wg, inp.bias, w1, w2, cfg)


def reference_sample_tokens(w: mw.Workload) -> int:
    # full batch where one float64 forward takes about a second on the host
    flop_per_tok = (6 if w.act == mw.SWIGLU else 4) * w.d * w.F * w.k + 2 * w.d * w.E
    return int(max(64, min(w.T, 2.0e10 // flop_per_tok)))


def cpu_baseline(w: mw.Workload, inp: mw.Inputs, budget_s: float):
    Ts = reference_sample_tokens(w)
    fwd = oracle_forward_fn(w, inp, Ts)
    n, t0 = 0, time.perf_counter()
    while True:
        fwd()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": n * Ts / el, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} float64 oracle forwards of the first {Ts} of {w.T} tokens ({el:.1f} s, "
                      f"numpy/OpenBLAS on {blas_threads()} threads)"}


def run_reference(a):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    w = mw.WORKLOADS[a.workload]
    inp = mw.generate(w)
    Ts = reference_sample_tokens(w)
    fwd = oracle_forward_fn(w, inp, Ts)
    for _ in range(a.warmup):
        fwd()
    times = []
    for _ in range(a.steps):
        t0 = time.perf_counter()
        fwd()
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = Ts / (ms / 1e3)
    cores = blas_threads()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, 1, False, a.hidden),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"each step: float64 oracle forward of the first {Ts} of {w.T} tokens"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ clock sampling
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    p = [s.strip() for s in line.split(",")]
                    if len(p) >= 9 and p[1].replace(".", "").isdigit():
                        rows.append(p)
            os.unlink(self.path)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# --------------------------------------------------------------- roofline
def step_bytes(w: mw.Workload, offsets: np.ndarray):
    """Algorithmic bytes (and FLOPs for the experts) of one forward's steps."""
    b = 2 if w.dtype == mw.BF16 else 4
    T, d, F, k, E = w.T, w.d, w.F, w.k, w.E
    A = T * k
    kept = int(offsets[-1])
    F1 = F if w.act == mw.RELU else 2 * F
    touched = int(np.sum(np.diff(offsets) > 0))
    # h is 2-byte (bf16/fp16) on the bf16 path; yp and out are fp32 on both paths
    hb = 2 if w.dtype == mw.BF16 else 4
    return {
        "route": T * d * b + E * d * b + A * 8 + T * 4,
        "permute": (T * d + kept * d) * b + 4 * (2 * A + kept),
        # weights of the experts that received rows, xp read, h written and read, yp written
        "expert_ffn": touched * (F1 + F) * d * b + kept * (d * b + 2 * F * hb + d * 4),
        "combine": (kept * d + T * d) * 4 + 8 * A,
        # the fused steps 4-5: as expert_ffn, but out (T x d fp32) written instead of yp
        "experts_combine": touched * (F1 + F) * d * b + kept * (d * b + 2 * F * hb) + T * d * 4 + 8 * kept,
        "expert_flops": 2 * kept * d * (F1 + F),
        "weight_bytes": touched * (F1 + F) * d * b,
    }


def fused_combine(w: mw.Workload) -> bool:
    """The forward fuses step 5 into the expert kernel for bf16 layers with k <= 2."""
    return w.dtype == mw.BF16 and w.k <= 2


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summaries (profiles/traffic.json), if they were taken on the current
    kernel sources (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        e = d[f"{kernel}@{workload}"]
        if e["source_sha256_16"] == source_hash(kernel):
            return float(e["traffic_bytes_per_launch"])
    except Exception:
        pass
    return None


# ------------------------------------------------------- data-parallel plumbing
def replica_inputs(w: mw.Workload, rank: int) -> mw.Inputs:
    """Each rank is an independent replica: the same expert and gate weights,
    its own shard of tokens (x drawn with shard index = rank)."""
    return mw.generate(w, shard=rank)


def reduce_max_over_ranks(v: float, world: int, device) -> float:
    """The slowest rank's time (only collective of the benchmark, never on the
    data path)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_second(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's step time."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------------------------ main
class Layer:
    """One workload's inputs, weights and buffers on the device."""

    def __init__(self, moe, w: mw.Workload, rank: int, dev, hidden: str):
        import torch
        self.w = w
        self.inp = replica_inputs(w, rank)
        self.cfg = moe.make_config(w.T, w.d, w.E, w.F, w.k, w.act, w.dtype, w.capacity_factor, w.lam,
                                   hidden if w.dtype == mw.BF16 else None)
        self.tdt = torch.bfloat16 if w.dtype == mw.BF16 else torch.float32
        self.x = mw.to_device(self.inp.x, dev)
        self.wg, self.bias = mw.to_device(self.inp.wg, dev), mw.to_device(self.inp.bias, dev)
        self.w1 = mw.to_device(self.inp.w1, dev)
        # weight preparation at load time (not part of a step): W2 in the hidden type
        # (the bf16 original is kept for the FP8 weight preparation)
        self.w2_src = mw.to_device(self.inp.w2, dev)
        self.w2 = moe.prepare_w2(self.cfg, self.w2_src)
        nbytes, self.lay = moe.moe_workspace_size(self.cfg)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.out = torch.empty((w.T, w.d), dtype=torch.float32, device=dev)
        self.stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device=dev)
        self.moe = moe

    def fwd(self, x=None, out=None, stats=None):
        self.moe.moe_layer_forward(self.cfg, self.x if x is None else x, self.wg, self.bias, self.w1, self.w2,
                                   self.out if out is None else out, self.stats if stats is None else stats,
                                   self.ws)


def timed(fn, steps, flush):
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in evs:
        if flush is not None:
            flush.zero_()
        e0.record()
        fn()
        e1.record()
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in evs]


def capture(L: Layer, no_graph: bool):
    """(run, launches per step, graph): one forward captured as a CUDA graph;
    its kernel nodes are the launches of a step."""
    import torch
    L.fwd()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(graph):
        L.fwd()
    launches = graph_kernel_nodes(graph)
    if no_graph:
        graph.reset()
        return L.fwd, launches, None
    return graph.replay, launches, graph


def expert_kernel(w: mw.Workload):
    """(kernel name, launches per step, description) of the expert step the forward runs."""
    fused = fused_combine(w)
    pair = w.dtype == mw.BF16 and w.T * w.k >= 512 * w.E
    if w.dtype != mw.BF16:
        return "simt_grouped_gemm", 2, "simt_grouped_gemm (fp32 expert FFN, 2 launches)"
    if not pair:
        if fused:
            return "tc_expert_mlp", 1, "tc_expert_mlp (steps 4-5 in one launch: both expert layers + the combine)"
        return "tc_expert_mlp", 1, "tc_expert_mlp (step 4 in one launch: both expert layers, writing yp)"
    if fused:
        return ("tc_grouped_gemm_pair", 2, "tc_grouped_gemm_pair (2-SM pair tiles; layer 1 with the activation, "
                "then layer 2 with the combine fused: 2 launches)")
    return "tc_grouped_gemm_pair", 2, "tc_grouped_gemm_pair (2-SM pair tiles; layer 1 + layer 2: 2 launches)"


def breakdown_roofline(L: Layer, a, flush, pk, pk_src, dev):
    """Per-step times through the step entry points, and the roofline of the
    dominant kernel (the expert step the forward runs), from CUDA events."""
    import torch
    moe, w, lay, ws = L.moe, L.w, L.lay, L.ws
    A = w.T * w.k
    sv = lambda off, n, dt: ws[off:off + n * torch.tensor([], dtype=dt).element_size()].view(dt)  # noqa: E731
    idx, tw, gap = sv(lay.topk_idx, A, torch.int32), sv(lay.topk_w, A, torch.float32), sv(lay.gap, w.T, torch.float32)
    counts, kept = sv(lay.counts, w.E, torch.int32), sv(lay.kept, w.E, torch.int32)
    offs = sv(lay.offsets, w.E + 1, torch.int32)
    row_of, src_tok = sv(lay.row_of, A, torch.int32), sv(lay.src_tok, A, torch.int32)
    hdt = {moe.MOE_DTYPE_F16: torch.float16, moe.MOE_DTYPE_BF16: torch.bfloat16}.get(L.cfg.hidden_dtype,
                                                                                      torch.float32)
    xp, h, yp = sv(lay.xp, A * w.d, L.tdt), sv(lay.h, A * w.F, hdt), sv(lay.yp, A * w.d, torch.float32)
    scr = ws[lay.scratch:]
    pm = torch.empty(w.E, dtype=torch.float32, device=dev)
    zl = torch.empty(1, dtype=torch.float32, device=dev)
    names = ["route", "permute", "expert_ffn", "combine"]
    acc = {n: 0.0 for n in names}
    for i in range(a.warmup + a.steps):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        ev[0].record()
        moe.moe_route(L.cfg, L.x, L.wg, L.bias, idx, tw, gap, pm, scr, z_loss=zl)
        ev[1].record()
        moe.moe_permute(L.cfg, L.x, idx, gap, pm, counts, kept, offs, row_of, src_tok, xp, L.stats, scr)
        ev[2].record()
        moe.moe_expert_ffn(L.cfg, xp, offs, L.w1, L.w2, h, yp, L.stats, scr)
        ev[3].record()
        moe.moe_combine(L.cfg, yp, row_of, tw, L.out)
        ev[4].record()
        torch.cuda.synchronize()
        if i >= a.warmup:
            for j, n in enumerate(names):
                acc[n] += ev[j].elapsed_time(ev[j + 1])
    breakdown = {n: acc[n] / a.steps for n in names}
    offsets = offs.cpu().numpy()
    sb = step_bytes(w, offsets)
    # The forward's own steps 4-5 on bf16 layers with k <= 2: the expert kernel
    # with the combine fused in, fed the forward's permuted rows and row
    # weights; out is zeroed before each call, outside the events.
    fused = fused_combine(w)
    if fused:
        row_w = sv(lay.row_w, A, torch.float32)
        out_fc = torch.empty_like(L.out)
        t_fc = 0.0
        for i in range(a.warmup + a.steps):
            flush.zero_()
            out_fc.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            moe.moe_expert_ffn_combine(L.cfg, xp, offs, src_tok, row_w, L.w1, L.w2, h, out_fc, L.stats, ws)
            e1.record()
            torch.cuda.synchronize()
            if i >= a.warmup:
                t_fc += e0.elapsed_time(e1)
        breakdown["experts_combine"] = t_fc / a.steps
        del out_fc
    rl = {}
    for n in ["route", "permute", "combine"]:
        gbs = sb[n] / (breakdown[n] * 1e-3) / 1e9
        rl[n] = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                 "frac": gbs / pk["hbm_gbs"], "bytes": sb[n]}
    step = "experts_combine" if fused else "expert_ffn"
    t_ffn = breakdown[step] * 1e-3
    tflops = sb["expert_flops"] / t_ffn / 1e12
    gbs = sb[step] / t_ffn / 1e9
    t_hbm = sb[step] / (pk["hbm_gbs"] * 1e9)
    t_tc = sb["expert_flops"] / (pk["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    kname, nl, kdesc = expert_kernel(w)
    traffic = committed_traffic(kname, w.name) if kname in KERNEL_SOURCES else None
    if bound == "hbm":
        roofline = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": gbs / pk["hbm_gbs"], "traffic": traffic}
    else:
        roofline = {"bound": "tensor", "achieved": tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": tflops / pk["bf16_tflops"], "traffic": traffic}
    roofline.update({
        "kernel": kdesc, "peak_kind": "burst (the expert step is timed on its own)",
        "launches_per_step": nl, "algorithmic_bytes_per_launch": sb[step] / nl,
        "algorithmic_flops_per_launch": sb["expert_flops"] / nl, "launch_ms": breakdown[step] / nl,
        "tensor_tflops": tflops, "tensor_frac": tflops / pk["bf16_tflops"],
        "tensor_frac_of_sustained": tflops / pk["bf16_tflops_sustained"], "hbm_gbs": gbs,
        "hbm_frac": gbs / pk["hbm_gbs"], "weight_bytes": sb["weight_bytes"],
        "peak_source": "measured (MEASURED_PEAKS.json)" if pk_src == "measured" else "fallback (recipe)",
        "other_steps": rl})
    return breakdown, roofline


def backward_measure(L: Layer, a, flush, pk, dev):
    """The layer's backward (moe_layer_backward: all five expert GEMMs, the
    gate's gradient, dx and dW_gate) after a forward of the same inputs,
    timed with CUDA events, L2 flushed before each call."""
    import torch
    moe, w = L.moe, L.w
    F1 = w.F if w.act == mw.RELU else 2 * w.F
    dout = torch.randn((w.T, w.d), dtype=torch.float32, device=dev, generator=torch.Generator(dev).manual_seed(0))
    dx = torch.empty((w.T, w.d), dtype=torch.float32, device=dev)
    dwg = torch.empty((w.E, w.d), dtype=torch.float32, device=dev)
    dbg = torch.empty((w.E,), dtype=torch.float32, device=dev)
    dw1 = torch.empty((w.E, F1, w.d), dtype=torch.float32, device=dev)
    dw2 = torch.empty((w.E, w.d, w.F), dtype=torch.float32, device=dev)
    stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device=dev)
    bws = torch.empty(moe.moe_backward_workspace_size(L.cfg), dtype=torch.uint8, device=dev)
    L.fwd()

    def bwd():
        moe.moe_layer_backward(L.cfg, L.x, L.wg, L.bias, L.w1, L.w2, dout, 0.01, 0.001, L.ws, dx, dwg, dbg,
                               dw1, dw2, None, stats, bws)

    timed(bwd, a.warmup, flush)
    t = timed(bwd, a.steps, flush)
    ms = sum(t) / len(t)
    st = moe.read_stats(stats)
    assert st["status"] == 0, f"device status {st['status']} in the backward"
    kept = int(moe.read_stats(L.stats)["rows_kept"])
    flops = 2.0 * kept * w.d * (3 * F1 + 2 * w.F)
    tf = flops / (ms * 1e-3) / 1e12
    res = {"ms_per_step": ms, "tokens_per_s": w.T / (ms * 1e-3), "expert_gemm_flops": flops, "tflops": tf,
           "tensor_frac": tf / pk["bf16_tflops"], "tensor_frac_of_sustained": tf / pk["bf16_tflops_sustained"],
           "what": "moe_layer_backward after a forward: u recomputed, dh with the activation backward, dxp, dW2, "
                   "dW1 (tcgen05), gate gradient, dx, dW_gate; L2 flushed before each call"}
    del dw1, dw2, bws
    return res


def mxfp8_measure(moe, name: str, a, flush, pk, dev):
    """The layer with MX FP8 expert weights (moe_layer_forward_mxfp8) on one
    workload, replayed from a CUDA graph with the L2 flushed between steps,
    and its expert step (the padded quantised rows, both FP8 GEMMs) against
    the HBM bytes of the touched experts' FP8 weights."""
    import torch
    w = mw.WORKLOADS[name]
    L = Layer(moe, w, 0, dev, "f16")
    w1q, w1s, w2q, w2s = moe.prepare_mxfp8(L.cfg, L.w1, L.w2_src)
    ws = torch.empty(moe.moe_workspace_size_mxfp8(L.cfg), dtype=torch.uint8, device=dev)

    def fwd():
        moe.moe_layer_forward_mxfp8(L.cfg, L.x, L.wg, L.bias, w1q, w1s, w2q, w2s, L.out, L.stats, ws)

    fwd()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    timed(g.replay, a.warmup, flush)
    t = timed(g.replay, a.steps, flush)
    ms = sum(t) / len(t)
    st = moe.read_stats(L.stats)
    assert st["status"] == 0, f"device status {st['status']} on the FP8 layer"
    n, lay = moe.moe_workspace_size(L.cfg)
    offs = ws[lay.offsets:lay.offsets + 4 * (w.E + 1)].view(torch.int32).cpu().numpy()
    touched = int(np.sum(np.diff(offs) > 0))
    F1 = w.F1
    wbytes = touched * (F1 * w.d + w.d * w.F) * (1 + 1 / 32)   # E4M3 elements + one scale byte per 32
    kept = int(offs[-1])
    flops = 2.0 * kept * w.d * (F1 + w.F)
    res = {"value": w.T / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms, "workload": name,
           "weights": "MX FP8 (E4M3, UE8M0 scale per 32 along K), both expert layers",
           "touched_expert_weight_bytes": wbytes,
           "weight_stream_gbs_over_whole_forward": wbytes / (ms * 1e-3) / 1e9,
           "expert_flops": flops, "tflops_over_whole_forward": flops / (ms * 1e-3) / 1e12}
    del g, L, ws, w1q, w1s, w2q, w2s
    torch.cuda.empty_cache()
    return res


def e2e_measure(L: Layer, a, flush, graph_ok: bool, barrier, max_over_ranks, world: int, dev):
    """Every step copies its tokens from pinned host memory to the device, runs
    the layer through the C ABI and reads the output and statistics back.  Two
    buffer slots and three streams (host-to-device, compute, device-to-host)
    let the copies of one step overlap the compute of the next; each step
    still starts from a flushed L2."""
    import torch
    moe, w, x, out, stats = L.moe, L.w, L.x, L.out, L.stats
    x_host = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for _ in range(2)]
    for xh in x_host:
        xh.copy_(x.cpu())
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    st_host = [torch.empty(stats.shape, dtype=stats.dtype).pin_memory() for _ in range(2)]
    xs = [x, torch.empty_like(x)]
    outs = [out, torch.empty_like(out)]
    sts = [stats, torch.zeros_like(stats)]
    s_h2d, s_comp, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    slot_runs = []
    for i in range(2):
        def slot_fwd(i=i):
            L.fwd(xs[i], outs[i], sts[i])
        if not graph_ok:
            slot_runs.append(slot_fwd)
        else:
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s_comp):
                slot_fwd()
            slot_runs.append(g)
    ev_h2d = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_d2h = [torch.cuda.Event() for _ in range(2)]

    def pipelined(steps):
        for i in range(steps):
            k = i % 2
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(ev_comp[k])        # the layer of step i-2 has read xs[k]
                xs[k].copy_(x_host[k], non_blocking=True)
                ev_h2d[k].record(s_h2d)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_h2d[k])
                if i >= 2:
                    s_comp.wait_event(ev_d2h[k])        # step i-2's output has been read back
                flush.zero_()
                r = slot_runs[k]
                r.replay() if hasattr(r, "replay") else r()
                ev_comp[k].record(s_comp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_comp[k])
                out_host[k].copy_(outs[k], non_blocking=True)
                st_host[k].copy_(sts[k], non_blocking=True)
                ev_d2h[k].record(s_d2h)

    pipelined(a.warmup)
    torch.cuda.synchronize()
    barrier()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(s_h2d)
    s_comp.wait_event(e_start)
    s_d2h.wait_event(e_start)
    pipelined(a.steps)
    s_h2d.wait_stream(s_d2h)
    s_h2d.wait_stream(s_comp)
    e_end.record(s_h2d)
    torch.cuda.synchronize()
    barrier()
    e_ms = max_over_ranks(e_start.elapsed_time(e_end)) / a.steps
    assert int(st_host[(a.steps - 1) % 2].view(torch.int32)[6]) == 0, "device status after the e2e steps"
    res = {"value": world * w.T / (e_ms / 1e3), "unit": UNIT, "ms_per_step": e_ms,
           "h2d_bytes_per_step": x.numel() * x.element_size(),
           "d2h_bytes_per_step": out.numel() * out.element_size() + stats.numel(),
           "pipeline": "2 buffer slots; host-to-device, compute and device-to-host streams overlap across steps"}
    del slot_runs
    return res


def main():
    a = parse_args()
    if a.impl == "reference":
        return run_reference(a)

    import torch
    import torch.distributed as dist
    import mixture_experts_layer_logit_b200 as moe
    from mixture_experts_layer_logit_b200 import build as moe_build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != a.gpus:
        print(f"warning: --gpus {a.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0:
        moe_build.build()
    if world > 1:
        dist.barrier()
    moe.lib()

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(v: float) -> float:
        return reduce_max_over_ranks(v, world, dev)

    pk, pk_src = peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    # ---------------------------------------------------------- headline
    w = mw.WORKLOADS[a.workload]
    L = Layer(moe, w, rank, dev, a.hidden)
    run, launches_per_step, graph = capture(L, a.no_graph)
    timed(run, a.warmup, flush)
    barrier()
    gpu_id = str(local)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid).replace("GPU-", "")
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    barrier()
    times = timed(run, a.steps, flush)
    barrier()
    clocks = sampler.stop()
    total_ms = max_over_ranks(sum(times))
    ms = total_ms / a.steps
    value = job_tokens_per_second(world, w.T, ms)
    st = moe.read_stats(L.stats)
    assert st["status"] == 0, f"device status {st['status']}"

    breakdown = roofline = None
    if not a.no_breakdown:
        breakdown, roofline = breakdown_roofline(L, a, flush, pk, pk_src, dev)
    e2e = None
    if not a.no_e2e:
        e2e = e2e_measure(L, a, flush, graph is not None, barrier, max_over_ranks, world, dev)
    backward = None
    if world == 1 and not a.no_backward and w.dtype == mw.BF16:
        backward = backward_measure(L, a, flush, pk, dev)
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(w, L.inp, a.cpu_seconds)
    if graph is not None:
        del graph
    del run, L
    torch.cuda.empty_cache()

    # ------------------------------------------ further workloads (1 GPU only)
    extra = {}
    names = [n for n in a.extra.split(",") if n and n != a.workload] if world == 1 else []
    for name in names:
        we = mw.WORKLOADS[name]
        Le = Layer(moe, we, rank, dev, a.hidden)
        run_e, nl_e, g_e = capture(Le, a.no_graph)
        timed(run_e, a.warmup, flush)
        t_e = timed(run_e, a.steps, flush)
        ms_e = sum(t_e) / a.steps
        st_e = moe.read_stats(Le.stats)
        assert st_e["status"] == 0, f"device status {st_e['status']} on {name}"
        ent = {"value": we.T / (ms_e / 1e3), "unit": UNIT, "ms_per_step": ms_e,
               "config": workload_config(we, 1, g_e is not None, a.hidden), "gpu_launches_per_step": nl_e}
        if not a.no_breakdown:
            ent["breakdown_ms"], ent["roofline"] = breakdown_roofline(Le, a, flush, pk, pk_src, dev)
        extra[name] = ent
        if g_e is not None:
            del g_e
        del run_e, Le
        torch.cuda.empty_cache()

    if world == 1 and not a.no_fp8:
        extra["fine_decode_dropless_mxfp8"] = mxfp8_measure(moe, "fine_decode_dropless", a, flush, pk, dev)
        if a.workload != "fine_decode_dropless":
            extra[a.workload + "_mxfp8"] = mxfp8_measure(moe, a.workload, a, flush, pk, dev)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.dtype == mw.BF16 else "f32", "data": "synthetic",
                "config": workload_config(w, world, not a.no_graph, a.hidden),
                "gpu_launches": launches_per_step * a.steps,
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
                "breakdown_ms": breakdown,
                "stats": {"drop_rate": st["drop_rate"], "aux_loss": st["aux_loss"], "z_loss": st["z_loss"],
                          "rows_kept": st["rows_kept"],
                          "capacity": st["capacity"], "near_tie_count": st["near_tie_count"]},
                "backward": backward, "extra": extra}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
