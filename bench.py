#!/usr/bin/env python
"""Benchmark of the routed MoE expert forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--only] [--impl ours|reference]

A step is one pass of the whole hot path on one batch of synthetic input:
moe_route (router top-k) followed by moe_forward (permute, gate/up with
SwiGLU, down, combine) of one layer. The headline workload is the large FP8
layer (T=4096, H=7168, I=2048, E=256, k=8, e4m3 experts with UE8M0 block
scales), the largest of the layers; the line's top-level numbers are its own.
Every other workload (tiny, decode, prefill, skewed, fp8_decode, fp4,
fp4_decode) is measured
the same way in the same process and reported under "per_config" (--only
skips them; --workload picks another headline).

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream, with a 256 MiB buffer written between steps (outside
the events) so that no step finds the previous step's data in L2. Inputs are
resident in HBM when a step starts. Multi-GPU (torchrun, one process per GPU)
runs independent replicas: the layer has no data-path exchange; the elapsed
time is the max over ranks and the value counts the tokens of all ranks.

Each workload's entry carries: tokens/s and TFLOP/s, the stage breakdown
(events recorded by moe_forward_timed), the roofline of the dominant kernel
(algorithmic bytes or FLOPs per launch over its measured duration, against
MEASURED_PEAKS.json), the end-to-end number through the public API with host
buffers (H2D of x and logits, D2H of the output inside the timed region:
batches pipelined through MoEPipeline, copies overlapping the previous and
next batch's compute, where a step streams more than twice L2; else one batch
at a time with L2 flushed between them; the other mode's figure rides along),
the CPU oracle timed on a bounded sample (rank 0, N=1), the number of our
kernel launches in the timed region, and the SM clocks sampled while the
GPU was busy with it.

--impl reference times the CPU oracle (test infrastructure, unmodified) on the
headline workload, a bounded sample of tokens per step, on rank 0 only.
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
import torch  # noqa: E402

from mixture_experts_routed_moe_b200 import inputs as G  # noqa: E402

METRIC = "MoE layer tokens/sec and TFLOP/s (% of BF16/FP8 peak or HBM BW) on 1 B200"
DEFAULT_WORKLOAD = "fp8"
# measured after the headline, in this order, under "per_config"
OTHER_WORKLOADS = ["tiny", "decode", "prefill", "skewed", "fp8_decode", "fp4", "fp4_decode"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20  # B200 L2

# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture each; a record counts only while its kernel's source file is
# unchanged (first 16 hex digits of the .cu file's SHA-256). "scaled" says how
# a capture of a smaller case was brought to one full launch.
NCU_TRAFFIC = {
    ("decode", "small_gemm_bf16_kernel<true>"): {"bytes": 489132032, "src": "166e86239f1883b1", "scaled": None},
    ("prefill", "grouped_gemm_bf16_kernel<256,true>"): {"bytes": 1211534704, "src": "d64f0e084cc41143",
                                                         "scaled": None},
    ("fp8", "grouped_gemm_e4m3_kernel<true>"): {"bytes": 8316361440, "src": "dc4eb5e6a4256cd9",
                                                "scaled": "T=1024, E=64 capture x4 (rows and experts)"},
    ("skewed", "grouped_gemm_bf16_kernel<256,true>"): {"bytes": 2192461184, "src": "d64f0e084cc41143",
                                                        "scaled": None},
    ("fp8_decode", "decode_e4m3_gate_up_kernel"): {
        "bytes": 2906970427, "src": "308da7bb6a248115",
        "scaled": "T=16, E=64 capture (59 experts touched) x 1.593, the ratio of algorithmic bytes (94 touched)"},
    ("fp4", "grouped_gemm_fp4_kernel<1,0>"): {"bytes": 6701524992, "src": "1c31b7fc99a0883e",
                                             "scaled": "T=1024, E=64 capture x4 (rows and experts)"},
    ("fp4_decode", "decode_fp4_gate_up_kernel"): {
        "bytes": 1757986265, "src": "6fbeaf275d39845d",
        "scaled": "T=16, E=64 capture (59 experts touched) x 1.627, the ratio of algorithmic bytes (96 touched)"},
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_hash(name):
    path = os.path.join(ROOT, "mixture_experts_routed_moe_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_init(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:  # host-only runs of the multi-rank plumbing (barrier, max over ranks)
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU oracle (the baseline and the reference arm)
# ---------------------------------------------------------------------------

class _HostExperts:
    """Host copies of the experts a sample touches (made outside the timing)."""

    def __init__(self, wl, seed, experts, name, codes=False):
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        self.shape = (wl.E,)
        self.d = {}
        for e in experts:
            t = G.make_expert_weights(wl, seed, int(e), device=dev)[name].cpu()
            self.d[int(e)] = t.view(torch.uint8).numpy() if codes else t.float().numpy()

    def __getitem__(self, e):
        return self.d[int(e)]


def oracle_sample_rate(wl, seed, n_tokens, steps=1, warmup=0, min_seconds=0.0):
    """Times the oracle's route + eager forward on the first n_tokens tokens,
    `steps` passes, or more until the timed passes add up to min_seconds (at
    most 200). Returns (tokens/s, seconds per step, BLAS threads, times)."""
    from oracle import moe_oracle as O

    x, logits = G.make_activations(wl, seed)
    toks = np.arange(min(n_tokens, wl.T))
    L = logits.numpy()[toks]
    xs = x.float().numpy()[toks]
    idx0, _, _ = O.route(L, wl.k)
    experts = np.unique(idx0)
    fp8 = wl.wdtype == "e4m3"
    fp4 = wl.wdtype == "e2m1"
    V = {n: _HostExperts(wl, seed, experts, n, codes=fp8 or fp4) for n in
         (("w_gate_up", "w_down", "sw_gate_up", "sw_down") if fp8 or fp4 else ("w_gate_up", "w_down"))}
    times = []
    i = 0
    while i < warmup + steps or (sum(times) < min_seconds and len(times) < 200):
        t0 = time.perf_counter()
        idx, w, _ = O.route(L, wl.k)
        if fp8:
            O.moe_forward_fp8(xs, idx, w, V["w_gate_up"], V["sw_gate_up"], V["w_down"], V["sw_down"])
        elif fp4:
            O.moe_forward_fp4(xs, idx, w, V["w_gate_up"], V["sw_gate_up"], V["w_down"], V["sw_down"])
        else:
            O.moe_forward(xs, idx, w, V["w_gate_up"], V["w_down"])
        if i >= warmup:
            times.append(time.perf_counter() - t0)
        i += 1
    try:
        from threadpoolctl import threadpool_info

        threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count() or 1
    per_step = sum(times) / len(times)
    return len(toks) / per_step, per_step, threads, times


def oracle_sample_tokens(wl):
    """Tokens per oracle sample, sized for roughly 10-30 s of CPU work: the
    eager loop's cost is dominated by converting each touched expert's weights
    to float64 (dequantising them for e4m3), about 3*H*I elements per expert."""
    per_expert = 3 * wl.H * wl.I * (4 if wl.wdtype in ("e4m3", "e2m1") else 1)
    budget = 3.0e9  # element conversions
    experts = max(1, int(budget // per_expert))
    return max(1, min(wl.T, 16, experts // wl.k))


def run_reference(args, world, rank):
    wl = G.WORKLOADS[args.workload]
    if rank != 0:
        return
    n = oracle_sample_tokens(wl)
    rate, per_step, threads, times = oracle_sample_rate(wl, G.default_seed(wl), n, steps=args.steps,
                                                        warmup=args.warmup)
    sample = f"first {n} of {wl.T} tokens per step (route + eager expert loop + combine, float64 NumPy)"
    line = {
        "metric": METRIC, "impl": "reference", "value": rate, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, "oracle"),
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def workload_config(wl, path):
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k, "wdtype": wl.wdtype,
            "path": path, "l2": "flushed between steps (256 MiB write)", "parallelism": "replicas",
            "launch": "CUDA graph of moe_route + moe_forward" if path != "oracle" else "cpu"}


def stage_roofline(wl, path, stage_ms, n_touched, peaks, peak_src):
    """Roofline of the slowest stage (its one kernel), algorithmic work per launch."""
    A, H, I = wl.A, wl.H, wl.I
    welem = {"e4m3": 1, "e2m1": 0.5}.get(wl.wdtype, 2)
    fp4 = wl.wdtype == "e2m1"
    names = {1: "gate_up", 2: "down"}
    s = max((1, 2), key=lambda i: stage_ms[i])
    dur_s = stage_ms[s] / 1e3
    if path == "fused":
        # one launch does the whole forward (its time is the gate_up stage):
        # every touched expert's weights, x read and out written once
        dur_s = stage_ms[1] / 1e3
        byts = n_touched * 3 * I * H * 2 + wl.T * H * 2 * 2
        ach = byts / dur_s / 1e9
        peak = peaks["hbm_gbs"]
        out = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
               "kernel": "fused_decode_kernel", "stage": "fused", "algorithmic_bytes": byts}
        kern, src = "fused_decode_kernel", "fused_decode.cu"
    elif path == "decode":
        fp8 = wl.wdtype == "e4m3"
        # e4m3: one UE8M0 byte per 128x128 weight block, h stored as e4m3 codes;
        # e2m1: one UE8M0 byte per 32 weights, h stored as bf16
        s_gu = (n_touched * (2 * I // 128) * (H // 128) if fp8 else
                n_touched * 2 * I * (H // 32) if fp4 else 0)
        s_d = (n_touched * (H // 128) * (I // 128) if fp8 else
               n_touched * H * (I // 32) if fp4 else 0)
        h_bytes = A * I * (1 if fp8 else 2)
        if s == 1:
            byts = int(n_touched * 2 * I * H * welem) + s_gu + wl.T * H * 2 + h_bytes
            kern, src = (("decode_e4m3_gate_up_kernel", "decode_e4m3.cu") if fp8 else
                         ("decode_fp4_gate_up_kernel", "decode_fp4.cu") if fp4 else
                         ("small_gemm_bf16_kernel<true>", "gemm_small.cu"))
        else:
            byts = int(n_touched * H * I * welem) + s_d + h_bytes + A * H * 2
            kern, src = (("decode_e4m3_down_kernel", "decode_e4m3.cu") if fp8 else
                         ("decode_fp4_down_kernel", "decode_fp4.cu") if fp4 else
                         ("small_gemm_bf16_kernel<false>", "gemm_small.cu"))
        # the bf16 DECODE GEMMs run on the tensor cores (bf16 MMAs, an
        # expert's tokens as N): many tokens per expert make them
        # tensor-bound, few make them HBM-bound; the e4m3 and e2m1 ones stream
        # on the CUDA cores
        flops = (4 if s == 1 else 2) * A * H * I
        t_tensor = 0.0 if (fp8 or fp4) else flops / (peaks["bf16_tflops"] * 1e12)
        if t_tensor > byts / (peaks["hbm_gbs"] * 1e9):
            ach = flops / dur_s / 1e12
            out = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                   "frac": ach / peaks["bf16_tflops"], "peak_source": "measured bf16 burst (the MMA is bf16)",
                   "algorithmic_flops": flops}
        else:
            ach = byts / dur_s / 1e9
            peak = peaks["hbm_gbs"]
            out = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak}
        out.update({"kernel": kern, "stage": names[s], "algorithmic_bytes": byts})
    else:
        # the stage is bound by the tensor pipe or by HBM, whichever takes
        # longer at its measured peak: bf16 prefill shapes are tensor-bound,
        # the FP8 layer (256 experts, ~128 rows each) streams ~11 GB of weights
        # and is HBM-bound
        flops = (4 if s == 1 else 2) * A * H * I
        fp8 = wl.wdtype == "e4m3"
        aelem = 1 if fp8 else 2  # activation bytes (e4m3 codes, or bf16 for the bf16 and e2m1 layers)
        if s == 1:
            byts = int(n_touched * 2 * I * H * welem + A * H * aelem + A * I * aelem
                       + (n_touched * (2 * I // 128) * (H // 128) + A * (H // 128) * 4 + A * (I // 128) * 4 if fp8
                          else n_touched * 2 * I * (H // 32) if fp4 else 0))
        else:
            byts = int(n_touched * H * I * welem + A * I * aelem + A * H * 2
                       + (n_touched * (H // 128) * (I // 128) + A * (I // 128) * 4 if fp8
                          else n_touched * H * (I // 32) if fp4 else 0))
        if fp4:
            # the codes are widened to bf16 ahead of bf16 MMAs
            tpeak, how = peaks["bf16_tflops"], "measured bf16 burst (the MMA is bf16)"
            kern, src = ("grouped_gemm_fp4_kernel<1,0>" if s == 1 else "grouped_gemm_fp4_kernel<0,0>"), \
                "gemm_fp4.cu"
        elif fp8:
            tpeak, how = 2.0 * peaks["bf16_tflops"], "2x measured bf16 (nominal fp8:bf16 ratio)"
            kern, src = ("grouped_gemm_e4m3_kernel<true>" if s == 1 else "grouped_gemm_e4m3_kernel<false>"), \
                "gemm_e4m3.cu"
        else:
            tpeak, how = peaks["bf16_tflops"], "measured bf16 burst"
            # gate/up: single-CTA kernel; down: the CTA-pair kernel when H % 256 == 0
            if s == 1:
                kern, src = "grouped_gemm_bf16_kernel<256,true>", "gemm_bf16.cu"
            else:
                kern, src = (("grouped_gemm_bf16_pair_kernel", "gemm_bf16_pair.cu") if H % 256 == 0
                             else ("grouped_gemm_bf16_kernel<128,false>", "gemm_bf16.cu"))
        t_tensor = flops / (tpeak * 1e12)
        t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
        if t_tensor >= t_hbm:
            ach = flops / dur_s / 1e12
            out = {"bound": "tensor", "achieved": ach, "peak": tpeak, "unit": "TFLOP/s", "frac": ach / tpeak,
                   "peak_source": how}
        else:
            ach = byts / dur_s / 1e9
            out = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                   "frac": ach / peaks["hbm_gbs"], "tensor_frac": flops / dur_s / 1e12 / tpeak}
        out.update({"kernel": kern, "stage": names[s], "algorithmic_flops": flops, "algorithmic_bytes": byts})
    rec = NCU_TRAFFIC.get((wl.name, kern))
    live = rec is not None and rec["src"] == src_hash(src)
    out["traffic"] = rec["bytes"] if live else None
    if live and rec["scaled"]:
        out["traffic_scaled_from"] = rec["scaled"]
    out["peak_from"] = peak_src
    return out


def time_router(moe, wl, seed, xd, flush, stream, K, W, world, peaks):
    """The fused router (moe_router: x W_r^T and the top-k routing in one
    kernel) on the workload's tokens, with router weights ~ N(0, 0.02): its own
    CUDA-event time per launch, L2 flushed between launches, and its roofline
    (algorithmic bytes x + W_r + routing outputs; FLOPs 2*T*H*E)."""
    w_r = G.make_router_weights(wl, seed, device=xd.device)
    # one launch captured in a CUDA graph, so the events time the kernel and
    # not the host's call overhead
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(max(W, 1)):
            moe.router(xd, w_r, wl.k)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.router(xd, w_r, wl.k)
    for _ in range(W):
        g.replay()
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        ev_s[i].record(stream)
        g.replay()
        ev_e[i].record(stream)
    torch.cuda.synchronize()
    del g
    ms = max_over_ranks(sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(K)), world) / K
    flops = 2 * wl.T * wl.H * wl.E
    byts = wl.T * wl.H * 2 + wl.E * wl.H * 2 + wl.T * wl.k * 8
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        ach = flops / (ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"]}
    else:
        ach = byts / (ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"]}
    roof.update({"kernel": "router_kernel", "algorithmic_flops": flops, "algorithmic_bytes": byts})
    return {"ms": ms, "tokens_per_s": wl.T / (ms / 1e3), "launches": K, "roofline": roof}


def measure(moe, wl, args, world, rank, local, peaks, peak_src):
    """One workload: the timed graph steps, the eager stage breakdown, the
    end-to-end steps with host buffers, the roofline of the dominant kernel and
    (rank 0, N=1) the CPU oracle on a bounded sample. Returns its JSON dict."""
    seed = G.default_seed(wl)
    dev = torch.device("cuda", local if world > 1 else 0)
    x, logits = G.make_activations(wl, seed)
    W = G.make_weights(wl, seed, device=dev)
    xd, ld = x.to(dev), logits.to(dev)
    layer = moe.MoELayer(W["w_gate_up"], W["w_down"], wl.k, W.get("sw_gate_up"), W.get("sw_down"), path=args.path)
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, wl.wdtype, args.path)
    lay = moe.workspace_layout(shape)
    path = moe.PATH_NAMES[lay.path]
    stream = torch.cuda.current_stream()

    def new_events(n):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    # the timed step is the captured graph of moe_route + moe_forward
    graph = moe.MoEGraph(layer, wl.T, dev)
    graph.x.copy_(xd)
    graph.logits.copy_(ld)
    for _ in range(args.warmup):
        flush.zero_()
        graph.replay()
        layer(xd, ld, out=out)
    torch.cuda.synchronize()
    ws = layer._workspace(wl.T, dev)
    if moe.read_device_status(ws) != 0:
        raise RuntimeError("device status reports an error after warm-up")
    n_touched = int(ws[lay.hdr:lay.hdr + 12].view(torch.int32)[1].item())

    K = args.steps
    ev_s, ev_e = new_events(K), new_events(K)
    clocks = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    for i in range(K):
        flush.zero_()
        ev_s[i].record(stream)
        graph.replay()
        ev_e[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    step_ms = [ev_s[i].elapsed_time(ev_e[i]) for i in range(K)]
    total_ms = max_over_ranks(sum(step_ms), world)

    # stage breakdown (and the dominant kernel's duration): the same kernels
    # launched eagerly through moe_forward_timed, on the same inputs
    st_s, st_ev = new_events(K), [new_events(5) for _ in range(K)]
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        st_s[i].record(stream)
        layer(xd, ld, out=out, events=st_ev[i])
    torch.cuda.synchronize()
    stage_ms = {j: sum(st_ev[i][j - 1].elapsed_time(st_ev[i][j]) for i in range(K)) / K for j in range(1, 5)}
    route_ms = sum(st_s[i].elapsed_time(st_ev[i][0]) for i in range(K)) / K
    eager_ms = sum(st_s[i].elapsed_time(st_ev[i][4]) for i in range(K)) / K

    # end to end through the public API with host buffers. Serial: per step,
    # H2D of x and logits into the graph's inputs, the graph, D2H of the
    # output, on one stream (L2 flushed before each step, outside the events).
    xh = x.pin_memory()
    lh = logits.pin_memory()
    oh = [torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    e2e_s, e2e_e = new_events(K), new_events(K)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        e2e_s[i].record(stream)
        res = graph(xh, lh)
        oh[0].copy_(res, non_blocking=True)
        e2e_e[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_serial_ms = max_over_ranks(sum(e2e_s[i].elapsed_time(e2e_e[i]) for i in range(K)), world)
    if not torch.equal(graph.out, out) or not torch.equal(oh[0], out.cpu()):
        raise RuntimeError("graph replay and eager forward disagree")
    # Pipelined (MoEPipeline): batch i's copy-in and batch i-1's copy-out
    # overlap batch i's graph; one device-timed span from the first copy-in to
    # the last copy-out. Larger layers stream more than L2 every step, so the
    # span needs no flush; where the touched weights fit twice in L2 the flush
    # has to run on the compute stream before every batch, inside the span,
    # and the serial figure (flush outside the events) is the e2e value.
    weight_bytes = n_touched * 3 * wl.H * wl.I * {"e4m3": 1, "e2m1": 0.5}.get(wl.wdtype, 2)
    flush_inside = weight_bytes < 2 * L2_BYTES
    pipe = moe.MoEPipeline(layer, wl.T, dev)
    hook = flush.zero_ if flush_inside else None
    for i in range(max(args.warmup, 2)):
        pipe.submit(xh, lh, oh[i % 2], before_compute=hook)
    pipe.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(pipe.copy_in)
    for i in range(K):
        pipe.submit(xh, lh, oh[i % 2], before_compute=hook)
    pipe.compute.wait_stream(pipe.copy_in)
    pipe.copy_out.wait_stream(pipe.compute)
    ev1.record(pipe.copy_out)
    pipe.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    if not (torch.equal(oh[0], out.cpu()) and torch.equal(oh[1], out.cpu())):
        raise RuntimeError("pipelined steps and eager forward disagree")
    del pipe

    router_line = None
    if args.router and wl.E <= 256:
        router_line = time_router(moe, wl, seed, xd, flush, stream, K, args.warmup, world, peaks)

    # route, permute, gate/up, down, combine; the e4m3 DECODE path adds the
    # per-token x quantisation and the h quantisation; FUSED is route + one kernel
    # route, permute (one kernel up to 256 tokens, else three) plus a row-staging
    # kernel where the single-block permute does not copy the rows itself
    # (more than 32768 elements to copy, or the e4m3 DECODE path's per-token
    # quantisation), gate/up, down (and the e4m3 DECODE path's h quantisation),
    # combine; FUSED is route + one kernel
    copies_rows = path == "prefill" or (path == "decode" and wl.wdtype == "bf16")
    stage_launch = ((wl.T <= 256 and copies_rows and wl.A * wl.H > 32768)
                    or (path == "decode" and wl.wdtype == "e4m3"))
    per_step_launches = (2 if path == "fused" else
                         1 + (1 if wl.T <= 256 else 3) + int(stage_launch) + 2 + 1
                         + (1 if path == "decode" and wl.wdtype == "e4m3" else 0))
    tokens = wl.T * K * world
    line = {
        "value": tokens / (total_ms / 1e3), "unit": "tokens/s", "ms_per_step": total_ms / K,
        "tflops": wl.flops() * K * world / (total_ms / 1e3) / 1e12,
        "dtype": wl.wdtype, "config": workload_config(wl, path),
        "stages_ms": {"route": route_ms, "permute": stage_ms[1], "gate_up": stage_ms[2], "down": stage_ms[3],
                      "combine": stage_ms[4], "eager_step": eager_ms},
        "touched_experts": n_touched,
        "roofline": stage_roofline(wl, path, {1: stage_ms[2], 2: stage_ms[3]}, n_touched, peaks, peak_src),
        "e2e": ({"value": tokens / (e2e_serial_ms / 1e3), "unit": "tokens/s",
                 "h2d_bytes_per_step": x.numel() * 2 + logits.numel() * 4, "d2h_bytes_per_step": wl.T * wl.H * 2,
                 "mode": "serial: copy-in, graph, copy-out on one stream per step, L2 flushed between steps",
                 "pipelined_value": tokens / (e2e_ms / 1e3),
                 "pipelined_l2": "flushed before every batch inside the span"}
                if flush_inside else
                {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                 "h2d_bytes_per_step": x.numel() * 2 + logits.numel() * 4, "d2h_bytes_per_step": wl.T * wl.H * 2,
                 "mode": "MoEPipeline: copy-in, graph and copy-out on three streams, two batches in flight",
                 "l2": f"not flushed: each step streams {weight_bytes / 1e9:.2f} GB of weights, more than L2",
                 "serial_value": tokens / (e2e_serial_ms / 1e3)}),
        "gpu_launches": per_step_launches * K,
        "clocks": clk,
    }
    if router_line is not None:
        line["router"] = router_line
    del graph, layer, W, ws, flush, out, xd, ld
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = oracle_sample_tokens(wl)
        rate, per_step, threads, times = oracle_sample_rate(wl, seed, n, steps=1, warmup=0, min_seconds=10.0)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": f"first {n} of {wl.T} tokens, {len(times)} passes "
                                          f"({per_step:.2f} s each, {sum(times):.1f} s in all)"}
    return line


def run_ours(args, world, rank, local):
    import mixture_experts_routed_moe_b200 as moe

    peaks, peak_src = load_peaks()
    wl = G.WORKLOADS[args.workload]
    head = measure(moe, wl, args, world, rank, local, peaks, peak_src)
    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.wdtype,
            "data": "synthetic (seeded N(0,1) activations and logits, N(0,0.02) weights)"}
    line.update({k: v for k, v in head.items() if k not in ("value", "unit", "ms_per_step", "dtype")})
    if not args.only and wl.name != "custom":
        per = {}
        for name in [n for n in [DEFAULT_WORKLOAD] + OTHER_WORKLOADS if n != wl.name]:
            log(f"measuring {name}")
            per[name] = measure(moe, G.WORKLOADS[name], args, world, rank, local, peaks, peak_src)
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(G.WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", action="store_true", help="measure the chosen workload alone (no per_config)")
    ap.add_argument("--path", choices=["auto", "prefill", "decode", "fused"], default="auto",
                    help="execution path of every measured layer (default: the library's choice)")
    ap.add_argument("--router", action="store_true",
                    help="also time the fused router (router GEMM + top-k) on the workload's tokens")
    ap.add_argument("--shape", default=None,
                    help="T,H,I,E,k,wdtype: a custom layer instead of a named workload (profiling-sized cases)")
    args = ap.parse_args()
    if args.shape:
        T, H, I, E, k, wd = args.shape.split(",")
        G.WORKLOADS["custom"] = G.Workload("custom", int(T), int(H), int(I), int(E), int(k), wdtype=wd)
        args.workload = "custom"
    if args.warmup < 3 and args.impl == "ours":
        log("note: fewer than 3 warm-up steps")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_init(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
