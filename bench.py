#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 frozen-base linear layer on B200.

One step = forward + backward of the adapted projections of one workload, each
Y = X deq(W)^T + s (X A) B followed by dX, dA and dB, with the weights stored as
NF4 with double-quantized constants and quantized once before timing (model
load).  The headline workload is the largest single-GPU one: the three
LLaMA-65B-shaped projections W 8192x8192, 22016x8192 and 8192x22016 with 8192
tokens per GPU, LoRA r = 64, alpha = 16.  The LLaMA-7B-shaped projections (4096
tokens, r = 16) and the small single layer (16 tokens on W 1024x1024, reported in
microseconds) are measured after it.  Metric: fwd+bwd TFLOP/s of the algorithmic
FLOPs 4MNK + 6Mr(K+N) per projection.  Multi-GPU: data-parallel replicas (weak
scaling), each rank its own tokens, dA/dB all-reduced over NCCL each step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import tempfile
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS  # noqa: E402  (shapes and distributions of every workload)

METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4-weight HBM GB/s vs roofline, 1 B200"
HEADLINE = "llama65b"
WORKLOAD_TEXT = {
    "llama65b": ("LLaMA-65B-shaped projections W[N,K] in {8192x8192, 22016x8192, 8192x22016}, NF4 "
                 "block 64 / double-quant 256, W ~ N(0,0.015); 8192 tokens per GPU; LoRA r=64 "
                 "alpha=16; fwd+bwd"),
    "llama7b": ("LLaMA-7B-shaped projections W[N,K] in {4096x4096, 11008x4096, 4096x11008}, NF4 "
                "block 64 / double-quant 256, W ~ N(0,0.02); 4096 tokens per GPU; LoRA r=16 alpha=32; "
                "fwd+bwd"),
    "small": "single QLoRA linear W 1024x1024 NF4, 16 tokens, LoRA r=8 alpha=16; fwd+bwd",
}
WORKLOAD = WORKLOAD_TEXT[HEADLINE]
FLUSH_BYTES = 256 << 20
SKINNY = [(m, n, 4096) for n in (4096, 11008) for m in (1, 4, 16)]
BIG_N = 1_000_000_000
MERGE_SHAPE = (22016, 8192, 64)  # merge subpath: W [N, K] and adapter rank
GRAPH_STREAM_BYTES = 320 << 20   # weights streamed per graph replay of the decode measurement
SMALL_CALLS = 50


def step_flops(M, N, K, r):
    return 4.0 * M * N * K + 6.0 * M * r * (K + N)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p["bf16_tflops_sustained"]), sm_max_mhz=p.get("sm_max_mhz"),
                    src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sm_max_mhz=1965.0, src="fallback")


def source_hash(kernel_key):
    """Hash of the code that defines one kernel's launch: its own header, the
    shared device helpers, and the host function that configures the launch."""
    csrc = os.path.join(ROOT, "bit_nf4_quantized_19_b200", "csrc")
    files, launcher = {
        "qlora_gemm_kernel": (["gemm_kernel.cuh", "common.cuh"], "qlora_status launch_gemm("),
        "qlora_skinny_kernel": (["skinny_kernel.cuh", "common.cuh"], "qlora_status launch_skinny("),
    }[kernel_key]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(csrc, "qlora_nf4.cu")) as fh:
        text = fh.read()
    i = text.find(launcher)
    h.update(text[i:text.find("\n}\n", i)].encode() if i >= 0 else b"")
    return h.hexdigest()[:16]


def traffic_for(kernel_key):
    """dram bytes per launch from a committed ncu summary, or None when the
    summary is missing or was taken on different kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t.get(kernel_key)
        if e and e.get("source_hash") == source_hash(kernel_key):
            return e.get("bytes_per_launch")
    except Exception:
        pass
    return None


def smi_device_id(local: int, visible: str | None) -> str:
    """nvidia-smi's --id for CUDA device `local`: its entry in CUDA_VISIBLE_DEVICES
    (a physical index or a GPU UUID, both of which nvidia-smi accepts), else the
    index itself."""
    if visible:
        ids = [v.strip() for v in visible.split(",") if v.strip()]
        if 0 <= local < len(ids) and (ids[local].isdigit() or ids[local].startswith("GPU-")):
            return ids[local]
    return str(local)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 20 ms while running.
    Each sample carries nvidia-smi's own timestamp; summary() keeps the samples
    taken between entering and leaving the block (the timed region).  If
    nvidia-smi refuses that query, the sampler falls back to the same fields
    without the timestamp every 200 ms, and summary() then uses every sample."""
    BASIC = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    FIELDS = BASIC + ",timestamp"
    INTERVAL_MS = 20
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.fh = None
        self.t0 = self.t1 = None
        self.interval = self.INTERVAL_MS
        self.path = os.environ.get("QLORA_CLOCKS_CSV") or \
            os.path.join(tempfile.gettempdir(), f"qlora_clocks_{os.getpid()}_gpu{gpu_index}.csv")

    def _start(self, fields, interval_ms):
        """Start sampling.  False only if nvidia-smi is missing or exits within 3 s
        (a refused query); a slow first sample is not a failure."""
        self.interval = interval_ms
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={smi_device_id(self.gpu, os.environ.get('CUDA_VISIBLE_DEVICES'))}",
                 f"--query-gpu={fields}",
                 "--format=csv,noheader,nounits", "-lms", str(interval_ms)], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except Exception:
            self._stop()
            return False
        deadline = time.time() + 3.0
        while time.time() < deadline:
            if self.proc.poll() is not None:
                self._stop()
                return False
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)
        return True

    def _stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.proc = None
        if self.fh is not None:
            self.fh.close()
            self.fh = None

    def __enter__(self):
        if not self._start(self.FIELDS, self.INTERVAL_MS):
            self._start(self.BASIC, 200)
        time.sleep(0.1)
        self.t0 = time.time()
        return self

    def __exit__(self, *a):
        self.t1 = time.time()
        if self.proc is not None:
            time.sleep(2 * self.interval / 1000.0)
        self._stop()

    @staticmethod
    def _stamp(text):
        import datetime
        return datetime.datetime.strptime(text.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()

    def summary(self):
        try:
            rows = [l.strip().split(", ") for l in open(self.path) if l.strip()]
        except Exception:
            return None
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return None
        window = None
        if self.t0 is not None and self.t1 is not None:
            try:
                lo, hi = self.t0 - self.interval / 1000.0, self.t1 + self.interval / 1000.0
                inside = [r for r in rows if len(r) >= 10 and lo <= self._stamp(r[9]) <= hi]
                window = inside
            except Exception:
                window = None
        use = window if window else rows
        sm = [float(r[1]) for r in use if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in use if r[2].replace(".", "").isdigit()]
        watts = [float(r[3]) for r in use if r[3].replace(".", "").isdigit()]
        reasons = sorted({self.REASONS[i] for r in use for i in range(4)
                          if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(use), "in_timed_region": bool(window),
                "power_w": statistics.median(watts) if watts else None,
                "interval_ms": self.interval}


# ------------------------------------------------------------------ oracle baseline
def sample_problems(name, tokens, wrows):
    """The leading part of every projection of a workload, bit-identical to what the
    GPU arm runs on: the first `wrows` output features (rows of W) and the first
    `tokens` tokens; A and B whole."""
    from synth import linear_problem_rows
    wl = WORKLOADS[name]
    out = []
    for (M, N, K) in wl["shapes"]:
        p = linear_problem_rows(M, N, K, wl["r"], wl["alpha"], wl["w_std"], tokens, wrows, seed=0)
        out.append(dict(M=M, N=N, K=K, r=wl["r"], s=wl["alpha"] / wl["r"], W=p.W, X=p.X, A=p.A,
                        B=p.B, dY=p.dY))
    return out


def oracle_sample(problems, tokens, wrows, repeats=1):
    """Oracle fwd+bwd on a bounded sample of every projection: the first
    `tokens` tokens and the first `wrows` output features (dequant of those W
    rows included, as the method dequantizes every step).  Returns (flops, s)."""
    from oracle import linear as olin, nf4 as onf4
    quant = []
    for p in problems:
        rows_q = onf4.quantize_bf16(p["W"][:wrows].ravel())
        quant.append(rows_q)
    flops, t0 = 0.0, time.perf_counter()
    for _ in range(repeats):
        for p, q in zip(problems, quant):
            N, K = wrows, p["K"]
            Wd = onf4.dequantize(q["codes"], q["q8"], q["step"], N * K).reshape(N, K)
            X, A, B, dY = p["X"][:tokens], p["A"], p["B"][:, :wrows], p["dY"][:tokens, :wrows]
            Y, XA = olin.forward(X, Wd, A, B, p["s"])
            olin.backward(dY, X, Wd, A, B, p["s"], XA=XA)
            flops += step_flops(tokens, N, K, p["r"])
    return flops, time.perf_counter() - t0


def cpu_info():
    cores = len(os.sched_getaffinity(0))
    blas = None
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 0) for i in threadpool_info()), default=None)
    except Exception:
        pass
    return cores, blas


def host_problems(name, rank=0):
    """Seeded inputs of one workload (bf16 bits on the host).  The frozen W, A and B
    are the same on every rank; X and dY are each rank's own tokens."""
    from synth import linear_problem, normal_bf16
    wl = WORKLOADS[name]
    r, alpha, w_std = wl["r"], wl["alpha"], wl["w_std"]
    out = []
    for (M, N, K) in wl["shapes"]:
        p = linear_problem(M, N, K, r, alpha, w_std, seed=0)
        X, dY = p.X, p.dY
        if rank:
            X = normal_bf16(rank, f"X{M}x{N}x{K}r{r}", (M, K), 1.0)
            dY = normal_bf16(rank, f"dY{M}x{N}x{K}r{r}", (M, N), 1.0)
        out.append(dict(M=M, N=N, K=K, r=r, s=alpha / r, W=p.W, X=X, A=p.A, B=p.B, dY=dY))
    return out


def workload_flops(name):
    wl = WORKLOADS[name]
    return sum(step_flops(M, N, K, wl["r"]) for (M, N, K) in wl["shapes"])


def gemm_flops(name):
    """FLOPs of the fused GEMM launches of one step: forward 2MNK + 2MNr (its LoRA
    K-steps), dX 2MNK + 2MKr."""
    wl = WORKLOADS[name]
    r = wl["r"]
    return sum(4.0 * M * N * K + 2.0 * M * N * r + 2.0 * M * K * r for (M, N, K) in wl["shapes"])


# the bounded oracle samples: (tokens, output features) of every projection
CPU_SAMPLE = {"llama65b": (256, 1024), "llama7b": (512, 2048)}
REF_SAMPLE = {"llama65b": (64, 256)}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    tokens, wrows = REF_SAMPLE[HEADLINE]
    problems = sample_problems(HEADLINE, tokens, wrows)
    for _ in range(max(0, args.warmup)):
        oracle_sample(problems, tokens, wrows)
    fl, t = 0.0, 0.0
    for _ in range(args.steps):
        f, s = oracle_sample(problems, tokens, wrows)
        fl += f
        t += s
    cores, blas = cpu_info()
    v = fl / t / 1e12
    sample = (f"oracle (NumPy/SciPy, fp64 GEMMs) per step: all 3 projections, first {tokens} "
              f"tokens x first {wrows} output features, dequant of those rows included")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": blas or cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
class Workload:
    """Device-resident state of one workload: quantized weights, inputs, outputs,
    workspaces, the gradient bucket and pinned host copies of the inputs."""

    def __init__(self, q, torch, dev, name, rank, pinned=True):
        from bit_nf4_quantized_19_b200.dp import GradBucket
        self.q, self.torch, self.dev, self.name = q, torch, dev, name
        wl = WORKLOADS[name]
        self.shapes = wl["shapes"]
        self.r = wl["r"]
        hp = host_problems(name, rank)
        self.bucket = GradBucket([(N, K, self.r) for (_, N, K) in self.shapes], dev)
        self.layers = []

        def to_dev(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

        def to_pinned(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()

        for p, (dA, dB) in zip(hp, self.bucket.views):
            M, N, K, r = p["M"], p["N"], p["K"], p["r"]
            L = dict(M=M, N=N, K=K, r=r, s=p["s"], Wq=q.nf4_quantize(to_dev(p["W"])),
                     X=to_dev(p["X"]), dY=to_dev(p["dY"]), A=to_dev(p["A"]), B=to_dev(p["B"]),
                     Y=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                     XA=torch.empty(M, r, dtype=torch.float32, device=dev),
                     dX=torch.empty(M, K, dtype=torch.bfloat16, device=dev),
                     dA=dA, dB=dB, ws=q.make_workspace(M, N, K, r, dev))
            if pinned:
                L["hX"], L["hdY"] = to_pinned(p["X"]), to_pinned(p["dY"])
            self.layers.append(L)
        del hp
        self.flops = workload_flops(name)
        self.gemm_flops = gemm_flops(name)

    def run(self, inputs=None):
        """One fwd+bwd of every projection (optionally on other X / dY buffers), then
        the one exchange of data-parallel adapter training."""
        q = self.q
        for i, L in enumerate(self.layers):
            X, dY = (L["X"], L["dY"]) if inputs is None else inputs[i]
            q.linear_fwd(X, L["Wq"], L["A"], L["B"], L["s"], workspace=L["ws"], Y=L["Y"], XA=L["XA"])
            q.linear_bwd(dY, X, L["XA"], L["Wq"], L["A"], L["B"], L["s"],
                         workspace=L["ws"], dX=L["dX"], dA=L["dA"], dB=L["dB"])
        self.bucket.allreduce_()


def time_steps(torch, run, steps, flush, stream, barrier):
    """CUDA-event time of each of `steps` steps, the L2 flushed (256 MiB write)
    before every step; a barrier and a device synchronize on both sides."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        run()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    return [a.elapsed_time(b) for a, b in evs]


def kernel_profile(q, torch, run, steps, flush, stream, barrier):
    """A second pass of the same steps with the library's per-launch CUDA events on
    (kept out of the headline pass): per-kernel launches, time and share, and the
    launches per step."""
    q.profile_enable(True)
    time_steps(torch, run, steps, flush, stream, barrier)
    prof, nlaunch = q.profile_read()
    q.profile_enable(False)
    by = {}
    for kind, ms in prof:
        d = by.setdefault(kind, [0, 0.0])
        d[0] += 1
        d[1] += ms
    tot = sum(v[1] for v in by.values()) or 1.0
    kernels = {k: {"launches": v[0], "ms_total": round(v[1], 4), "share": round(v[1] / tot, 4)}
               for k, v in sorted(by.items(), key=lambda kv: -kv[1][1])}
    return kernels, by, nlaunch // max(1, steps)


def pick_peak(P, clk):
    """The bf16 denominator.  The burst figure applies to a timed region whose SM
    clock stayed at its maximum; the fraction at the sampled clock and against the
    sustained figure are reported beside it."""
    sm = (clk or {}).get("sm_mhz")
    smax = (clk or {}).get("sm_max_mhz") or P.get("sm_max_mhz")
    return P["bf16"], (sm / smax if sm and smax else None)


def gemm_roofline(wl, by, steps, P, clk):
    g_ms = by.get("gemm_fwd", [0, 0.0])[1] + by.get("gemm_dx", [0, 0.0])[1]
    g_n = by.get("gemm_fwd", [0, 0.0])[0] + by.get("gemm_dx", [0, 0.0])[0]
    achieved = wl.gemm_flops * steps / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None
    peak, clk_ratio = pick_peak(P, clk)
    return {"kernel": "qlora_gemm_kernel (fused NF4 dequant + tcgen05 GEMM + LoRA K-steps; fwd and dX)",
            "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": (achieved / peak) if achieved else None,
            "peak_source": f"{P['src']} bf16 burst (MEASURED_PEAKS.json: cuBLAS bf16, best of 10)",
            "frac_vs_sustained": (achieved / P["bf16_sus"]) if achieved else None,
            "frac_at_sampled_clock": (achieved / (peak * clk_ratio)) if achieved and clk_ratio else None,
            "avg_launch_ms": g_ms / max(1, g_n), "launches_per_step": g_n // max(1, steps),
            "flops_per_launch": wl.gemm_flops / max(1, g_n // max(1, steps)),
            "traffic": traffic_for("qlora_gemm_kernel"),
            "timing": "CUDA events around every GEMM launch, in a second timed pass of the same steps"}


def e2e_measure(torch, wl, steps, stream, barrier, world, dev):
    """The same step end to end through the public API: pinned host X and dY copied
    to the device every step (the next step's inputs upload on their own stream into
    the other of two device buffers while the current step computes, as a data
    loader would) and the fp32 gradients read back; every copy lies inside the
    timed region."""
    import torch.distributed as dist
    layers = wl.layers
    flat = wl.bucket.flat
    flat_host = torch.empty(flat.numel(), dtype=torch.float32).pin_memory()
    h2d = sum(L["hX"].numel() * 2 + L["hdY"].numel() * 2 for L in layers)
    d2h = flat_host.numel() * 4
    xfer = torch.cuda.Stream(device=dev)
    bufs = [[(L["X"], L["dY"]) for L in layers],
            [(torch.empty_like(L["X"]), torch.empty_like(L["dY"])) for L in layers]]
    uploaded = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]

    def upload(b):
        xfer.wait_event(consumed[b])
        with torch.cuda.stream(xfer):
            for (X, dY), L in zip(bufs[b], layers):
                X.copy_(L["hX"], non_blocking=True)
                dY.copy_(L["hdY"], non_blocking=True)
        uploaded[b].record(xfer)

    def step_on(b):
        stream.wait_event(uploaded[b])
        wl.run(bufs[b])
        consumed[b].record(stream)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    xfer.wait_event(e0)
    upload(0)
    for i in range(steps):
        if i + 1 < steps:
            upload((i + 1) % 2)
        step_on(i % 2)
        flat_host.copy_(flat, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    del bufs
    return {"value": world * wl.flops * steps / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "uploads": "next step's inputs overlap the current step (two buffers)"}


def secondary_workload(q, torch, dev, name, steps, warmup, flush, stream, P):
    """A further large-token workload at N = 1: median step, whole-step and GEMM
    roofline fractions."""
    wl = Workload(q, torch, dev, name, 0, pinned=False)
    for _ in range(warmup):
        wl.run()
    torch.cuda.synchronize()
    ms = time_steps(torch, wl.run, steps, flush, stream, lambda: None)
    kernels, by, per_step = kernel_profile(q, torch, wl.run, steps, flush, stream, lambda: None)
    med = statistics.median(ms)
    roof = gemm_roofline(wl, by, steps, P, None)
    out = {"workload": WORKLOAD_TEXT[name], "value": wl.flops / (med * 1e-3) / 1e12, "unit": "TFLOP/s",
           "ms_per_step": med, "ms_mean": statistics.mean(ms), "steps": steps,
           "step_frac_of_peak": wl.flops / (med * 1e-3) / 1e12 / P["bf16"],
           "gemm_achieved": roof["achieved"], "gemm_frac": roof["frac"],
           "launches_per_step": per_step, "kernels": kernels}
    del wl
    torch.cuda.empty_cache()
    return out


def small_layer(q, torch, dev, stream):
    """The small single layer (16 tokens, W 1024x1024, r = 8): fwd+bwd in
    microseconds, as separate calls (median of SMALL_CALLS, each bracketed by
    events) and inside one CUDA graph of SMALL_CALLS back-to-back calls."""
    wl = Workload(q, torch, dev, "small", 0, pinned=False)
    for _ in range(5):
        wl.run()
    torch.cuda.synchronize()
    ts = []
    for _ in range(SMALL_CALLS):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        wl.run()
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    plain_us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in ts)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(SMALL_CALLS):
            wl.run()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    a.record(cur)
    g.replay()
    b.record(cur)
    torch.cuda.synchronize()
    graph_us = 1e3 * a.elapsed_time(b) / SMALL_CALLS
    del g, wl
    return {"workload": WORKLOAD_TEXT["small"], "us_per_fwd_bwd": plain_us,
            "us_per_fwd_bwd_in_graph": graph_us, "calls": SMALL_CALLS,
            "TFLOP/s_in_graph": workload_flops("small") / (graph_us * 1e-6) / 1e12}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-subpaths", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the LLaMA-7B-shaped and small-layer measurements")
    ap.add_argument("--case", default=None,
                    help="M,N,K[,r]: small profiling case (two fwd+bwd of one projection), no JSON")
    ap.add_argument("--quant-case", type=int, default=None,
                    help="N: profiling case, quantize + dequant of N heavy-tailed values twice, no JSON")
    ap.add_argument("--merge-case", default=None,
                    help="N,K,r: profiling case, the adapter merged into W from the NF4 and the bf16 "
                         "base, twice each, no JSON")
    args = ap.parse_args()
    if args.case:
        return profile_case(*[int(v) for v in args.case.split(",")])
    if args.quant_case:
        return profile_quant_case(args.quant_case)
    if args.merge_case:
        return profile_merge_case(*[int(v) for v in args.merge_case.split(",")])
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    import bit_nf4_quantized_19_b200 as q

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    P = peaks()
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    wl = Workload(q, torch, dev, HEADLINE, rank)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        wl.run()
    torch.cuda.synchronize()
    code, flags = q.device_status()
    if code != 0:
        raise RuntimeError(f"device status {code} flags {flags} after warm-up")

    # ---- headline timed region: K steps, L2 flushed before each, CUDA events per step,
    # no library event recording inside it
    with ClockSampler(local) as clk:
        step_ms = time_steps(torch, wl.run, args.steps, flush, stream, barrier)
    med = statistics.median(step_ms)
    if world > 1:
        t = torch.tensor([med], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        med = float(t.item())
    code, flags = q.device_status()
    if code != 0:
        raise RuntimeError(f"device status {code} flags {flags} after timing")
    value = world * wl.flops / (med * 1e-3) / 1e12
    clocks = clk.summary()
    units = q.gemm_units()

    # ---- per-kernel breakdown and the dominant kernel's roofline (second pass)
    kernels, by, launches_per_step = kernel_profile(q, torch, wl.run, args.steps, flush, stream, barrier)
    roof = gemm_roofline(wl, by, args.steps, P, clocks)
    roof["step_frac_of_peak"] = wl.flops / (med * 1e-3) / 1e12 / roof["peak"]

    e2e = e2e_measure(torch, wl, max(3, min(args.steps, 10)), stream, barrier, world, dev)
    del wl
    torch.cuda.empty_cache()

    # ---- single-GPU extras at N = 1 only, so a multi-GPU run stays short and symmetric
    others, subpaths = None, None
    if world == 1 and not args.no_secondary:
        others = {"llama7b": secondary_workload(q, torch, dev, "llama7b", args.steps, args.warmup,
                                                flush, stream, P),
                  "small": small_layer(q, torch, dev, stream)}
    if not args.no_subpaths and world == 1:
        subpaths = hbm_subpaths(q, torch, dev, stream, P, flush)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N=1 only)
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tokens, wrows = CPU_SAMPLE[HEADLINE]
        fl, sec = oracle_sample(sample_problems(HEADLINE, tokens, wrows), tokens, wrows)
        cores, blas = cpu_info()
        cpu_baseline = {"value": fl / sec / 1e12, "unit": "TFLOP/s", "cores": blas or cores,
                        "kind": "oracle",
                        "sample": f"all 3 projections, first {tokens} tokens x first {wrows} "
                                  f"output features, dequant of those rows included; {sec:.1f} s"}

    if world > 1:
        dist.barrier()
    if rank == 0:
        wld = WORKLOADS[HEADLINE]
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": med,
                "ms_per_step_mean": statistics.mean(step_ms),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded): W ~ N(0,0.015) bf16 quantized to NF4, X, dY ~ N(0,1), "
                        "A ~ N(0,1/r), B ~ N(0,0.01)",
                "config": {"workload": WORKLOAD, "global_batch": wld["shapes"][0][0] * world,
                           "tokens_per_gpu": wld["shapes"][0][0], "lora_r": wld["r"],
                           "lora_alpha": wld["alpha"], "parallelism": f"dp{world}",
                           "l2": "flushed (256 MiB write) before every timed step",
                           "step_time": "median of the timed steps",
                           "flops_per_step_per_gpu": workload_flops(HEADLINE),
                           "gemm_units": {"ctas": units[0], "pairs": units[1]}},
                "roofline": roof, "cpu_baseline": cpu_baseline, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "clocks": clocks, "kernels": kernels,
                "other_workloads": others, "subpaths": subpaths}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def profile_case(M, N, K, r=16):
    """Two forward + backward passes of one projection through the public API
    (seeded device inputs); the case that the ncu captures under profiles/ use."""
    import torch
    import bit_nf4_quantized_19_b200 as q
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    W = (torch.randn(N, K, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    X = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    dY = torch.randn(M, N, generator=g, device="cuda").to(torch.bfloat16)
    A = (torch.randn(K, r, generator=g, device="cuda") / r).to(torch.bfloat16)
    B = (torch.randn(r, N, generator=g, device="cuda") * 0.01).to(torch.bfloat16)
    Wq = q.nf4_quantize(W)
    ws = q.make_workspace(M, N, K, r, X.device)
    for _ in range(2):
        Y, XA = q.linear_fwd(X, Wq, A, B, 2.0, workspace=ws)
        q.linear_bwd(dY, X, XA, Wq, A, B, 2.0, workspace=ws)
    torch.cuda.synchronize()
    code, flags = q.device_status()
    print("case", M, N, K, "status", code, flags)
    return 0 if code == 0 else 1


def heavy_tail_device(torch, dev, n, seed=0):
    """n bf16 values ~ N(0, 0.02), each scaled by 8 with probability 1e-3 (seeded, on the device)."""
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    W = torch.empty(n, dtype=torch.bfloat16, device=dev)
    chunk = 1 << 26
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        z = torch.randn(m, generator=g, device=dev, dtype=torch.float32) * 0.02
        z[torch.rand(m, generator=g, device=dev) < 1e-3] *= 8.0
        W[i:i + m] = z.to(torch.bfloat16)
    return W


def profile_quant_case(n):
    """Quantize + dequant of n heavy-tailed values, twice, through the public API;
    the case that the quantize/dequant ncu captures under profiles/ use."""
    import torch
    import bit_nf4_quantized_19_b200 as q
    W = heavy_tail_device(torch, torch.device("cuda"), n)
    out = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    Wq = q.nf4_quantize(W.view(1, n))
    for _ in range(2):
        q.nf4_quantize(W.view(1, n), out=Wq)
        q.nf4_dequant(Wq, out.view(1, n))
    torch.cuda.synchronize()
    code, flags = q.device_status()
    print("quant case", n, "status", code, flags)
    return 0 if code == 0 else 1


def profile_merge_case(N, K, r):
    """The merge of a seeded adapter into a seeded W [N, K], from the NF4 base then from
    the bf16 base, twice each, through the public API; the case that the merge ncu
    capture under profiles/ uses (launch order: nf4, nf4, bf16, bf16)."""
    import torch
    import bit_nf4_quantized_19_b200 as q
    g = torch.Generator(device="cuda")
    g.manual_seed(2)
    Wb = (torch.randn(N, K, generator=g, device="cuda") * 0.015).to(torch.bfloat16)
    Wq = q.nf4_quantize(Wb)
    A = (torch.randn(K, r, generator=g, device="cuda") / r).to(torch.bfloat16)
    B = (torch.randn(r, N, generator=g, device="cuda") * 0.01).to(torch.bfloat16)
    out = torch.empty(N, K, dtype=torch.bfloat16, device="cuda")
    for kw in ({"Wq": Wq}, {"W16": Wb}):
        for _ in range(2):
            q.nf4_merge(A, B, 0.25, out=out, **kw)
    torch.cuda.synchronize()
    code, flags = q.device_status()
    print("merge case", N, K, r, "status", code, flags)
    return 0 if code == 0 else 1


def hbm_subpaths(q, torch, dev, stream, P, flush):
    out = {}
    # 1e9-value heavy-tailed tensor, generated on the device (seeded)
    W = heavy_tail_device(torch, dev, BIG_N)
    Wq = q.nf4_quantize(W.view(1, BIG_N))
    out_bf = torch.empty(BIG_N, dtype=torch.bfloat16, device=dev)
    q.nf4_dequant(Wq, out_bf.view(1, BIG_N))
    torch.cuda.synchronize()
    nbytes = BIG_N * 2 + Wq.nbytes
    q.profile_enable(True)
    for _ in range(3):
        q.nf4_quantize(W.view(1, BIG_N), out=Wq)
        q.nf4_dequant(Wq, out_bf.view(1, BIG_N))
    prof, _ = q.profile_read()
    q.profile_enable(False)
    tq = min(ms for k, ms in prof if k == "quantize")
    td = min(ms for k, ms in prof if k == "dequant")
    out["quantize_1e9"] = {"ms": tq, "GB/s": nbytes / tq / 1e6, "frac": nbytes / tq / 1e6 / P["hbm"],
                           "bytes": nbytes}
    out["dequant_1e9"] = {"ms": td, "GB/s": nbytes / td / 1e6, "frac": nbytes / td / 1e6 / P["hbm"],
                          "bytes": nbytes}
    del W, Wq, out_bf
    torch.cuda.empty_cache()
    # merge of a trained adapter into a 16-bit weight (the serving export), from the NF4
    # base and from the bf16 original: W 22016 x 8192 (the 65B up-projection), r = 64;
    # L2 flushed before each call
    gen = torch.Generator(device=dev)
    gen.manual_seed(2)
    N, K, r = MERGE_SHAPE
    Wb = (torch.randn(N, K, generator=gen, device=dev) * 0.015).to(torch.bfloat16)
    Wq = q.nf4_quantize(Wb)
    A = (torch.randn(K, r, generator=gen, device=dev) / r).to(torch.bfloat16)
    B = (torch.randn(r, N, generator=gen, device=dev) * 0.01).to(torch.bfloat16)
    Wm = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    for base in ("nf4", "bf16"):
        kw = {"Wq": Wq} if base == "nf4" else {"W16": Wb}
        for _ in range(2):
            q.nf4_merge(A, B, 0.25, out=Wm, **kw)
        torch.cuda.synchronize()
        ts = []
        for i in range(5):
            flush.fill_(float(i))
            q.profile_enable(True)
            q.nf4_merge(A, B, 0.25, out=Wm, **kw)
            prof, _ = q.profile_read()
            q.profile_enable(False)
            ts += [ms for k, ms in prof if k == "merge"]
        t = min(ts)
        by = (Wq.nbytes if base == "nf4" else 2 * N * K) + 2 * N * K + 2 * K * r + 2 * r * N
        out[f"merge_{base}_{N}x{K}_r{r}"] = {"ms": t, "GB/s": by / t / 1e6, "frac": by / t / 1e6 / P["hbm"],
                                             "bytes": by}
    del Wb, Wq, Wm
    torch.cuda.empty_cache()
    # skinny forward: M in {1,4,16}, L2 flushed before each call, whole call timed
    gen = torch.Generator(device=dev)
    gen.manual_seed(1)
    for (M, N, K) in SKINNY:
        r = 16
        Wb = (torch.randn(N, K, generator=gen, device=dev) * 0.02).to(torch.bfloat16)
        Wq = q.nf4_quantize(Wb)
        X = torch.randn(M, K, generator=gen, device=dev).to(torch.bfloat16)
        A = (torch.randn(K, r, generator=gen, device=dev) / r).to(torch.bfloat16)
        B = (torch.randn(r, N, generator=gen, device=dev) * 0.01).to(torch.bfloat16)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        XA = torch.empty(M, r, dtype=torch.float32, device=dev)
        ws = q.make_workspace(M, N, K, r, dev)
        for _ in range(3):
            q.linear_fwd(X, Wq, A, B, 2.0, workspace=ws, Y=Y, XA=XA)
        ts = []
        for i in range(20):
            flush.fill_(float(i))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            q.linear_fwd(X, Wq, A, B, 2.0, workspace=ws, Y=Y, XA=XA)
            b.record(stream)
            ts.append((a, b))
        torch.cuda.synchronize()
        t = statistics.median(a.elapsed_time(b) for a, b in ts)
        by = Wq.nbytes + 2 * M * K + 2 * M * N + 2 * K * r + 2 * r * N + 4 * M * r
        out[f"skinny_M{M}_{N}x{K}"] = {"ms": t, "GB/s": by / t / 1e6, "frac": by / t / 1e6 / P["hbm"],
                                       "bytes": by}
        del Wb, Wq
    # skinny forward inside one CUDA graph: L distinct weights whose NF4 storage
    # together exceeds 2.5x the L2, called back to back as the consecutive layers of
    # a decode step are, so every call streams its weight from HBM
    for (N, K) in sorted({(n, k) for _, n, k in SKINNY}):
        r = 16
        Wb = (torch.randn(N, K, generator=gen, device=dev) * 0.02).to(torch.bfloat16)
        Wq0 = q.nf4_quantize(Wb)
        L = max(8, -(-GRAPH_STREAM_BYTES // Wq0.nbytes))
        Wqs = [Wq0] + [q.nf4_quantize(Wb) for _ in range(L - 1)]
        del Wb
        for M in sorted({m for m, n, k in SKINNY if (n, k) == (N, K)}):
            X = torch.randn(M, K, generator=gen, device=dev).to(torch.bfloat16)
            A = (torch.randn(K, r, generator=gen, device=dev) / r).to(torch.bfloat16)
            B = (torch.randn(r, N, generator=gen, device=dev) * 0.01).to(torch.bfloat16)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            XA = torch.empty(M, r, dtype=torch.float32, device=dev)
            ws = q.make_workspace(M, N, K, r, dev)
            for Wq in Wqs:
                q.linear_fwd(X, Wq, A, B, 2.0, workspace=ws, Y=Y, XA=XA)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for Wq in Wqs:
                    q.linear_fwd(X, Wq, A, B, 2.0, workspace=ws, Y=Y, XA=XA)
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize()
            reps = 10
            cur = torch.cuda.current_stream()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(cur)
            for _ in range(reps):
                graph.replay()
            b.record(cur)
            torch.cuda.synchronize()
            t = a.elapsed_time(b) / (reps * L)
            by = Wqs[0].nbytes + 2 * M * K + 2 * M * N + 2 * K * r + 2 * r * N + 4 * M * r
            out[f"skinny_graph_M{M}_{N}x{K}"] = {"ms": t, "GB/s": by / t / 1e6, "frac": by / t / 1e6 / P["hbm"],
                                                 "bytes": by, "layers": L}
            del graph
        del Wqs, Wq0
        torch.cuda.empty_cache()
    out["hbm_peak_GBps"] = P["hbm"]
    out["hbm_peak_source"] = P["src"]
    return out


if __name__ == "__main__":
    sys.exit(main())
