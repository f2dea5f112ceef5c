#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 frozen-base linear layer on B200.

One step = forward + backward of the three LLaMA-7B-shaped adapted projections
(W 4096x4096, 11008x4096, 4096x11008 stored as NF4 with double-quantized
constants; 4096 tokens per GPU; LoRA r=16, alpha=32): per projection
Y = X deq(W)^T + s (X A) B, then dX, dA, dB.  Weights are quantized once before
timing (model load).  Metric: fwd+bwd TFLOP/s of algorithmic FLOPs
4MNK + 6Mr(K+N) per projection.  Multi-GPU: data-parallel replicas (weak
scaling), each rank its own 4096 tokens, dA/dB all-reduced over NCCL each step.

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

METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4-weight HBM GB/s vs roofline, 1 B200"
SHAPES = [(4096, 4096, 4096), (4096, 11008, 4096), (4096, 4096, 11008)]   # (M, N, K)
RANK_R, ALPHA, W_STD = 16, 32.0, 0.02
WORKLOAD = ("LLaMA-7B-shaped projections W[N,K] in {4096x4096, 11008x4096, 4096x11008}, NF4 "
            "block 64 / double-quant 256; 4096 tokens per GPU; LoRA r=16 alpha=32; fwd+bwd")
FLUSH_BYTES = 256 << 20
SKINNY = [(m, n, 4096) for n in (4096, 11008) for m in (1, 4, 16)]
BIG_N = 1_000_000_000
GRAPH_STREAM_BYTES = 320 << 20   # weights streamed per graph replay of the decode measurement


def step_flops(M, N, K, r):
    return 4.0 * M * N * K + 6.0 * M * r * (K + N)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


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


def host_problems(seed):
    from synth import linear_problem
    out = []
    for (M, N, K) in SHAPES:
        p = linear_problem(M, N, K, RANK_R, ALPHA, W_STD, seed=0)      # frozen W: same on all ranks
        if seed:
            q = linear_problem(M, N, K, RANK_R, ALPHA, W_STD, seed=seed)
            p.X, p.dY = q.X, q.dY                                      # per-rank tokens
        out.append(dict(M=M, N=N, K=K, r=RANK_R, s=ALPHA / RANK_R, W=p.W, X=p.X, A=p.A, B=p.B,
                        dY=p.dY))
    return out


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    problems = host_problems(0)
    tokens, wrows = 128, 512
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
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-subpaths", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None,
                    help="M,N,K: small profiling case (two fwd+bwd of one projection), no JSON")
    ap.add_argument("--quant-case", type=int, default=None,
                    help="N: profiling case, quantize + dequant of N heavy-tailed values twice, no JSON")
    args = ap.parse_args()
    if args.case:
        return profile_case(*[int(v) for v in args.case.split(",")])
    if args.quant_case:
        return profile_quant_case(args.quant_case)
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

    hp = host_problems(rank)
    P = peaks()
    stream = torch.cuda.current_stream()

    # ---- device-resident state (weights quantized once, like a model load)
    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    from bit_nf4_quantized_19_b200.dp import GradBucket
    layers = []
    bucket = GradBucket([(N, K, RANK_R) for (_, N, K) in SHAPES], dev)
    flat_grads = bucket.flat
    flat_host = torch.empty(flat_grads.numel(), dtype=torch.float32).pin_memory()
    for p, (dA, dB) in zip(hp, bucket.views):
        M, N, K, r = p["M"], p["N"], p["K"], p["r"]
        Wq = q.nf4_quantize(to_dev(p["W"]))
        L = dict(M=M, N=N, K=K, r=r, s=p["s"], Wq=Wq, X=to_dev(p["X"]), dY=to_dev(p["dY"]),
                 A=to_dev(p["A"]), B=to_dev(p["B"]),
                 Y=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                 XA=torch.empty(M, r, dtype=torch.float32, device=dev),
                 dX=torch.empty(M, K, dtype=torch.bfloat16, device=dev),
                 dA=dA, dB=dB, ws=q.make_workspace(M, N, K, r, dev))
        L["hX"] = torch.from_numpy(np.ascontiguousarray(p["X"]).view(np.int16)).view(torch.bfloat16).pin_memory()
        L["hdY"] = torch.from_numpy(np.ascontiguousarray(p["dY"]).view(np.int16)).view(torch.bfloat16).pin_memory()
        layers.append(L)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()

    def step():
        for L in layers:
            q.linear_fwd(L["X"], L["Wq"], L["A"], L["B"], L["s"], workspace=L["ws"], Y=L["Y"],
                         XA=L["XA"])
            q.linear_bwd(L["dY"], L["X"], L["XA"], L["Wq"], L["A"], L["B"], L["s"],
                         workspace=L["ws"], dX=L["dX"], dA=L["dA"], dB=L["dB"])
        bucket.allreduce_()       # the one exchange of data-parallel adapter training

    flops_per_step_rank = sum(step_flops(M, N, K, RANK_R) for (M, N, K) in SHAPES)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    code, flags = q.device_status()
    if code != 0:
        raise RuntimeError(f"device status {code} flags {flags} after warm-up")

    # ---- timed region: K steps, L2 flushed before each, CUDA events per step
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    q.profile_enable(True)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
    prof, nlaunch = q.profile_read()
    q.profile_enable(False)
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = sum(step_ms)
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    code, flags = q.device_status()
    if code != 0:
        raise RuntimeError(f"device status {code} flags {flags} after timing")
    value = world * flops_per_step_rank * args.steps / (total_ms * 1e-3) / 1e12

    # ---- per-kernel breakdown and the dominant kernel's roofline
    by = {}
    for kind, ms in prof:
        d = by.setdefault(kind, [0, 0.0])
        d[0] += 1
        d[1] += ms
    kern_total = sum(v[1] for v in by.values()) or 1.0
    kernels = {k: {"launches": v[0], "ms_total": round(v[1], 4), "share": round(v[1] / kern_total, 4)}
               for k, v in sorted(by.items(), key=lambda kv: -kv[1][1])}
    gemm_flops = args.steps * sum(2.0 * M * N * K + 2.0 * M * N * RANK_R + 2.0 * M * N * K
                                  + 2.0 * M * K * RANK_R for (M, N, K) in SHAPES)
    gemm_ms = by.get("gemm_fwd", [0, 0.0])[1] + by.get("gemm_dx", [0, 0.0])[1]
    gemm_launches = by.get("gemm_fwd", [0, 0.0])[0] + by.get("gemm_dx", [0, 0.0])[0]
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None
    roof = {"kernel": "qlora_gemm_kernel (fused NF4 dequant + tcgen05 GEMM + LoRA K-steps; fwd and dX)",
            "bound": "tensor", "achieved": achieved, "peak": P["bf16_sus"], "unit": "TFLOP/s",
            "frac": (achieved / P["bf16_sus"]) if achieved else None,
            "peak_source": f"{P['src']} bf16 sustained (MEASURED_PEAKS.json)",
            "avg_launch_ms": gemm_ms / max(1, gemm_launches),
            "traffic": traffic_for("qlora_gemm_kernel")}

    # ---- end to end through the public API: pinned host inputs -> device -> grads back.
    # As a data loader would, the next step's inputs are uploaded (on their own stream,
    # into the other of two device buffers) while the current step computes; every
    # upload and every read-back of the gradients lies inside the timed region.
    e2e_steps = max(3, min(args.steps, 30))
    h2d = sum(L["hX"].numel() * 2 + L["hdY"].numel() * 2 for L in layers)
    d2h = flat_host.numel() * 4
    xfer = torch.cuda.Stream(device=dev)
    bufs = [[(L["X"], L["dY"]) for L in layers],
            [(torch.empty_like(L["X"]), torch.empty_like(L["dY"])) for L in layers]]
    uploaded = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]

    def upload(b):
        xfer.wait_event(consumed[b])          # the step that last read buffer b is done
        with torch.cuda.stream(xfer):
            for (X, dY), L in zip(bufs[b], layers):
                X.copy_(L["hX"], non_blocking=True)
                dY.copy_(L["hdY"], non_blocking=True)
        uploaded[b].record(xfer)

    def step_on(b):
        stream.wait_event(uploaded[b])
        for (X, dY), L in zip(bufs[b], layers):
            q.linear_fwd(X, L["Wq"], L["A"], L["B"], L["s"], workspace=L["ws"], Y=L["Y"], XA=L["XA"])
            q.linear_bwd(dY, X, L["XA"], L["Wq"], L["A"], L["B"], L["s"],
                         workspace=L["ws"], dX=L["dX"], dA=L["dA"], dB=L["dB"])
        bucket.allreduce_()
        consumed[b].record(stream)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    xfer.wait_event(e0)
    upload(0)
    for i in range(e2e_steps):
        if i + 1 < e2e_steps:
            upload((i + 1) % 2)
        step_on(i % 2)
        flat_host.copy_(flat_grads, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e = {"value": world * flops_per_step_rank * e2e_steps / (e2e_ms * 1e-3) / 1e12,
           "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "steps": e2e_steps, "uploads": "next step's inputs overlap the current step (two buffers)"}

    # ---- HBM-bound subpaths (quantize / dequant of 1e9 values, skinny forward): single-GPU
    # measurements, taken at N = 1 only so a multi-GPU run stays short and symmetric
    subpaths = None
    if not args.no_subpaths and world == 1:
        subpaths = hbm_subpaths(q, torch, dev, stream, P, flush)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N=1 only)
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        hp0 = host_problems(0)
        tokens, wrows = 512, 2048
        fl, sec = oracle_sample(hp0, tokens, wrows)
        cores, blas = cpu_info()
        cpu_baseline = {"value": fl / sec / 1e12, "unit": "TFLOP/s", "cores": blas or cores,
                        "kind": "oracle",
                        "sample": f"all 3 projections, first {tokens} tokens x first {wrows} "
                                  f"output features, dequant of those rows included; {sec:.1f} s"}

    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded): W ~ N(0,0.02) bf16 quantized to NF4, X, dY ~ N(0,1), "
                        "A ~ N(0,1/r), B ~ N(0,0.01)",
                "config": {"workload": WORKLOAD, "global_batch": 4096 * world,
                           "tokens_per_gpu": 4096, "parallelism": f"dp{world}",
                           "l2": "flushed (256 MiB write) before every timed step",
                           "flops_per_step_per_gpu": flops_per_step_rank},
                "roofline": roof, "cpu_baseline": cpu_baseline, "e2e": e2e,
                "gpu_launches": nlaunch, "clocks": clk.summary(), "kernels": kernels,
                "subpaths": subpaths}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def profile_case(M, N, K, r=RANK_R):
    """Two forward + backward passes of one projection through the public API
    (seeded device inputs); the case that the ncu captures under profiles/ use."""
    import torch
    import bit_nf4_quantized_19_b200 as q
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    W = (torch.randn(N, K, generator=g, device="cuda") * W_STD).to(torch.bfloat16)
    X = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    dY = torch.randn(M, N, generator=g, device="cuda").to(torch.bfloat16)
    A = (torch.randn(K, r, generator=g, device="cuda") / r).to(torch.bfloat16)
    B = (torch.randn(r, N, generator=g, device="cuda") * 0.01).to(torch.bfloat16)
    Wq = q.nf4_quantize(W)
    ws = q.make_workspace(M, N, K, r, X.device)
    for _ in range(2):
        Y, XA = q.linear_fwd(X, Wq, A, B, ALPHA / r, workspace=ws)
        q.linear_bwd(dY, X, XA, Wq, A, B, ALPHA / r, workspace=ws)
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
    # skinny forward: M in {1,4,16}, L2 flushed before each call, whole call timed
    gen = torch.Generator(device=dev)
    gen.manual_seed(1)
    for (M, N, K) in SKINNY:
        r = RANK_R
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
        r = RANK_R
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
