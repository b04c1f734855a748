#!/usr/bin/env python
"""Benchmark of the TTQ linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one TTQ linear forward through the C ABI -- activation statistic
with the scaled binary16 X, quantise-and-pack with the dequantised binary16
weight, tensor-core GEMM -- on one batch of seeded
synthetic input: the Llama-7B-like q_proj prefill, d = d' = 4096, T = 2048
tokens, INT4 with groups of 128, p = 2, lambda = 1e-3, alpha = 0.5.

Metric: tokens/s of the layer (whole job over all ranks; each rank runs its
own independent problem, so scaling is weak and there is no collective on the
data path).  Timing: exactly K steps after W warm-up steps, captured once
as a CUDA graph whose replay is bracketed by CUDA events on the launching
stream, barrier + synchronize on both sides, max over ranks.  The inputs rotate over enough (X, W) sets that each step's operands
exceed the 126 MB L2, so no step reads its inputs from a warm L2.

Extra keys: roofline of the dominant kernel (live CUDA-event timing of each
kernel over the same K steps), the CPU oracle as a baseline (rank 0, N = 1),
an end-to-end figure with host buffers and host<->device copies inside the
timed region, clocks sampled during the run, and the number of our kernel
launches in the timed region.

--impl reference times the CPU oracle (the method written as plain loops) on
a bounded sample of the same workload; under torchrun only rank 0 runs it.
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

WORKLOAD = dict(name="q_proj_prefill_4096", d=4096, dp=4096, T=2048, bits=4, group=128, r=0,
                p=2.0, lam=1e-3, alpha=0.5)
METRIC = "TTQ linear tokens/s @4096^2, T=2048 (INT4 g128)"
L2_BYTES = 126 * 2 ** 20

# DRAM bytes per launch of the dominant kernel from one ncu capture, keyed by
# the hash of the kernel source it was taken on (stale entries read as null).
NCU_TRAFFIC = {
    # ttq_gemm_kernel<0, 256, 0> on the binary16 dequantised weight:
    # dram__bytes_read.sum + dram__bytes_write.sum of one launch (ncu flushes
    # L2 before it, so the W_hat and X D^-1/2 the previous kernels left in L2
    # are read from DRAM here)
    "2186cde2763e9e93": 52763136,
}


def _host_cpu() -> dict:
    """The host the CPU oracle ran on: its logical core count and CPU model."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def _rank_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def _measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def _kernel_hash():
    h = hashlib.sha256()
    for name in ("gemm_tc.cu", "ttq_device.cuh"):
        with open(os.path.join(ROOT, "test_weight_quantization_ttq_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clocks/throttle sampling in the background."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = []
        for line in self.file.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "util": float(parts[4]),
                             "hw": parts[6], "hwt": parts[7], "swt": parts[8], "pc": parts[9]})
            except ValueError:
                continue
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        busy = [r for r in rows if r["util"] >= 50] or rows
        reasons = set()
        for r in busy:
            if r["hw"] == "Active":
                reasons.add("hw_slowdown")
            if r["hwt"] == "Active":
                reasons.add("hw_thermal_slowdown")
            if r["swt"] == "Active":
                reasons.add("sw_thermal_slowdown")
            if r["pc"] == "Active":
                reasons.add("sw_power_cap")
        return {"sm_mhz": statistics.median(r["sm"] for r in busy), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(busy)}


# ----------------------------------------------------------------- oracle
def _oracle_sample(data, rows_sample: int):
    """Times the oracle on one bounded sample of the workload: the statistic
    and the quantiser in full, the projection for `rows_sample` output rows.
    Returns (seconds extrapolated to the whole layer, seconds spent)."""
    import numpy as np

    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import ttq_oracle

    from test_weight_quantization_ttq_b200 import synth

    O = ttq_oracle.get()
    w = WORKLOAD
    X = data["X"].astype(np.float64)
    t0 = time.perf_counter()
    D, Dr, _ = O.act_norm(X, w["p"], w["lam"], w["alpha"])
    codes, sc, ze, _ = O.quantize(data["W"], D.astype(np.float32), w["bits"], w["group"])
    t1 = time.perf_counter()
    rows = synth.sample_rows(w["dp"], rows_sample, seed=int(t0 * 1000) % 100000)
    What = O.dequant_rows(codes, sc, ze, Dr, w["d"], w["bits"], w["group"], rows)
    O.project(What, X)
    t2 = time.perf_counter()
    est = (t1 - t0) + (t2 - t1) * (w["dp"] / len(rows))
    return est, t2 - t0


def run_reference(args):
    rank, world, _ = _rank_env()
    if rank != 0:
        return
    from test_weight_quantization_ttq_b200 import synth

    spec = synth.C2
    data = synth.generate(spec)
    rows_sample = 64
    for _ in range(args.warmup):
        _oracle_sample(data, rows_sample)
    ests = []
    spent = 0.0
    for _ in range(args.steps):
        est, s = _oracle_sample(data, rows_sample)
        ests.append(est)
        spent += s
    t_step = sum(ests) / len(ests)
    value = WORKLOAD["T"] / t_step
    sample = (f"per step: statistic and quantiser over the full layer, projection for {rows_sample} of "
              f"{WORKLOAD['dp']} output rows, extrapolated linearly in d'")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample,
                         "host": _host_cpu(),
                         "cpu_seconds": spent},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


SCHEMES = {"asym": None, "sym": "symmetric INT", "fp8": "FP8 E4M3"}


def _config(scheme: str = "asym"):
    w = WORKLOAD
    code = f"INT{w['bits']}" if scheme == "asym" else (f"symmetric INT{w['bits']}" if scheme == "sym" else "FP8 E4M3")
    cfg = {"workload": f"{w['name']}: TTQ linear, d=d'={w['d']}, T={w['T']}, {code} g{w['group']}, "
                       f"p={w['p']}, lambda={w['lam']}, alpha={w['alpha']}, bf16 X/W/Y",
           "d": w["d"], "d_out": w["dp"], "tokens": w["T"], "bits": w["bits"] if scheme != "fp8" else 8,
           "group": w["group"],
           "l2": "inputs rotate over sets whose size exceeds L2 (no warm-L2 reads of X or W)",
           "timing": "the K steps captured in one CUDA graph; CUDA events around its replay"}
    if scheme != "asym":
        cfg["scheme"] = SCHEMES[scheme]
    return cfg


def _metric(scheme: str = "asym") -> str:
    if scheme == "asym":
        return METRIC
    return METRIC.replace("(INT4", "(symmetric INT4" if scheme == "sym" else "(FP8 E4M3")


# ------------------------------------------------------- multi-rank helpers
def _max_over_ranks(v: float, world: int, device: str) -> float:
    """The largest of the ranks' values (every rank gets it); a time taken
    on each rank's device becomes the job's time."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _job_throughput(world: int, steps: int, tokens: int, ms: float) -> float:
    """Tokens per second of the whole job: every rank runs `steps` forwards
    of `tokens` tokens on its own problem within the max-over-ranks time."""
    return world * steps * tokens / (ms / 1e3)


# ------------------------------------------------------------------- ours
def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from test_weight_quantization_ttq_b200 import synth, ttq

    rank, world, local = _rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return _max_over_ranks(v, world, "cuda")

    w = WORKLOAD
    spec = synth.C2
    d, dp, T, bits, group = w["d"], w["dp"], w["T"], w["bits"], w["group"]
    scheme = {"asym": None, "sym": ttq.TTQ_QSCHEME_SYMMETRIC, "fp8": ttq.TTQ_QSCHEME_FP8_E4M3}[args.scheme]
    if args.scheme == "fp8":
        bits = 8
    set_bytes = 2 * (d * dp + T * d + T * dp)
    nsets = max(2, -(-2 * L2_BYTES // set_bytes))
    # each rotating set is its own seeded draw of the workload: each step
    # reads cold memory, and a step that read another set's buffers would
    # give another result
    sets = [synth.generate(spec.with_(seed=rank * nsets + k)) for k in range(nsets)]
    data = sets[0]
    Xs, Ws, Ys = [], [], []
    for k in range(nsets):
        Xs.append(torch.from_numpy(sets[k]["X"]).to(torch.bfloat16).cuda())
        Ws.append(torch.from_numpy(sets[k]["W"]).to(torch.bfloat16).cuda())
        Ys.append(torch.empty((T, dp), dtype=torch.bfloat16, device="cuda"))
    del sets
    ws = ttq.new_workspace(d, dp, T, 0, bits, group)
    stream = torch.cuda.current_stream()

    def step(i):
        k = i % nsets
        ttq.ttq_linear_forward(Xs[k], Ws[k], None, None, w["p"], w["lam"], w["alpha"], bits, group,
                               ws=ws, Y=Ys[k], scheme=scheme)

    sampler = ClockSampler(local)
    sampler.start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    # the K timed steps are captured once in a CUDA graph and the graph is
    # replayed: a forward is a few tens of microseconds, about what the host
    # takes to launch its kernels, so launching them one by one would time
    # the host
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(args.steps):
            step(i)
    graph.replay()
    torch.cuda.synchronize()
    # keep the GPU busy for ~1.5 s so the clock samples describe a loaded GPU
    t_end = time.time() + (0.0 if args.profile else 1.5)
    while time.time() < t_end:
        graph.replay()
        torch.cuda.synchronize()

    # ---- value: exactly K forward steps (one replay of the K-step graph)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1))
    del graph
    clocks = sampler.stop()
    st, flags = ttq.ttq_get_status(ws)
    if st != ttq.TTQ_OK:
        raise RuntimeError(f"device status {ttq.status_string(st)} (flags {flags:#x})")
    value = _job_throughput(world, args.steps, T, ms)

    # ---- per-kernel durations over K steps: the forward's kernels, one entry
    # point each (statistic fused with X D^{-1/2} in binary16, quantiser with
    # the dequantised binary16 weight, product on it)
    n_kernels = ttq.ttq_linear_forward_kernels(d, dp, T, 0, w["p"], ttq.TTQ_BF16, bits, group,
                                               scheme if scheme is not None else ttq.TTQ_QSCHEME_ASYMMETRIC)
    views = ttq.workspace_views(ws, d, dp, T, 0, bits, group)
    Dbuf = views["D"]  # written in place by ttq_act_norm_scale (copy_out=False)
    Xsbuf = torch.empty((T, d), dtype=torch.float16, device="cuda")
    W_hat = torch.empty((dp, d), dtype=torch.float16, device="cuda")
    def stat(i):
        ttq.ttq_act_norm_scale(Xs[i % nsets], w["p"], w["lam"], w["alpha"], ws=ws, Xs=Xsbuf, copy_out=False)

    def quant(i):
        # as in the forward, the materialised weight alone (no codes)
        if scheme is None:
            ttq.ttq_quantize_dequant_weight(Ws[i % nsets], Dbuf, bits, group, ws=ws, W_hat=W_hat,
                                            with_codes=False)
        else:
            ttq.ttq_quantize_weight_ex(Ws[i % nsets], Dbuf, bits, group, scheme, ws=ws, W_hat=W_hat,
                                       with_codes=False)

    def gemm(i):
        ttq.ttq_dequantized_gemm(W_hat, Xsbuf, ws=ws, Y=Ys[i % nsets])

    def per_call(fn):
        """K calls of one entry point captured in a CUDA graph (inputs
        rotating over the sets, as in the forward); the replay is timed with
        CUDA events on the launching stream: the average launch duration."""
        fn(0)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(args.steps):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / 1e3 / args.steps

    barrier()
    torch.cuda.synchronize()
    t_stat = per_call(stat)
    t_qdq = per_call(quant)
    t_gemm = per_call(gemm)

    peaks = _measured_peaks()
    flops = 2.0 * dp * d * T
    hbm = peaks["hbm_gbs"]
    # algorithmic bytes of each step (what the method must move): the
    # statistic reads X and writes D, D^{-1/2}; the quantiser reads W and D
    # and writes codes, scales and zeros
    stat_alg = 2.0 * d * T + 8.0 * d
    qdq_alg = 2.0 * dp * d + dp * d * bits / 8 + 4.0 * dp * d / group + 4.0 * d
    # bytes this implementation moves: the statistic also writes the
    # product's binary16 X D^{-1/2}; the quantiser reads W and D and writes
    # the binary16 dequantised weight that the prefill product reads, in
    # place of the codes, scales and zeros
    stat_moved = stat_alg + 2.0 * d * T
    qdq_moved = 2.0 * dp * d + 2.0 * dp * d + 4.0 * d
    gemm_tflops = flops / t_gemm / 1e12
    traffic = NCU_TRAFFIC.get(_kernel_hash())
    roofline = {"kernel": "ttq_gemm_kernel<0, 256> (tcgen05 GEMM on the binary16 dequantised weight)", "bound": "tensor",
                "achieved": gemm_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": gemm_tflops / peaks["bf16_tflops"], "traffic": traffic,
                "peak_source": f"{peaks['source']} bf16 burst (cuBLAS 8192^3)",
                "algorithmic_flops_per_launch": flops}

    def hbm_entry(name, t, alg, moved):
        return {"kernel": name, "ms": t * 1e3, "bound": "hbm", "bytes": alg,
                "achieved_gbs": alg / t / 1e9, "frac": alg / t / 1e9 / hbm,
                "bytes_moved": moved, "moved_gbs": moved / t / 1e9, "frac_of_moved": moved / t / 1e9 / hbm}

    kernels = [
        hbm_entry("act_norm_scale_kernel", t_stat, stat_alg, stat_moved),
        hbm_entry("qdq_fp8_kernel" if args.scheme == "fp8" else "qdq_stage_kernel", t_qdq, qdq_alg, qdq_moved),
        {"kernel": "ttq_gemm_kernel", "ms": t_gemm * 1e3, "bound": "tensor", "flops": flops,
         "achieved_tflops": gemm_tflops, "frac": gemm_tflops / peaks["bf16_tflops"]},
    ]
    # the paper's relative cost of the test-time steps against the product
    # (gist.science/zh/paper/2603.19296, section 2.3) and the blog's per-step
    # overhead Delta / T (blog.lo0.es, "Test-time quantization", section "The
    # overhead: the cost of measuring at every step"): Delta = statistic +
    # quantiser, T = the whole forward
    rho = {"measured": (t_stat + t_qdq) / t_gemm, "closed_form": 1.0 / dp + 3.0 / T,
           "delta_over_forward": (t_stat + t_qdq) / (ms / args.steps / 1e3)}

    if args.profile:
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"metric": _metric(args.scheme), "value": value, "unit": "tokens/s", "profile_run": True,
                              "roofline": roofline, "kernels": kernels}), flush=True)
        return

    # ---- end to end: pinned host X in, host Y out, inside the timed region;
    # step i copies in set i's X and multiplies by set i's W
    Xh = [Xs[k].cpu().pin_memory() for k in range(nsets)]
    Yh = torch.empty((T, dp), dtype=torch.bfloat16).pin_memory()

    def fwd_on(Xd, k, Yd, s=None):
        ttq.ttq_linear_forward(Xd, Ws[k % nsets], None, None, w["p"], w["lam"], w["alpha"], bits, group, ws=ws,
                               Y=Yd, scheme=scheme, stream=s)

    def e2e_serial():
        """One stream: copy in, forward, copy out, step after step."""
        Xd = torch.empty_like(Xs[0])
        for i in range(2):
            Xd.copy_(Xh[i % nsets], non_blocking=True)
            fwd_on(Xd, i, Ys[0])
            Yh.copy_(Ys[0], non_blocking=True)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(args.steps):
            Xd.copy_(Xh[i % nsets], non_blocking=True)
            fwd_on(Xd, i, Ys[0])
            Yh.copy_(Ys[0], non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize()
        return f0.elapsed_time(f1)

    def pipeline():
        """Three streams (copy in, forward, copy out) over two device buffers
        of X and Y: step i's copies overlap the forwards of steps i - 1 and
        i + 1.  Each step still copies its own X in and its own Y out."""
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        Xd = [torch.empty_like(Xs[0]) for _ in range(2)]
        Yd = [torch.empty((T, dp), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        in_done = [torch.cuda.Event() for _ in range(2)]
        cmp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]

        def step(i):
            b = i % 2
            if i >= 2:
                s_in.wait_event(cmp_done[b])      # the forward of step i - 2 has read Xd[b]
            with torch.cuda.stream(s_in):
                Xd[b].copy_(Xh[i % nsets], non_blocking=True)
                in_done[b].record(s_in)
            s_cmp.wait_event(in_done[b])
            if i >= 2:
                s_cmp.wait_event(out_done[b])     # step i - 2's Y has left Yd[b]
            fwd_on(Xd[b], i, Yd[b], s_cmp)
            cmp_done[b].record(s_cmp)
            s_out.wait_event(cmp_done[b])
            with torch.cuda.stream(s_out):
                Yh.copy_(Yd[b], non_blocking=True)
                out_done[b].record(s_out)

        return step, (s_in, s_cmp, s_out)

    def e2e_pipelined():
        """The pipelined steps enqueued one by one from the host."""
        step, (s_in, s_cmp, s_out) = pipeline()
        torch.cuda.synchronize()
        for i in range(4):
            step(i)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s_in)
        s_cmp.wait_stream(s_in)
        s_out.wait_stream(s_in)
        h0 = time.perf_counter()
        for i in range(args.steps):
            step(i)
        f1.record(s_out)
        host_s[0] = time.perf_counter() - h0   # the host's time to enqueue the steps
        torch.cuda.synchronize()
        return f0.elapsed_time(f1)

    def copy_floor():
        """The same bytes with no forward: each step's X copied in on one
        stream and a Y copied out on another, both from and to pinned host
        memory, for K steps.  The per-step time the end-to-end form cannot
        beat on this host link."""
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        Xd, Yd = torch.empty_like(Xs[0]), torch.empty((T, dp), dtype=torch.bfloat16, device="cuda")

        def run(n):
            with torch.cuda.stream(s_in):
                for i in range(n):
                    Xd.copy_(Xh[i % nsets], non_blocking=True)
            with torch.cuda.stream(s_out):
                for i in range(n):
                    Yh.copy_(Yd, non_blocking=True)

        run(4)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        run(args.steps)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
        f1.record(stream)
        torch.cuda.synchronize()
        return f0.elapsed_time(f1)

    barrier()
    torch.cuda.synchronize()
    host_s = [None]
    eager_mode = "pipelined: copy-in, forward and copy-out streams over two device buffers of X and Y"
    try:
        eager_local = e2e_pipelined()
    except Exception as exc:  # keep the bench line: time the one-stream form instead
        torch.cuda.synchronize()
        eager_mode = f"serial, one stream (pipelined form failed: {type(exc).__name__}: {exc})"[:300]
        eager_local = e2e_serial()
    # the last step's Y, read back, equals a forward of that step's own set
    last = (args.steps - 1) % nsets
    Yref = torch.empty((T, dp), dtype=torch.bfloat16, device="cuda")
    fwd_on(Xs[last], last, Yref)
    e2e_check = bool(torch.equal(Yh, Yref.cpu()))
    floor_local = copy_floor()
    barrier()
    e2e_ms = max_over_ranks(eager_local)
    floor_ms = max_over_ranks(floor_local)
    e2e_value = _job_throughput(world, args.steps, T, e2e_ms)
    floor_value = _job_throughput(world, args.steps, T, floor_ms)
    e2e = {"value": e2e_value, "unit": "tokens/s",
           "h2d_bytes_per_step": int(Xh[0].numel() * 2), "d2h_bytes_per_step": int(Yh.numel() * 2),
           "mode": eager_mode, "result_check": e2e_check,
           "host_enqueue_us_per_step": None if host_s[0] is None else host_s[0] / args.steps * 1e6,
           "copy_floor": {"value": floor_value, "unit": "tokens/s", "us_per_step": floor_ms / args.steps * 1e3,
                          "what": "the same copies in and out with no forward (pinned host memory, two streams)"},
           "frac_of_copy_floor": e2e_value / floor_value}

    # ---- the other regimes the layer serves, measured in the same run (one
    # GPU): decode at 1 and 16 tokens (HBM-bound, the test-time steps
    # dominate) and the 70B-like MLP shape at 1 and 4096 tokens
    extra = {}
    if world == 1 and not args.no_extra:
        for t in (1, 16):
            try:
                extra[f"decode_T{t}"] = _decode_point(t, 50, 5, peaks)
            except Exception as exc:
                torch.cuda.synchronize()
                extra[f"decode_T{t}"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        cache = _WeightCache()
        for t in (1, 4096):
            try:
                extra[f"mlp70b_T{t}"] = _time_forward(synth.C5.with_(T=t, p=2.0, alpha=0.5), 50, 5, cache, peaks)
            except Exception as exc:
                torch.cuda.synchronize()
                extra[f"mlp70b_T{t}"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        cache.drop(torch)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows_sample = 512
        est, spent = _oracle_sample(data, rows_sample)
        cpu = {"value": T / est, "unit": "tokens/s", "cores": 1, "kind": "oracle", "host": _host_cpu(),
               "sample": f"statistic and quantiser over the full layer, projection for {rows_sample} of {dp} "
                         f"output rows, extrapolated linearly in d' ({spent:.1f} s of CPU work)"}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": _metric(args.scheme), "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": _config(args.scheme),
        "roofline": roofline, "kernels": kernels,
        "kernels_timing": "each entry point's K calls captured in one CUDA graph; CUDA events around its replay",
        "rho": rho, "cpu_baseline": cpu, "e2e": e2e,
        "clocks": clocks, "gpu_launches": n_kernels * args.steps,
    }
    line.update(extra)
    print(json.dumps(line), flush=True)


def _decode_point(T, steps, warmup, peaks):
    """The decode workload (d = 4096, d' = 14336, INT4 g128) at T <= 16
    tokens: K forwards (statistic, then the single-pass product that reads
    W once), then K calls of each of its two entry points, and for
    comparison the two-pass form (quantiser writing codes, then the product
    reading them).  A few-token step is shorter than its host-side launch
    cost, so each batch of K calls is captured once in a CUDA graph and the
    graph replay is timed.  W rotates over enough copies that every step
    reads it from HBM.  Returns one dict."""
    import torch

    from test_weight_quantization_ttq_b200 import synth, ttq

    spec = synth.C4.with_(T=T)
    d, dp, bits, group = spec.d, spec.dp, spec.bits, spec.group
    data = synth.generate(spec)
    X = torch.from_numpy(data["X"]).to(torch.bfloat16).cuda()
    W0 = torch.from_numpy(data["W"]).to(torch.bfloat16)
    nsets = max(2, -(-2 * L2_BYTES // (2 * d * dp)))
    Ws = [W0.cuda() for _ in range(nsets)]
    Y = torch.empty((T, dp), dtype=torch.bfloat16, device="cuda")
    ws = ttq.new_workspace(d, dp, T, 0, bits, group)
    views = ttq.workspace_views(ws, d, dp, T, 0, bits, group)
    Dbuf = views["D"]
    Xsbuf = torch.empty((T, d), dtype=torch.float16, device="cuda")
    # the two-pass form's quantiser writes, and its product reads, one of ncs
    # code sets in turn (more than L2 together)
    ncs = max(2, -(-2 * L2_BYTES // (dp * d * bits // 8)))
    codes = [torch.empty((dp, d * bits // 32), dtype=torch.int32, device="cuda") for _ in range(ncs)]
    sc = [torch.empty((dp, d // group), dtype=torch.int16, device="cuda") for _ in range(ncs)]
    ze = [torch.empty((dp, d // group), dtype=torch.int16, device="cuda") for _ in range(ncs)]
    stream = torch.cuda.current_stream()

    def fwd(i):
        ttq.ttq_linear_forward(X, Ws[i % nsets], None, None, spec.p, spec.lam, spec.alpha, bits,
                               group, ws=ws, Y=Y)

    def stat(i):
        ttq.ttq_act_norm_scale(X, spec.p, spec.lam, spec.alpha, ws=ws, Xs=Xsbuf, copy_out=False)

    def one_pass(i):
        ttq.ttq_quantize_gemm(Ws[i % nsets], Dbuf, Xsbuf, None, None, None, bits, group, ws=ws, Y=Y)

    def qdq(i):
        k = i % ncs
        ttq.ttq_quantize_weight(Ws[i % nsets], Dbuf, bits, group, codes=codes[k], scales=sc[k],
                                zeros=ze[k])

    def prod(i):
        k = i % ncs
        ttq.ttq_dequant_gemm(codes[k], sc[k], ze[k], None, Xsbuf, None, None, bits, group, Y=Y)

    def graph_of(fn):
        for i in range(warmup):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        return g

    def time_graph(g):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3   # seconds for K calls

    stat(0)
    for k in range(ncs):   # every code set holds real codes before the product is timed
        qdq(k)
    g_fwd = graph_of(fwd)
    t_fwd = time_graph(g_fwd)
    st, flags = ttq.ttq_get_status(ws)
    if st != ttq.TTQ_OK:
        raise RuntimeError(f"device status {ttq.status_string(st)} (flags {flags:#x})")
    t = [time_graph(graph_of(fn)) / steps for fn in (stat, one_pass, qdq, prod)]
    hbm = peaks["hbm_gbs"]
    code_bytes = dp * d * bits / 8 + 4.0 * dp * d / group
    stat_bytes = 2.0 * T * d + 8.0 * d
    # the single pass reads W, X D^(-1/2) and sqrt(D) and writes Y
    one_bytes = 2.0 * dp * d + 2.0 * T * d + 4.0 * d + 2.0 * T * dp
    qdq_bytes = 2.0 * dp * d + code_bytes + 4.0 * d
    prod_bytes = code_bytes + 2.0 * T * d + 2.0 * T * dp
    t_fwd_step = t_fwd / steps
    # the forward's floor: W read once at HBM bandwidth (a layer that looks at
    # every weight at every step can do no better)
    read_once = 2.0 * dp * d + 2.0 * T * d + 2.0 * T * dp

    def entry(name, tt, nbytes):
        return {"kernel": name, "us": tt * 1e6, "bytes": nbytes, "achieved_gbs": nbytes / tt / 1e9,
                "frac": nbytes / tt / 1e9 / hbm}

    kernels = [
        entry("act_norm_scale_kernel", t[0], stat_bytes),
        entry("ttq_fused_decode_kernel (ttq_quantize_gemm: + a sqrt(D) pass of 8d bytes)", t[1], one_bytes),
    ]
    two_pass = [entry("qdq_pack_kernel", t[2], qdq_bytes), entry("ttq_decode_kernel", t[3], prod_bytes)]
    return {"workload": f"decode_4096x14336_T{T}", "d": d, "dp": dp, "T": T, "bits": bits, "group": group,
            "us": t_fwd_step * 1e6, "tokens_per_s": T / t_fwd_step,
            "read_once_floor_us": read_once / (hbm * 1e9) * 1e6,
            "frac_of_read_once_floor": read_once / (hbm * 1e9) / t_fwd_step,
            "kernels_per_call": ttq.ttq_linear_forward_kernels(d, dp, T, 0, spec.p, ttq.TTQ_BF16, bits, group),
            "l2": f"W rotates over {nsets} copies and the codes over {ncs} sets (each more than L2)",
            "timing": "CUDA graph of K calls, CUDA events around its replay",
            "kernels": kernels, "two_pass_for_comparison": two_pass}


def run_decode(args):
    """--decode T: the decode workload alone, one JSON line (see
    _decode_point), with the clocks sampled while it runs."""
    T = int(args.decode)
    if not 1 <= T <= 16:
        raise SystemExit("--decode takes 1..16 tokens")
    peaks = _measured_peaks()
    sampler = ClockSampler(0)
    sampler.start()
    row = _decode_point(T, args.steps, args.warmup, peaks)
    clocks = sampler.stop()
    print(json.dumps({"metric": "TTQ linear decode tokens/s", "value": row["tokens_per_s"], "unit": "tokens/s",
                      "ms_per_step": row["us"] / 1e3, "steps": args.steps, "warmup": args.warmup,
                      "dtype": "bf16", "data": "synthetic", "config": {k: row[k] for k in
                      ("workload", "d", "dp", "T", "bits", "group", "l2", "timing")},
                      "read_once_floor_us": row["read_once_floor_us"],
                      "frac_of_read_once_floor": row["frac_of_read_once_floor"],
                      "kernels": row["kernels"], "hbm_peak_gbs": peaks["hbm_gbs"], "clocks": clocks}),
          flush=True)


def _floor_us(spec, hbm, tc):
    """Lower bound on one forward (microseconds) from the method's
    algorithmic bytes and flops at the measured peaks: the statistic and
    quantiser at HBM bandwidth, the product at the slower of its bytes and
    its flops.  The bytes are what the method must move (X in, the scaled X,
    W in, codes and scales out and back in, Y out); the binary16 W_hat this
    implementation adds for long inputs is not part of the floor."""
    d, dp, T, b, g, r = spec.d, spec.dp, spec.T, spec.bits, spec.group, spec.r
    e = 4 if spec.dtype == "f32" else 2
    stat = e * d * T + 2 * d * T + 8 * d                       # X in, X D^-1/2 out, D and D^-1/2
    codes = dp * d * b / 8 + 4 * dp * d / g
    qdq = e * dp * d + codes + 4 * d
    prod = codes + 2 * d * T + e * T * dp + (2 * r * (d + dp) + 2 * r * T if r else 0)
    flops = 2.0 * dp * d * T + 2.0 * r * (d + dp) * T
    return 1e6 * ((stat + qdq) / hbm + max(prod / hbm, flops / tc)), stat + qdq + prod, flops


class _WeightCache:
    """The weight copies of one workload recipe on the device (enough
    copies that together they exceed L2, at most 8); one recipe is held at a
    time."""

    def __init__(self):
        self.key, self.Ws = None, None

    def get(self, spec, data_w, torch):
        key = (spec.name, spec.seed, spec.dtype)
        if self.key != key:
            self.key, self.Ws = None, None
            torch.cuda.empty_cache()
            tdt = torch.float32 if spec.dtype == "f32" else torch.bfloat16
            W0 = torch.from_numpy(data_w).to(tdt).cuda()
            n = max(1, min(8, -(-2 * L2_BYTES // (W0.numel() * W0.element_size()))))
            self.key, self.Ws = key, [W0] + [W0.clone() for _ in range(n - 1)]
        return self.Ws

    def drop(self, torch):
        self.key, self.Ws = None, None
        torch.cuda.empty_cache()


def _time_forward(spec, steps, warmup, cache, peaks):
    """Device time of one ttq_linear_forward at one workload point: K calls
    captured in a CUDA graph, CUDA events around its replay, W rotating over
    copies that exceed L2.  Returns a dict with the time next to the floor
    of the point's algorithmic bytes and flops at the measured peaks."""
    import numpy as np
    import torch

    from test_weight_quantization_ttq_b200 import synth, ttq

    hbm, tc = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops"] * 1e12
    stream = torch.cuda.current_stream()
    f32 = spec.dtype == "f32"
    tdt = torch.float32 if f32 else torch.bfloat16
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(tdt).cuda()
    need_w = cache.key != (spec.name, spec.seed, spec.dtype)
    data = synth.generate(spec, need_w=need_w)
    Ws = cache.get(spec, data.get("W"), torch)
    X = dev(data["X"])
    A = dev(data["A"]) if spec.r else None
    B = dev(data["B"]) if spec.r else None
    Y = torch.empty((spec.T, spec.dp), dtype=tdt, device="cuda")
    dt = ttq.TTQ_F32 if f32 else ttq.TTQ_BF16
    ws = ttq.new_workspace(spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group, dt)
    floor_us, nbytes, flops = _floor_us(spec, hbm, tc)
    k = steps if floor_us < 200 else max(5, steps // 10)

    def fwd(i):
        ttq.ttq_linear_forward(X, Ws[i % len(Ws)], A, B, spec.p, spec.lam, spec.alpha, spec.bits,
                               spec.group, ws=ws, Y=Y)

    for i in range(warmup):
        fwd(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(k):
            fwd(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / k
    st, flags = ttq.ttq_get_status(ws)
    if st != ttq.TTQ_OK:
        raise RuntimeError(f"{spec.name} T={spec.T}: device status {ttq.status_string(st)} (flags {flags:#x})")
    out = {"workload": f"{spec.name}_T{spec.T}", "d": spec.d, "dp": spec.dp, "T": spec.T, "bits": spec.bits,
           "group": spec.group, "r": spec.r, "p": spec.p, "alpha": spec.alpha, "dtype": spec.dtype,
           "us": us, "tokens_per_s": spec.T / us * 1e6, "floor_us": floor_us, "frac_of_floor": floor_us / us,
           "algorithmic_bytes": nbytes, "flops": flops, "calls_timed": k,
           "kernels_per_call": ttq.ttq_linear_forward_kernels(spec.d, spec.dp, spec.T, spec.r, spec.p, dt,
                                                               spec.bits, spec.group)}
    del g
    return out


def run_table(args):
    """Forward time of ttq_linear_forward at every configured workload point
    (the fp32 d = 256 case, the q_proj prefill, the three MLP projections at
    T = 512 and their block, decode at T = 1, 4, 16, and the 70B-like MLP
    shape at T = 1 .. 4096 with p = 2, alpha = 0.5), each next to the floor
    its algorithmic bytes and flops give at the measured peaks.  K calls are
    captured in a CUDA graph and its replay is timed with CUDA events; W
    rotates over enough copies to exceed L2.  One GPU; one JSON line per
    point and a closing line with the clocks."""
    import torch

    from test_weight_quantization_ttq_b200 import synth

    peaks = _measured_peaks()
    points = [synth.C1, synth.C2, synth.C3_GATE, synth.C3_UP, synth.C3_DOWN]
    points += [synth.C4.with_(T=t) for t in synth.C4_TOKENS]
    points += [synth.C5.with_(T=t, p=2.0, alpha=0.5) for t in synth.C5_TOKENS]
    if args.only:
        points = [sp for sp in points if args.only in f"{sp.name}_T{sp.T}"]
    sampler = ClockSampler(0)
    sampler.start()
    cache = _WeightCache()
    block_us = 0.0
    for spec in points:
        try:
            row = _time_forward(spec, args.steps, args.warmup, cache, peaks)
            if spec.name.startswith("mlp_") and spec.T == 512:
                block_us += row["us"]
            print(json.dumps({"table": "forward", **row}), flush=True)
        except Exception as exc:  # one point failing does not lose the others
            torch.cuda.synchronize()
            print(json.dumps({"table": "forward", "workload": f"{spec.name}_T{spec.T}",
                              "error": f"{type(exc).__name__}: {exc}"[:300]}), flush=True)
    print(json.dumps({"table": "mlp_block_4096x11008_T512", "us": block_us, "tokens_per_s": 512 / block_us * 1e6 if block_us > 0 else None,
                      "note": "gate + up + down projections; the SiLU gating between them is not timed",
                      "hbm_peak_gbs": peaks["hbm_gbs"], "bf16_peak_tflops": peaks["bf16_tflops"],
                      "peak_source": peaks["source"], "clocks": sampler.stop()}), flush=True)


def run_ab_dequant(args):
    """Where the prefill product gets its weight operand: the
    materialised form (the quantiser also writes the binary16 s (q - z), the
    plain tcgen05 GEMM reads it by TMA) against dequantisation inside the
    product's main loop (the quantiser writes codes only; the GEMM's
    producer warps turn each TMA-fed code tile into the binary16 operand in
    shared memory).  At the q_proj prefill (d = d' = 4096, T = 2048, INT4
    g128) and the 70B-like MLP shape at T = 4096 (INT2 g64, no low-rank
    term), each pair of entry points and each kernel in a CUDA graph of K
    calls, W rotating over copies larger than L2.  One JSON line per
    workload."""
    import torch

    from test_weight_quantization_ttq_b200 import synth, ttq

    stream = torch.cuda.current_stream()
    peaks = _measured_peaks()

    def graph_time(fn, k):
        for i in range(args.warmup):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(k):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / k

    for spec in (synth.C2, synth.C5.with_(T=4096, r=0)):
        data = synth.generate(spec)
        X = torch.from_numpy(data["X"]).to(torch.bfloat16).cuda()
        W0 = torch.from_numpy(data["W"]).to(torch.bfloat16).cuda()
        n = max(2, -(-2 * L2_BYTES // (W0.numel() * 2)))
        Ws = [W0] + [W0.clone() for _ in range(n - 1)]
        d, dp, T, b, g = spec.d, spec.dp, spec.T, spec.bits, spec.group
        D, Dr, Xs = ttq.ttq_act_norm_scale(X, spec.p, spec.lam, spec.alpha)
        ws = ttq.new_workspace(d, dp, T, 0, b, g)
        codes = torch.empty((dp, d * b // 32), dtype=torch.int32, device="cuda")
        sc = torch.empty((dp, d // g), dtype=torch.int16, device="cuda")
        ze = torch.empty_like(sc)
        Wh = torch.empty((dp, d), dtype=torch.float16, device="cuda")
        Y = torch.empty((T, dp), dtype=torch.bfloat16, device="cuda")
        k = max(3, min(args.steps, 20))

        def quant_wq(i):
            ttq.ttq_quantize_dequant_weight(Ws[i % n], D, b, g, ws=ws, codes=codes, scales=sc, zeros=ze, W_hat=Wh)

        def gemm_wq(i):
            ttq.ttq_dequantized_gemm(Wh, Xs, ws=ws, Y=Y)

        def quant(i):
            ttq.ttq_quantize_weight(Ws[i % n], D, b, g, ws=ws, codes=codes, scales=sc, zeros=ze)

        def gemm_codes(i):
            ttq.ttq_dequant_gemm(codes, sc, ze, None, Xs, None, None, b, g, ws=ws, Y=Y)

        t = {name: graph_time(fn, k) for name, fn in (
            ("materialised_quantiser", quant_wq), ("materialised_gemm", gemm_wq),
            ("materialised_pair", lambda i: (quant_wq(i), gemm_wq(i))),
            ("in_mainloop_quantiser", quant), ("in_mainloop_gemm", gemm_codes),
            ("in_mainloop_pair", lambda i: (quant(i), gemm_codes(i))))}
        st, flags = ttq.ttq_get_status(ws)
        flops = 2.0 * dp * d * T
        print(json.dumps({"ab": "prefill weight operand: materialised binary16 W_hat vs in-mainloop dequantisation",
                          "workload": f"{spec.name}_T{T}", "d": d, "dp": dp, "T": T, "bits": b, "group": g,
                          "us": t, "gemm_tflops": {"materialised": flops / t["materialised_gemm"] / 1e6,
                                                   "in_mainloop": flops / t["in_mainloop_gemm"] / 1e6},
                          "bf16_peak_tflops": peaks["bf16_tflops"], "calls_timed": k,
                          "status": ttq.status_string(st)}), flush=True)
        del Ws, W0
        torch.cuda.empty_cache()


def run_lowrank(args):
    """The static low-rank initialisation at the 70B-like MLP shape
    (d' = 28672, d = 8192, bf16 W, r = 64, 8 extra sampled directions, 2
    subspace iterations): K calls timed with CUDA events.  Reported against
    the fp32 CUDA-core peak (148 SMs x 128 lanes x 2 flops x the max SM
    clock), since its products run on CUDA cores.  One GPU; one JSON line."""
    import torch

    from test_weight_quantization_ttq_b200 import synth, ttq

    dp, d, r, over, q = 28672, 8192, 64, 8, 2
    l = r + over
    g = torch.Generator(device="cuda").manual_seed(1)
    W = (torch.randn((dp, d), generator=g, device="cuda") * 0.015).to(torch.bfloat16)
    Om = torch.from_numpy(synth.gaussian_test_matrix(d, l, seed=7)).cuda()
    n = ttq.ttq_lowrank_workspace_size(dp, d, r, over)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    ttq.ttq_workspace_init(ws)
    B = torch.empty((dp, r), dtype=torch.bfloat16, device="cuda")
    A = torch.empty((r, d), dtype=torch.bfloat16, device="cuda")
    R = torch.empty_like(W)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        ttq.ttq_lowrank_init(W, r, Om, power_iters=q, ws=ws, B=B, A=A, W_res=R)
    torch.cuda.synchronize()
    sampler = ClockSampler(0)
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        ttq.ttq_lowrank_init(W, r, Om, power_iters=q, ws=ws, B=B, A=A, W_res=R)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    t = e0.elapsed_time(e1) / 1e3 / args.steps
    st, flags = ttq.ttq_get_status(ws)
    # multiply-adds: W passes (W Omega, q x (W^T Q, W Z), W^T Q) of 2 d' d l
    # each, the residual 2 d' d r, the Gram matrices and l-column products
    passes = 2 + 2 * q
    flops = passes * 2.0 * dp * d * l + 2.0 * dp * d * r
    flops += (3 * (1 + 2 * q)) * (2.0 * dp * l * l * 2) + 2.0 * d * l * l + 2.0 * (dp + d) * l * r
    sm_max = clocks.get("sm_max_mhz") or 1965.0
    peak = 148 * 128 * 2 * sm_max * 1e6 / 1e12
    achieved = flops / t / 1e12
    print(json.dumps({"metric": "TTQ low-rank init ms", "value": t * 1e3, "unit": "ms", "higher_is_better": False,
                      "steps": args.steps, "warmup": args.warmup, "dtype": "bf16 W, fp32 products",
                      "data": "synthetic", "status": ttq.status_string(st), "flags": flags,
                      "config": {"workload": "lowrank_init_28672x8192_r64", "dp": dp, "d": d, "r": r,
                                 "oversample": over, "power_iters": q},
                      "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                                   "frac": achieved / peak,
                                   "peak_source": "148 SMs x 128 fp32 lanes x 2 flops x max SM clock"},
                      "hbm_bytes_of_W_passes": (passes + 2) * 2.0 * dp * d,
                      "clocks": clocks}), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the decode and 70B-like MLP points added to the default line")
    ap.add_argument("--profile", action="store_true",
                    help="short run for a profiler: no clock warm-up loop, no CPU baseline, no e2e leg")
    ap.add_argument("--scheme", choices=sorted(SCHEMES), default="asym",
                    help="code scheme of the q_proj prefill workload (asym: the default INT4; fp8 uses 8-bit E4M3 codes)")
    ap.add_argument("--decode", type=int, default=0, metavar="T",
                    help="time the decode workload (d = 4096, d' = 14336, INT4 g128) at T <= 16 tokens instead")
    ap.add_argument("--lowrank", action="store_true",
                    help="time the static low-rank initialisation (d' = 28672, d = 8192, r = 64) instead")
    ap.add_argument("--table", action="store_true",
                    help="time the forward at every configured workload point, one JSON line each, instead")
    ap.add_argument("--ab-dequant", action="store_true",
                    help="A/B of the prefill weight operand: materialised W_hat vs dequantisation in the "
                         "product's main loop, instead")
    ap.add_argument("--only", default="", metavar="NAME",
                    help="with --table: only the points whose workload name (e.g. mlp70b_8192x28672_T128) "
                         "contains NAME")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.table:
        run_table(args)
    elif args.ab_dequant:
        run_ab_dequant(args)
    elif args.lowrank:
        run_lowrank(args)
    elif args.decode:
        run_decode(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
