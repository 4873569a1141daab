#!/usr/bin/env python
"""Benchmark of the per-layer SliM-LLM quantize path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one slim_quantize_layer call (hessian -> hinv_diag -> salience ->
sba_search -> sqc) on a synthetic layer, inputs resident in HBM. The default is
the largest single-GPU benchmark layer: the LLaMA-13B up_proj shape (W
13824x5120) at group 32 (k = 160, 81 candidates), X 262144 x 5120 bf16;
--workload selects the others (q_proj 4096x4096, down_proj 4096x11008, up_proj
at groups 128 / 64). Prints one JSON line (rank 0).

Metric: weights quantized per second per layer, Mparam/s = m*n / step time.
With --gpus N (torchrun) every rank quantizes its own independent layer
(replicas, no data-path collective); value = N*m*n / max-over-ranks step time.

--impl reference times the float64 CPU oracle on the host cores instead, on a
bounded token/row sample of the same workload per step, extrapolated to the
full layer (rank 0 only): ms_per_step is the sample's own wall time, value the
extrapolated full-layer throughput.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from post_weight_quantization_hessian_b200 import synthetic as syn  # noqa: E402

METRIC = "weights quantized/sec per layer (Mparam/s)"
UNIT = "Mparam/s"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0:     # first sample before the timed region
                time.sleep(0.05)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle sample
def oracle_sample(spec: syn.LayerSpec, W: np.ndarray, tokens: int, rows: int, threads: int):
    """Time the oracle's stages on a bounded sample and extrapolate to the full layer.

    Token-proportional stages (hessian, sba_search) run on `tokens` tokens and
    are scaled by N / tokens; hinv_diag and salience run in full; sqc runs on
    `rows` rows and is scaled by m / rows. Returns (seconds for the full layer,
    description).
    """
    from oracle import slim_oracle as O
    x = syn.activations_f64(spec, rows=np.arange(tokens))
    t0 = time.perf_counter()
    H = O.hessian(x)
    t1 = time.perf_counter()
    h = O.hinv_diag(H)
    t2 = time.perf_counter()
    S = O.group_salience(W, h, spec.group)
    order = O.salience_order(S)
    t3 = time.perf_counter()
    sba = O.sba_search(W, x, order, spec.group, spec.avg_bits, reassociate=True)
    t4 = time.perf_counter()
    O.sqc_calibrate(W[:rows], h, sba.bits, spec.group, spec.lam, spec.n_tau)
    t5 = time.perf_counter()
    scale_t = spec.N / tokens
    full = (t1 - t0) * scale_t + (t2 - t1) + (t3 - t2) + (t4 - t3) * scale_t + (t5 - t4) * spec.m / rows
    desc = (f"oracle stages on {tokens} of {spec.N} tokens (hessian, sba_search; x{scale_t:.0f}), full "
            f"hinv_diag and salience, sqc on {rows} of {spec.m} rows (x{spec.m / rows:.0f}); "
            f"{t5 - t0:.1f} s of CPU work, {threads} BLAS threads")
    return full, desc, t5 - t0


# ----------------------------------------------------------------------------- distributed plumbing
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """Largest value over the ranks (the job's step time is its slowest rank's)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_spec(spec: syn.LayerSpec, rank: int, world: int) -> syn.LayerSpec:
    """With N ranks every rank quantizes its own independent layer of the same shape
    (replicas; no data-path collective), seeded by its rank."""
    return spec if world == 1 else spec.replace(seed=spec.seed + 7919 * rank)


def job_value(world: int, spec: syn.LayerSpec, ms_per_step: float) -> float:
    """Whole-job throughput: the weights all ranks quantized per second (Mparam/s)."""
    return world * spec.m * spec.n / (ms_per_step * 1e-3) / 1e6


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, spec, world, rank):
    if rank != 0:
        return 0
    threads = host_cores()
    W = syn.make_weight(spec)
    tokens, rows = args.ref_tokens, args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(spec, W, tokens // 4, rows // 4, threads)
    times, walls = [], []
    desc = ""
    for _ in range(args.steps):
        full, desc, wall = oracle_sample(spec, W, tokens, rows, threads)
        times.append(full)
        walls.append(wall)
    sec = statistics.mean(times)
    value = spec.m * spec.n / sec / 1e6
    # ms_per_step: the wall time of one sample step as run; value: the full layer's
    # throughput from the extrapolated full-layer time
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(walls) * 1e3,
            "full_layer_ms_extrapolated": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec.name, "m": spec.m, "n": spec.n, "N": spec.N, "group": spec.group,
                       "avg_bits": spec.avg_bits, "lambda": spec.lam, "n_tau": spec.n_tau},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def sba_flops(spec, split=None, order=None):
    """Tensor-core flops of one sba_score launch as executed: y and d_0 over K = n
    (every 64-column box once, the split boxes twice: their hi and lo weight parts),
    then per further candidate p the two changed groups (each taken twice when its box
    is split): the regrouped incremental form. split: per-box 0/1; order: the group
    order of the search. Without them, every box once."""
    P = spec.k // 2 + 1
    nbox = (spec.n + 63) // 64
    sp = np.zeros(nbox, np.int64) if split is None else np.asarray(split, np.int64)
    tok = 2.0 * spec.N * spec.m
    phase_a = 2 * tok * 64 * float((1 + sp).sum())   # N = 256 MMAs: y and d together
    steps = 0.0
    if P > 1:
        order = np.arange(spec.k) if order is None else np.asarray(order)
        for p in range(1, P):
            for c in (order[p - 1], order[spec.k - p]):
                b0 = (c * spec.group) // 64
                nb = max(1, spec.group // 64)
                steps += tok * spec.group * (1 + sp[b0:b0 + nb].mean())
    return phase_a + steps


def sba_flops_pages(spec):
    """The same scores counted the pages' way: one dequant-GEMM per candidate
    (P of them) plus the full-precision outputs, (P + 1) 2 N n m."""
    P = spec.k // 2 + 1
    return (P + 1) * 2.0 * spec.N * spec.n * spec.m


def source_hash(*paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, workload: str, src_hash: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary
    (profiles/traffic.json), or None when absent or taken on other source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel, {}).get(workload)
    except (OSError, ValueError, AttributeError):
        return None
    if not rec or rec.get("source_hash") != src_hash:
        return None
    return rec.get("bytes_per_launch")


def timed(fn, reps, flush, stream):
    """Mean device time (ms) of fn() over reps calls, L2 flushed before each (CUDA events
    on the launching stream around each call alone)."""
    import torch
    ms = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        ms.append(a.elapsed_time(b))
    return statistics.mean(ms)


def extra_kernels(spec, Wd, Xd, d, stages, flush, stream):
    """fp64 peaks measured here, then: the inverse-Hessian and SQC stages against them
    (from the step's stage times), the GPTQ backbone (slim_gptq with this layer's H and
    bits) and the packed dequant GEMV (batch 1 and 8) on this layer's outputs."""
    import torch
    from post_weight_quantization_hessian_b200 import slim
    pk, _ = peaks()
    dmma, dfma = slim.slim_peak_fp64()
    m, n, k = spec.m, spec.n, spec.k
    out = {"fp64_peaks": {"dmma_tflops": dmma, "dfma_tflops": dfma, "note": "measured in this run"}}
    hinv_flops = 2.0 * n ** 3 / 3.0
    out["hinv_diag"] = {"ms": stages["hinv_diag"], "tflops": hinv_flops / (stages["hinv_diag"] * 1e-3) / 1e12,
                        "frac": hinv_flops / (stages["hinv_diag"] * 1e-3) / 1e12 / dmma,
                        "note": "2 n^3 / 3 fp64 flops (Cholesky and inverse), of the measured fp64 MMA rate; "
                                "in-step time (the SBA operand preparation runs beside it)"}
    sqc_ops = 12.0 * spec.n_tau * m * n
    out["sqc"] = {"ms": stages["sqc"], "fp64_tops": sqc_ops / (stages["sqc"] * 1e-3) / 1e12,
                  "frac": sqc_ops / (stages["sqc"] * 1e-3) / 1e12 / dfma,
                  "note": "about 12 fp64 operations per (weight, tau candidate), of the measured fp64 FMA rate"}
    H = slim.slim_hessian(Xd)
    bits = d["bits"]
    gws = torch.empty(slim._lib().slim_gptq_workspace_bytes(m, n), dtype=torch.uint8, device=Wd.device)
    g_ms = timed(lambda: slim.slim_gptq(Wd, H, bits, spec.group, spec.avg_bits, spec.lam, spec.n_tau, ws=gws),
                 3, flush, stream)
    g_flops = float(m) * n * n
    out["gptq"] = {"ms": g_ms, "tflops": g_flops / (g_ms * 1e-3) / 1e12, "frac": g_flops / (g_ms * 1e-3) / 1e12 / dmma,
                   "note": "m n^2 fp64 flops (the error-compensation updates), of the measured fp64 MMA rate; "
                           "includes its own factorization of the reversed Hessian and SQC per group"}
    del gws, H
    codes, scale, zero = d["codes"], d["scale"], d["zero"]
    rows = {}
    # the call is microseconds long: it is timed from a CUDA graph of back-to-back calls, each
    # on its own copy of the packed layer (copies together several times the L2), so the
    # device time is measured without host launch gaps and every call reads from DRAM
    layer_bytes = codes.numel() * 4 + 2 * scale.numel() * 4
    ncopy = max(2, int(3 * 126e6 // layer_bytes) + 1)
    copies = [(codes.clone(), scale.clone(), zero.clone()) for _ in range(ncopy)]
    reps = max(24, ncopy)
    for B in (1, 8):
        x = torch.randn((B, n), device=Wd.device).to(torch.bfloat16)
        ys = [torch.empty((B, m), dtype=torch.float32, device=Wd.device) for _ in range(ncopy)]
        gws = torch.empty(max(256, slim._lib().slim_dequant_gemv_workspace_bytes(m, n, spec.group, spec.avg_bits, B)), dtype=torch.uint8,
                          device=Wd.device)
        side = torch.cuda.Stream(device=Wd.device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(ncopy):
                c_, s_, z_ = copies[i]
                slim.slim_dequant_gemv(c_, bits, s_, z_, spec.group, spec.avg_bits, x, y=ys[i], ws=gws)
        stream.wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(reps):
                c_, s_, z_ = copies[i % ncopy]
                slim.slim_dequant_gemv(c_, bits, s_, z_, spec.group, spec.avg_bits, x, y=ys[i % ncopy], ws=gws)
        g.replay()
        torch.cuda.synchronize()
        ms = []
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            ms.append(a.elapsed_time(b))
        us = min(ms) * 1e3 / reps
        del g
        byt = layer_bytes + k + B * n * 2 + B * m * 4
        rows[f"batch{B}"] = {"us": us, "bytes": byt, "gbs": byt / (us * 1e-6) / 1e9,
                             "frac": byt / (us * 1e-6) / 1e9 / pk["hbm_gbs"]}
    del copies
    out["dequant_gemv"] = dict(rows, note="y = x W_hat^T on the packed codes; bytes = codes + fp32 scale and "
                                          "zero + bits + x + y, of the measured HBM copy bandwidth; device time "
                                          f"per call from a CUDA graph of {reps} calls over {ncopy} copies of the layer")
    return out


def run_ours(args, spec, world, rank, local):
    import torch
    from post_weight_quantization_hessian_b200 import build, slim
    if not os.path.exists(slim.LIB_PATH):
        build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    spec = replica_spec(spec, rank, world)
    W = syn.make_weight(spec)
    Xh_pinned = torch.empty((spec.N, spec.n), dtype=torch.int16, pin_memory=True)
    syn.make_activations(spec, out=Xh_pinned.numpy().view(np.uint16))
    W_pinned = torch.from_numpy(W).pin_memory()
    Wd = W_pinned.to(dev, non_blocking=True)
    Xd = Xh_pinned.to(dev, non_blocking=True).view(torch.bfloat16)
    torch.cuda.synchronize()
    ws = slim.alloc_workspace(Wd, Xd, spec.group, spec.avg_bits)
    out = slim._layer_outputs(Wd, spec.group, spec.avg_bits)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)     # > 126 MB L2
    stream = torch.cuda.current_stream()

    bufs = slim.layer_buffers(Wd, spec.group, spec.avg_bits, want_H=False)

    def step():
        return slim.slim_quantize_layer_ex(Wd, Xd, spec.group, spec.avg_bits, spec.lam, spec.n_tau, ws=ws,
                                           want_H=False, bufs=bufs)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    barrier(world)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    stage_ms, kern_ms = [], []
    n0 = slim.slim_launch_count()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            d = step()
            ev[i][1].record(stream)
            stage_ms.append(d["stage_ms"])
            kern_ms.append(d["kernel_ms"])
        torch.cuda.synchronize()
        barrier(world)
    launches = (slim.slim_launch_count() - n0) / args.steps
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms = max_over_ranks(statistics.mean(step_ms), world)
    spread = {"min": min(step_ms), "median": statistics.median(step_ms), "max": max(step_ms)}
    value = job_value(world, spec, ms)
    p_star = d["p_star"]

    # ---- end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        k = spec.k
        hc = (np.empty((spec.m, spec.n * spec.avg_bits // 32), np.uint32), np.empty((spec.m, k), np.float32),
              np.empty((spec.m, k), np.float32), np.empty(k, np.uint8))
        pinned_out = [torch.from_numpy(a).pin_memory() for a in hc]
        outs = tuple(t.numpy() for t in pinned_out)
        Wn, Xn = W_pinned.numpy(), Xh_pinned.numpy().view(np.uint16)
        slim.slim_quantize_layer_host(Wn, Xn, spec.group, spec.avg_bits, spec.lam, spec.n_tau, out=outs)
        barrier(world)
        torch.cuda.synchronize()
        e2e_ms = []
        for _ in range(max(1, min(args.steps, 5))):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            slim.slim_quantize_layer_host(Wn, Xn, spec.group, spec.avg_bits, spec.lam, spec.n_tau, out=outs)
            b.record(stream)
            b.synchronize()
            e2e_ms.append(a.elapsed_time(b))
        barrier(world)
        ems = max_over_ranks(statistics.mean(e2e_ms), world)
        e2e = {"value": job_value(world, spec, ems), "unit": UNIT,
               "h2d_bytes_per_step": int(Wn.nbytes + Xn.nbytes),
               "d2h_bytes_per_step": int(sum(o.nbytes for o in outs)), "ms_per_step": ems}

    # ---- roofline of the dominant kernel (sba scoring, tensor cores). The kernel
    # runs for tens of milliseconds inside the step, not seconds back to back, so
    # its denominator is the burst bf16 figure (fp16 operands run at the bf16 rate).
    pk, pk_kind = peaks()
    sba_ms = statistics.mean(k[1] for k in kern_ms)
    split = d["sba_split"].cpu().numpy()
    flops = sba_flops(spec, split=split, order=d["order"].cpu().numpy())
    achieved = flops / (sba_ms * 1e-3) / 1e12
    peak = pk["bf16_tflops"]
    pages = sba_flops_pages(spec)
    src = source_hash("post_weight_quantization_hessian_b200/csrc/sba.cu",
                      "post_weight_quantization_hessian_b200/csrc/common.cuh")
    roofline = {"kernel": "sba_score_kernel", "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic_record("sba_score_kernel", spec.name, src),
                "peak_kind": f"{pk_kind} bf16 dense burst (fp16 operands, same nominal rate)",
                "flops_per_launch": flops, "ms_per_launch": sba_ms,
                "flops_note": "executed: y and d_0 over K = n plus two groups per further candidate, "
                              "the boxes taken as fp16 hi/lo pairs twice",
                "split_boxes": int(split.sum()), "boxes": int(split.size),
                "pages_flops_per_launch": pages,
                "pages_equivalent_tflops": pages / (sba_ms * 1e-3) / 1e12}
    hs_ms = statistics.mean(k[0] for k in kern_ms)
    syrk_flops = float(spec.N) * spec.n * (spec.n + 1)
    stages = {nm: statistics.mean(s[i] for s in stage_ms)
              for i, nm in enumerate(["hessian", "hinv_diag", "salience", "sba_search", "sqc", "total"])}

    # ---- the other kernels of the path and of the next rows, each on this workload's shape
    kernels = {"hessian_syrk_tc": {"ms": hs_ms, "tflops": syrk_flops / (hs_ms * 1e-3) / 1e12,
                                   "frac": syrk_flops / (hs_ms * 1e-3) / 1e12 / pk["bf16_tflops"],
                                   "note": "N n (n + 1) flops (the symmetric product), of the burst bf16 peak"}}
    if not args.no_extras:
        kernels.update(extra_kernels(spec, Wd, Xd, d, stages, flush, stream))
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": spec.name, "m": spec.m, "n": spec.n, "N": spec.N, "x_dtype": spec.x_dtype,
                       "group": spec.group, "avg_bits": spec.avg_bits, "lambda": spec.lam, "n_tau": spec.n_tau,
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "arithmetic": "X bf16 in; tensor cores fp16 x fp16 -> fp32 (weight side as hi/lo "
                                     "fp16 pairs); inverse Hessian, salience, SQC in fp64",
                       "l2": "flushed between steps (256 MB write outside the timed events); X is 2.1 GB"},
            "roofline": roofline,
            "kernels": kernels,
            "stage_ms": stages, "step_ms_spread": spread, "p_star": p_star, "gpu_launches": launches, "e2e": e2e}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = host_cores()
        full, desc, _ = oracle_sample(spec, W, args.ref_tokens, args.ref_rows, threads)
        line["cpu_baseline"] = {"value": spec.m * spec.n / full / 1e6, "unit": UNIT, "cores": threads,
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        line["clocks"] = clk.summary()
        # the exponential pipe: one ex2 per token and output for phase A's e^(y - M) and
        # one per token, output and candidate for e^d (nominal 16 per clock per SM, at the
        # median SM clock sampled during the timed steps)
        mhz = line["clocks"].get("sm_mhz") or 1965.0
        nsm = torch.cuda.get_device_properties(dev).multi_processor_count
        exps = float(spec.N) * spec.m * (spec.k // 2 + 2)
        roofline["exp_units"] = {"achieved_per_s": exps / (sba_ms * 1e-3),
                                 "peak_per_s": 16.0 * nsm * mhz * 1e6,
                                 "frac": exps / (sba_ms * 1e-3) / (16.0 * nsm * mhz * 1e6),
                                 "note": "ex2 per launch N m (P + 1); nominal 16 per clock per SM at the sampled "
                                         "median clock"}
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- the 7B sweep
SWEEP = "llama7b_sweep"


def run_sweep(args, world, rank, local):
    """32 synthetic LLaMA-7B decoder blocks x (q, k, v, o 4096x4096; gate, up 11008x4096;
    down 4096x11008), quantized one after another, each layer with its own weights and
    262144 bf16 tokens drawn on the device (per-layer seed 1000 block + layer). Only the
    slim_quantize_layer calls are timed (CUDA events around each); the drawing of the next
    layer's inputs is not. With --manifest, one JSON line per finished layer is appended
    (block, layer, ms, p*, allocation) and --resume skips the layers already there. With
    --gpus N the layers are dealt round-robin to the ranks (no data-path collective)."""
    import torch
    from post_weight_quantization_hessian_b200 import build, slim
    if not os.path.exists(slim.LIB_PATH):
        build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    layers = [(b, l) for b in range(args.blocks) for l in range(len(syn.SWEEP_LAYERS))]
    mine = layers[rank::world]
    done = {}
    if args.manifest and args.resume and os.path.exists(args.manifest):
        with open(args.manifest) as f:
            for ln in f:
                r = json.loads(ln)
                done[(r["block"], r["layer"])] = r
    ws_bytes = max(slim.slim_workspace_bytes(m, n, syn.CALIB_TOKENS, 1, 128, 2) for _, m, n in syn.SWEEP_LAYERS)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    # warm-up: one layer of each shape
    for l in (0, 4, 6):
        W, X = syn.device_layer(syn.sweep_spec(0, l, N=16384), dev)
        slim.slim_quantize_layer(W, X, 128, 2, ws=ws)
    torch.cuda.synchronize()
    barrier(world)
    tot_ms, params, n_layers = 0.0, 0, 0
    with ClockSampler(local) as clk:
        for (b, l) in mine:
            spec = syn.sweep_spec(b, l)
            if (b, l) in done:
                tot_ms += done[(b, l)]["ms"]
                params += spec.m * spec.n
                n_layers += 1
                continue
            W, X = syn.device_layer(spec, dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            d = slim.slim_quantize_layer_ex(W, X, 128, 2, 0.1, 50, ws=ws, want_H=False)
            e1.record(stream)
            e1.synchronize()
            ms = e0.elapsed_time(e1)
            tot_ms += ms
            params += spec.m * spec.n
            n_layers += 1
            if args.manifest:
                bits = d["bits"].cpu().numpy()
                with open(args.manifest, "a") as f:
                    f.write(json.dumps({"block": b, "layer": l, "name": spec.name, "ms": ms, "p_star": d["p_star"],
                                        "bits": bits.tolist()}) + "\n")
            del W, X, d
    barrier(world)
    ms_all = max_over_ranks(tot_ms, world)
    params_all = params * world if world > 1 else params
    value = params_all / (ms_all * 1e-3) / 1e6
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": 1, "warmup": 3,
                "ms_per_step": ms_all, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f16", "data": "synthetic",
                "config": {"workload": f"{SWEEP}_{args.blocks}x7", "layers": len(layers), "params": params_all,
                           "N": syn.CALIB_TOKENS, "group": 128, "avg_bits": 2,
                           "l2": "inputs (1-6 GB per layer) far larger than L2",
                           "note": "a step is the whole sweep; per-layer inputs drawn on the device between "
                                   "the timed calls"},
                "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama13b_up_proj_13824x5120_g32", choices=sorted(syn.WORKLOADS) + [SWEEP])
    ap.add_argument("--blocks", type=int, default=32, help="sweep: decoder blocks")
    ap.add_argument("--manifest", default="", help="sweep: JSONL of finished layers")
    ap.add_argument("--resume", action="store_true", help="sweep: skip the layers already in the manifest")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the GPTQ / dequant / fp64-peak measurements")
    ap.add_argument("--ref-tokens", type=int, default=2048)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--tokens", type=int, default=0, help="override N (profiling runs on a smaller case)")
    args = ap.parse_args(argv)
    world, rank, local = dist_setup(args)
    if args.workload == SWEEP:
        try:
            return 0 if args.impl == "reference" and rank != 0 else (
                run_sweep(args, world, rank, local) if args.impl == "ours" else run_reference(
                    args, syn.sweep_spec(0, 6), world, rank))
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
    spec = syn.WORKLOADS[args.workload]
    if args.tokens:
        spec = spec.replace(N=args.tokens)
    try:
        if args.impl == "reference":
            return run_reference(args, spec, world, rank)
        return run_ours(args, spec, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
