#!/usr/bin/env python
"""Benchmark of the per-layer SliM-LLM quantize path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one slim_quantize_layer call (hessian -> hinv_diag -> salience ->
sba_search -> sqc) on a synthetic LLaMA-7B q_proj-shaped layer (W 4096x4096,
X 262144 x 4096 bf16), inputs resident in HBM. Prints one JSON line (rank 0).

Metric: weights quantized per second per layer, Mparam/s = m*n / step time.
With --gpus N (torchrun) every rank quantizes its own independent layer
(replicas, no data-path collective); value = N*m*n / max-over-ranks step time.

--impl reference times the float64 CPU oracle on the host cores instead, on a
bounded token/row sample of the same workload per step, extrapolated to the
full layer (rank 0 only).
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
    return full, desc


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
    times = []
    desc = ""
    for _ in range(args.steps):
        full, desc = oracle_sample(spec, W, tokens, rows, threads)
        times.append(full)
    sec = statistics.mean(times)
    value = spec.m * spec.n / sec / 1e6
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec.name, "m": spec.m, "n": spec.n, "N": spec.N, "group": spec.group,
                       "avg_bits": spec.avg_bits, "lambda": spec.lam, "n_tau": spec.n_tau},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def sba_flops(spec, ksplit=1):
    """Tensor-core flops of one sba_score launch: y and d_0 over K = n, then two
    g-column groups per further candidate (the regrouped incremental form)."""
    P = spec.k // 2 + 1
    return ksplit * (2 * 2.0 * spec.N * spec.n * spec.m + (P - 1) * 2 * 2.0 * spec.N * spec.group * spec.m)


def source_hash(*paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, src_hash: str):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != src_hash:
        return None
    return rec.get("bytes_per_launch")


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

    def step():
        return slim.slim_quantize_layer_ex(Wd, Xd, spec.group, spec.avg_bits, spec.lam, spec.n_tau, ws=ws,
                                           want_H=False)

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

    # ---- roofline of the dominant kernel (sba scoring, tensor cores)
    pk, pk_kind = peaks()
    sba_ms = statistics.mean(k[1] for k in kern_ms)
    flops = sba_flops(spec)
    achieved = flops / (sba_ms * 1e-3) / 1e12
    peak = pk["bf16_tflops_sustained"]
    src = source_hash("post_weight_quantization_hessian_b200/csrc/sba.cu",
                      "post_weight_quantization_hessian_b200/csrc/common.cuh")
    roofline = {"kernel": "sba_score_kernel", "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic_record("sba_score_kernel", src),
                "peak_kind": f"{pk_kind} bf16 dense sustained (fp16 operands, same nominal rate)",
                "flops_per_launch": flops, "ms_per_launch": sba_ms}
    hs_ms = statistics.mean(k[0] for k in kern_ms)
    syrk_flops = 2.0 * spec.N * spec.n * spec.n
    stages = {nm: statistics.mean(s[i] for s in stage_ms)
              for i, nm in enumerate(["hessian", "hinv_diag", "salience", "sba_search", "sqc", "total"])}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": spec.name, "m": spec.m, "n": spec.n, "N": spec.N, "x_dtype": spec.x_dtype,
                       "group": spec.group, "avg_bits": spec.avg_bits, "lambda": spec.lam, "n_tau": spec.n_tau,
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "flushed between steps (256 MB write outside the timed events); X is 2.1 GB"},
            "roofline": roofline,
            "kernels": {"hessian_syrk_tc": {"ms": hs_ms, "tflops": syrk_flops / (hs_ms * 1e-3) / 1e12,
                                            "note": "2Nn^2 flops counted (full square)"}},
            "stage_ms": stages, "p_star": p_star, "gpu_launches": launches, "e2e": e2e}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = host_cores()
        full, desc = oracle_sample(spec, W, args.ref_tokens, args.ref_rows, threads)
        line["cpu_baseline"] = {"value": spec.m * spec.n / full / 1e6, "unit": UNIT, "cores": threads,
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        line["clocks"] = clk.summary()
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=syn.Q_PROJ_7B.name, choices=sorted(syn.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-tokens", type=int, default=2048)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--tokens", type=int, default=0, help="override N (profiling runs on a smaller case)")
    args = ap.parse_args(argv)
    world, rank, local = dist_setup(args)
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
