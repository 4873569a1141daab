"""The multi-rank path of bench.py on CPU: two gloo ranks (no GPU).

With N GPUs the benchmark runs N independent replicas (one layer per rank, no
data-path collective); the only cross-rank steps are a barrier around the
timed region and the max over ranks of the step time. These tests run those
steps with world_size 2 on the gloo backend, check that the ranks' layers are
independent, and that a two-rank torchrun of the reference arm prints exactly
one JSON line (rank 0) and exits 0 on every rank.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from post_weight_quantization_hessian_b200 import synthetic as syn  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        mx = bench.max_over_ranks(10.0 + rank, world)      # per-rank step times 10 ms, 11 ms
        bench.barrier(world)
        out[rank] = mx
    finally:
        dist.destroy_process_group()


def test_barrier_and_max_over_ranks_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        assert dict(out) == {0: 11.0, 1: 11.0}


def test_replica_layers_are_independent_and_value_counts_all_ranks():
    spec = syn.WORKLOADS["tiny_256x512"]
    s0, s1 = bench.replica_spec(spec, 0, 2), bench.replica_spec(spec, 1, 2)
    assert bench.replica_spec(spec, 0, 1) is spec
    assert s0.seed != s1.seed and (s0.m, s0.n, s0.N) == (s1.m, s1.n, s1.N)
    assert not np.array_equal(syn.make_weight(s0), syn.make_weight(s1))
    # whole-job throughput: N layers per (max over ranks) step time
    assert bench.job_value(2, spec, 10.0) == pytest.approx(2 * bench.job_value(1, spec, 10.0))
    assert bench.job_value(4, spec, 20.0) == pytest.approx(2 * bench.job_value(1, spec, 10.0))


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny_256x512", "--steps", "1", "--warmup", "0",
           "--ref-tokens", "256", "--ref-rows", "16"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT,
                       env={**os.environ, "OMP_NUM_THREADS": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
