"""Write oracle decisions for a full-size workload to tests/golden/<name>.json.

    python tests/golden/make_golden.py [--workload llama7b_q_proj_4096x4096] [--procs 8] [--out-dir DIR]

Everything stored comes from oracle/ (float64 CPU) on the seeded synthetic
inputs: group salience S, the order and its consecutive relative gaps, the
mean KL of every SBA candidate over all N tokens, p* and its margin, the
allocation. Token chunks run in worker processes (spawn); each worker calls
the oracle on its chunk and the parent adds the per-chunk sums.
"""
from __future__ import annotations

import argparse
import json
import multiprocessing as mp
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)


def _worker_init():
    os.environ.setdefault("OMP_NUM_THREADS", "1")


def _hess_chunk(args):
    name, c = args
    from oracle import slim_oracle as O
    from post_weight_quantization_hessian_b200 import synthetic as syn
    spec = syn.WORKLOADS[name]
    x = syn.activation_chunk(spec, c)
    x = (syn.bf16_bits_to_f32(x) if spec.x_dtype == "bf16" else x).astype(np.float64)
    return O.hessian(x)


def _kl_chunk(args):
    name, c, order = args
    from oracle import slim_oracle as O
    from post_weight_quantization_hessian_b200 import synthetic as syn
    spec = syn.WORKLOADS[name]
    W = syn.make_weight(spec)
    x = syn.activation_chunk(spec, c)
    x = (syn.bf16_bits_to_f32(x) if spec.x_dtype == "bf16" else x).astype(np.float64)
    r = O.sba_search(W, x, np.asarray(order), spec.group, spec.avg_bits, reassociate=True)
    return r.kl * x.shape[0], x.shape[0]


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama7b_q_proj_4096x4096")
    ap.add_argument("--procs", type=int, default=os.cpu_count())
    ap.add_argument("--out-dir", default=os.path.dirname(os.path.abspath(__file__)),
                    help="where to write <workload>.json (default: beside this script)")
    a = ap.parse_args(argv)
    from oracle import slim_oracle as O
    from post_weight_quantization_hessian_b200 import synthetic as syn
    spec = syn.WORKLOADS[a.workload]
    nch = syn.n_chunks(spec)
    t0 = time.time()
    ctx = mp.get_context("spawn")
    with ctx.Pool(a.procs, initializer=_worker_init) as pool:
        H = None
        for part in pool.imap_unordered(_hess_chunk, [(a.workload, c) for c in range(nch)]):
            H = part if H is None else H + part
        t_h = time.time()
        h = O.hinv_diag(H)
        W = syn.make_weight(spec)
        S = O.group_salience(W, h, spec.group)
        order = O.salience_order(S)
        srt = S[order]
        gaps = np.abs(srt[:-1] - srt[1:]) / np.abs(srt[:-1])
        t_s = time.time()
        tot, ntok = None, 0
        for kl_sum, cnt in pool.imap_unordered(_kl_chunk, [(a.workload, c, order.tolist()) for c in range(nch)]):
            tot = kl_sum if tot is None else tot + kl_sum
            ntok += cnt
    kl = tot / ntok
    p_star = int(np.argmin(kl))
    s = np.sort(kl)
    out = {
        "workload": a.workload,
        "source": "oracle/slim_oracle.py (float64) on the seeded synthetic inputs; written by tests/golden/make_golden.py",
        "m": spec.m, "n": spec.n, "N": spec.N, "group": spec.group, "avg_bits": spec.avg_bits,
        "S": S.tolist(), "order": order.tolist(), "order_rel_gaps": gaps.tolist(),
        "h_min": float(h.min()), "h_max": float(h.max()),
        "kl": kl.tolist(), "p_star": p_star,
        "kl_margin": float((s[1] - s[0]) / s[0]),
        "bits": O.allocation(order, spec.avg_bits, p_star).tolist(),
        "seconds": {"hessian": t_h - t0, "hinv_salience": t_s - t_h, "sba": time.time() - t_s},
    }
    path = os.path.join(a.out_dir, f"{a.workload}.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps({k: out[k] for k in ("order", "p_star", "kl_margin", "seconds")}))
    print("min order gap", float(gaps.min()), "at", int(gaps.argmin()))


if __name__ == "__main__":
    main()
