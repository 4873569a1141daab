"""Seeded synthetic layers: weights W and calibration activations X.

This module only draws inputs. It holds none of the quantizer's arithmetic, so
both the CUDA path and the float64 CPU oracle may consume what it produces.

What the inputs stand in for
----------------------------
SliM-LLM calibrates on 128 WikiText2 sequences of 2048 tokens and quantizes the
linear layers of LLaMA/OPT models (rkmt.cn write-up of the ICML 2025 SliM-LLM
paper, section "实验设计与结果 / 评测协议"). Neither the text nor the trained
weights are available, so every layer is synthetic:

* W (out x in, float32, row-major) ~ N(0, 0.02^2). A few input columns are
  scaled up to make salient channels. For the LLaMA-shaped layers they form
  three contiguous 16-column clusters at the positions the write-up reports for
  LLaMA-7B layer 2 (around channels 2100, 3218 and 3853, section
  "为什么低比特量化精度会崩坏"), rescaled to the layer's input width.
* X (tokens x in) ~ N(0, 1), float32 or rounded once to bf16 (round to nearest
  even). A few outlier input channels are scaled up. Per the paper's Theorem 1
  (activation outlier channels produce the salient-weight clusters) they are
  drawn from inside the weight clusters.

Determinism: every draw uses numpy's PCG64 seeded by a tuple, and X is drawn in
independent chunks of ``CHUNK_ROWS`` tokens, so any token range can be
regenerated alone (the oracle can check a sample of tokens without holding X).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Iterator, Optional, Sequence, Tuple

import numpy as np

CHUNK_ROWS = 8192

# Cluster starts reported for LLaMA-7B layer 2 (input width 4096).
LLAMA7B_CLUSTER_STARTS = (2100, 3218, 3853)


@dataclass(frozen=True)
class LayerSpec:
    """Shape, distribution and quantizer settings of one synthetic layer."""

    name: str
    m: int                      # output features = rows of W
    n: int                      # input features = columns of W and of X
    N: int                      # calibration tokens = rows of X
    x_dtype: str = "bf16"       # "bf16" or "f32"
    group: int = 128
    avg_bits: int = 2
    lam: float = 0.1
    n_tau: int = 50
    seed: int = 0
    w_std: float = 0.02
    # Salient weight columns: either `n_w_salient` seeded columns anywhere, or
    # contiguous clusters of `cluster_width` columns at `cluster_starts`.
    n_w_salient: int = 0
    cluster_starts: Tuple[int, ...] = ()
    cluster_width: int = 16
    w_scale: float = 6.0
    # Activation outlier columns (drawn inside the clusters when there are any).
    n_x_outliers: int = 0
    x_scale: float = 25.0

    @property
    def k(self) -> int:
        return self.n // self.group

    @property
    def params(self) -> int:
        return self.m * self.n

    def replace(self, **kw) -> "LayerSpec":
        return dataclasses.replace(self, **kw)


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([int(v) for v in key])


def scaled_cluster_starts(n: int) -> Tuple[int, ...]:
    """The LLaMA-7B cluster starts rescaled to an input width of n."""
    return tuple(int(s * n // 4096) for s in LLAMA7B_CLUSTER_STARTS)


def salient_columns(spec: LayerSpec) -> np.ndarray:
    if spec.cluster_starts:
        cols = [np.arange(s, min(s + spec.cluster_width, spec.n)) for s in spec.cluster_starts]
        return np.unique(np.concatenate(cols)).astype(np.int64)
    if spec.n_w_salient:
        return np.sort(_rng(spec.seed, 10).choice(spec.n, spec.n_w_salient, replace=False)).astype(np.int64)
    return np.zeros(0, np.int64)


def outlier_columns(spec: LayerSpec) -> np.ndarray:
    if not spec.n_x_outliers:
        return np.zeros(0, np.int64)
    pool = salient_columns(spec) if spec.cluster_starts else np.arange(spec.n)
    cnt = min(spec.n_x_outliers, pool.size)
    return np.sort(_rng(spec.seed, 11).choice(pool, cnt, replace=False)).astype(np.int64)


def make_weight(spec: LayerSpec) -> np.ndarray:
    """W, float32 [m, n] row-major."""
    w = _rng(spec.seed, 0).standard_normal((spec.m, spec.n), dtype=np.float32)
    w *= np.float32(spec.w_std)
    cols = salient_columns(spec)
    if cols.size:
        w[:, cols] *= np.float32(spec.w_scale)
    return w


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def activation_chunk(spec: LayerSpec, chunk: int) -> np.ndarray:
    """Tokens [chunk*CHUNK_ROWS, ...) of X: float32 values, or uint16 bf16 bits."""
    r0 = chunk * CHUNK_ROWS
    rows = min(CHUNK_ROWS, spec.N - r0)
    if rows <= 0:
        raise IndexError("chunk out of range")
    x = _rng(spec.seed, 1, chunk).standard_normal((rows, spec.n), dtype=np.float32)
    cols = outlier_columns(spec)
    if cols.size:
        x[:, cols] *= np.float32(spec.x_scale)
    if spec.x_dtype == "bf16":
        return f32_to_bf16_bits(x)
    if spec.x_dtype == "f32":
        return x
    raise ValueError(spec.x_dtype)


def n_chunks(spec: LayerSpec) -> int:
    return (spec.N + CHUNK_ROWS - 1) // CHUNK_ROWS


def iter_activation_chunks(spec: LayerSpec) -> Iterator[np.ndarray]:
    for c in range(n_chunks(spec)):
        yield activation_chunk(spec, c)


def make_activations(spec: LayerSpec, out: Optional[np.ndarray] = None) -> np.ndarray:
    """All of X, [N, n]: uint16 bf16 bits for x_dtype 'bf16', float32 for 'f32'.

    `out` may be a preallocated (e.g. pinned, via torch) array of that shape and dtype.
    """
    dt = np.uint16 if spec.x_dtype == "bf16" else np.float32
    if out is None:
        out = np.empty((spec.N, spec.n), dtype=dt)
    for c in range(n_chunks(spec)):
        blk = activation_chunk(spec, c)
        out[c * CHUNK_ROWS: c * CHUNK_ROWS + blk.shape[0]] = blk
    return out


def activations_f64(spec: LayerSpec, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """X (or the given token rows of X) widened exactly to float64."""
    if rows is None:
        x = make_activations(spec)
        return (bf16_bits_to_f32(x) if spec.x_dtype == "bf16" else x).astype(np.float64)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, spec.n), dtype=np.float64)
    chunks = rows // CHUNK_ROWS
    for c in np.unique(chunks):
        sel = np.nonzero(chunks == c)[0]
        blk = activation_chunk(spec, int(c))
        blk = bf16_bits_to_f32(blk) if spec.x_dtype == "bf16" else blk
        out[sel] = blk[rows[sel] - c * CHUNK_ROWS]
    return out


# ---------------------------------------------------------------------------
# The workloads. Shapes follow LLaMA linears; tokens follow 128 x 2048.
# ---------------------------------------------------------------------------
CALIB_TOKENS = 128 * 2048

TINY = LayerSpec(name="tiny_256x512", m=256, n=512, N=2048, x_dtype="f32", group=128, avg_bits=2,
                 seed=0, n_w_salient=4, w_scale=8.0, n_x_outliers=2, x_scale=20.0)

Q_PROJ_7B = LayerSpec(name="llama7b_q_proj_4096x4096", m=4096, n=4096, N=CALIB_TOKENS, x_dtype="bf16",
                      group=128, avg_bits=2, seed=1, cluster_starts=LLAMA7B_CLUSTER_STARTS,
                      n_x_outliers=8)

DOWN_PROJ_7B = LayerSpec(name="llama7b_down_proj_4096x11008", m=4096, n=11008, N=CALIB_TOKENS,
                         x_dtype="bf16", group=128, avg_bits=3, seed=2,
                         cluster_starts=scaled_cluster_starts(11008), n_x_outliers=16)

UP_PROJ_13B = LayerSpec(name="llama13b_up_proj_13824x5120", m=13824, n=5120, N=CALIB_TOKENS,
                        x_dtype="bf16", group=128, avg_bits=2, seed=3,
                        cluster_starts=scaled_cluster_starts(5120), n_x_outliers=10)

def up_proj_13b(group: int) -> LayerSpec:
    """The 13B up_proj layer at another group size (same weights and tokens)."""
    return UP_PROJ_13B.replace(name=f"llama13b_up_proj_13824x5120_g{group}", group=group)


WORKLOADS = {s.name: s for s in (TINY, Q_PROJ_7B, DOWN_PROJ_7B, UP_PROJ_13B, up_proj_13b(64), up_proj_13b(32))}


# The 7B sweep: per block q,k,v,o (4096x4096), gate,up (11008 out x 4096 in), down (4096 out x 11008 in).
SWEEP_LAYERS = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))


def sweep_spec(block: int, layer: int, N: int = CALIB_TOKENS) -> LayerSpec:
    name, m, n = SWEEP_LAYERS[layer]
    return LayerSpec(name=f"llama7b_block{block}_{name}", m=m, n=n, N=N, x_dtype="bf16", group=128,
                     avg_bits=2, seed=1000 * block + layer, cluster_starts=scaled_cluster_starts(n),
                     n_x_outliers=8 if n == 4096 else 16)


def device_layer(spec: LayerSpec, device="cuda", chunk_rows: int = 16384):
    """W (float32 [m, n]) and X (bf16 [N, n]) of a layer drawn directly on the device
    with torch's generator, seeded by spec.seed: the same recipe as make_weight /
    make_activations (N(0, w_std^2) weights with the salient columns scaled,
    N(0, 1) tokens with the outlier columns scaled, rounded once to bf16), but
    another random stream. The 7B sweep uses it, where hundreds of layers with
    gigabytes of tokens each would take hours to draw on the host; copy a
    layer's tensors to the host to give the same values to the oracle.
    """
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(spec.seed))
    W = torch.randn((spec.m, spec.n), generator=g, device=device, dtype=torch.float32) * spec.w_std
    cols = torch.from_numpy(salient_columns(spec)).to(device)
    if cols.numel():
        W[:, cols] *= spec.w_scale
    X = torch.empty((spec.N, spec.n), dtype=torch.bfloat16, device=device)
    ocols = torch.from_numpy(outlier_columns(spec)).to(device)
    for r0 in range(0, spec.N, chunk_rows):
        r1 = min(spec.N, r0 + chunk_rows)
        x = torch.randn((r1 - r0, spec.n), generator=g, device=device, dtype=torch.float32)
        if ocols.numel():
            x[:, ocols] *= spec.x_scale
        X[r0:r1] = x.to(torch.bfloat16)
    return W, X
