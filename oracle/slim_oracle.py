"""Float64 CPU oracle for the SliM-LLM per-layer quantize path.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg may import this module. The library's product path never calls it,
and it shares no code with the CUDA path.

It restates, plainly and slowly, what SliM-LLM computes for one linear layer
(W: out x in, X: tokens x in). Sources are the pages about the method:

* [P1] rkmt.cn, "【ICML 2025】SliM-LLM 论文解读" (Chinese write-up of the paper),
  section 核心设计 (组件一 SBA, 组件二 SQC), section FAQ.
* [P2] atlas.scime.ai summary of "SliM-LLM: Salience-Driven Mixed-Precision
  Quantization for Large Language Models", section Approach.
* [P3] briefgpt.xyz, the arXiv 2405.14917 abstract.

Steps (each function below names the passage it follows):
  hessian       H = 2 X^T X                                  [P1 组件一 SBA]
  hinv_diag     h_j = [(H + damp I)^-1]_jj via Cholesky      [P1 组件一 SBA, delta formula]
  salience      delta_ij = w_ij^2 / h_j^2, group means, sort [P1 组件一 SBA; P2 Approach]
  sba_search    balanced promote/demote search, output KL     [P1 组件一 SBA; P2 Approach]
  sqc_calibrate 3-sigma mask, tau grid, weighted l2          [P1 组件二 SQC; P2 Approach; P3]
  pack_codes    group-structured bitstream, no bitmap         [P1 FAQ "零额外存储"]

Where the pages are silent or garbled, the reading taken is stated at the step
(dead columns, damping, population sigma, float zero-point, clipping form of
tau, linspace grid, loss form, RTN during the search, KL direction, ties).

Parity pins: every function here is checked by tests/test_oracle_*.py against
closed forms, hand-derived values, library routines or brute force.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Iterable, List, Optional, Sequence, Union

import numpy as np
from scipy.linalg import solve_triangular

ArrayOrChunks = Union[np.ndarray, Iterable[np.ndarray]]

DAMP_ALPHA = 0.01


class NotPositiveDefinite(ValueError):
    """The damped Hessian has no Cholesky factor."""


def _as_chunks(X: ArrayOrChunks) -> Iterable[np.ndarray]:
    if isinstance(X, np.ndarray):
        return (X,)
    return X


# ---------------------------------------------------------------------------
# Hessian
# ---------------------------------------------------------------------------
def hessian(X: ArrayOrChunks) -> np.ndarray:
    """H = 2 X^T X, float64 [n, n].

    [P1 组件一 SBA]: the layer Hessian is approximated from calibration
    activations, without backpropagation. X may be given as token chunks; H is a
    sum over tokens, so adding chunk contributions is the same sum.
    """
    H = None
    for x in _as_chunks(X):
        x = np.asarray(x, dtype=np.float64)
        part = 2.0 * (x.T @ x)
        H = part if H is None else H + part
    return H


# ---------------------------------------------------------------------------
# diag(H^-1)
# ---------------------------------------------------------------------------
def damped(H: np.ndarray, alpha: float = DAMP_ALPHA) -> np.ndarray:
    """Dead-column fix then diagonal damping.

    Pages silent. Readings: a column with H_jj == 0 (an input channel that never
    fires) gets H_jj = 1; then alpha * mean(diag H) is added to the diagonal,
    the damping of the GPTQ backbone that SliM-LLM plugs into [P1 核心设计].
    """
    Hd = np.array(H, dtype=np.float64, copy=True)
    d = np.diagonal(Hd).copy()
    dead = d == 0.0
    d[dead] = 1.0
    np.fill_diagonal(Hd, d)
    damp = alpha * float(np.mean(np.diagonal(Hd)))
    Hd[np.diag_indices_from(Hd)] += damp
    return Hd


def hinv_diag(H: np.ndarray, alpha: float = DAMP_ALPHA) -> np.ndarray:
    """h_j = [H_d^-1]_jj for the damped Hessian H_d, float64 [n].

    The salience formula needs the inverse-Hessian diagonal [P1 组件一 SBA].
    Computed as H_d = L L^T (Cholesky), then h_j = sum_i (L^-1)_ij^2, because
    H_d^-1 = L^-T L^-1.
    """
    Hd = damped(H, alpha)
    try:
        L = np.linalg.cholesky(Hd)
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e)) from e
    Linv = solve_triangular(L, np.eye(L.shape[0]), lower=True)
    return np.sum(Linv * Linv, axis=0)


# ---------------------------------------------------------------------------
# Salience
# ---------------------------------------------------------------------------
def element_salience(W: np.ndarray, h: np.ndarray) -> np.ndarray:
    """delta_ij = w_ij^2 / [H^-1]_jj^2.

    [P1 组件一 SBA] prints the SparseGPT-style elimination error with the
    denominator squared; that form is taken as printed.
    """
    W = np.asarray(W, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    return (W * W) / (h * h)[None, :]


def group_salience(W: np.ndarray, h: np.ndarray, group: int) -> np.ndarray:
    """S_c = mean of delta over all rows and the columns of group c, float64 [k].

    [P2 Approach]: bit-widths are allocated per group by average group salience.
    Groups are consecutive runs of `group` input columns [P1 核心设计].
    """
    d = element_salience(W, h)
    m, n = d.shape
    k = n // group
    return np.array([d[:, c * group:(c + 1) * group].mean() for c in range(k)])


def salience_order(S: np.ndarray) -> np.ndarray:
    """Groups by descending salience; equal salience keeps the lower index first."""
    return np.argsort(-np.asarray(S), kind="stable").astype(np.int64)


# ---------------------------------------------------------------------------
# Bit allocation (SBA)
# ---------------------------------------------------------------------------
def allocation(order: Sequence[int], avg_bits: int, p: int) -> np.ndarray:
    """Bits per group for p promotions.

    [P1 组件一 SBA]: the p most salient groups get avg_bits+1, the p least
    salient get avg_bits-1, so |G_{N-1}| = |G_{N+1}| and the average stays
    avg_bits. p <= k/2 keeps the two sets apart.
    """
    order = np.asarray(order)
    k = order.size
    if not 0 <= p <= k // 2:
        raise ValueError("p out of [0, k/2]")
    bits = np.full(k, avg_bits, dtype=np.int64)
    bits[order[:p]] = avg_bits + 1
    if p:
        bits[order[k - p:]] = avg_bits - 1
    return bits


# ---------------------------------------------------------------------------
# The asymmetric uniform quantizer
# ---------------------------------------------------------------------------
def minmax_params(w: np.ndarray, b: int):
    """Per-row min-max scale and zero of a [rows, g] block at b bits.

    Asymmetric uniform quantizer with per-group scale and zero [P2 Approach].
    Reading: the zero-point is kept as a float (not rounded). A row whose
    values are all equal is degenerate: scale 1, zero -lo (exact).
    Returns lo, hi, s0, z0, degenerate-mask.
    """
    w = np.asarray(w, dtype=np.float64)
    qmax = float(2 ** b - 1)
    lo = w.min(axis=1)
    hi = w.max(axis=1)
    deg = hi == lo
    s0 = np.where(deg, 1.0, (hi - lo) / qmax)
    z0 = np.where(deg, -lo, -lo / s0)
    return lo, hi, s0, z0, deg


def fake_quant(w: np.ndarray, s: np.ndarray, z: np.ndarray, b: int):
    """q = clamp(rint(w / s + z), 0, 2^b - 1) (rint: half to even); w_hat = s (q - z)."""
    w = np.asarray(w, dtype=np.float64)
    qmax = float(2 ** b - 1)
    s = np.asarray(s, dtype=np.float64)[:, None]
    z = np.asarray(z, dtype=np.float64)[:, None]
    q = np.minimum(np.maximum(np.rint(w / s + z), 0.0), qmax)
    return q, s * (q - z)


def rtn_dequant(W: np.ndarray, bits: Sequence[int], group: int) -> np.ndarray:
    """Round-to-nearest min-max quantize/dequantize of W with per-group bits (tau = 1).

    Reading: while SBA scores a candidate allocation it uses the plain min-max
    quantizer; the tau search of SQC is the separate, local step [P1 核心设计].
    """
    W = np.asarray(W, dtype=np.float64)
    out = np.empty_like(W)
    for c, b in enumerate(bits):
        blk = W[:, c * group:(c + 1) * group]
        lo, hi, s0, z0, deg = minmax_params(blk, int(b))
        _, wh = fake_quant(blk, s0, z0, int(b))
        wh[deg] = blk[deg]
        out[:, c * group:(c + 1) * group] = wh
    return out


# ---------------------------------------------------------------------------
# Output KL
# ---------------------------------------------------------------------------
def log_softmax(Z: np.ndarray) -> np.ndarray:
    Z = np.asarray(Z, dtype=np.float64)
    mx = Z.max(axis=1, keepdims=True)
    return Z - mx - np.log(np.exp(Z - mx).sum(axis=1, keepdims=True))


def kl_per_token(Y: np.ndarray, Yq: np.ndarray, ref=None) -> np.ndarray:
    """KL(softmax(y_t) || softmax(yq_t)) for every token t (row).

    [P1 组件一 SBA] scores an allocation by the KL divergence of the layer
    outputs. Reading: softmax over the output features, direction
    KL(full precision || quantized). `ref` may carry (log_softmax(Y), its
    exp) computed once for several Yq against the same Y: the same values.
    """
    lp, p = ref if ref is not None else kl_reference(Y)
    lq = log_softmax(Yq)
    return np.sum(p * (lp - lq), axis=1)


def kl_reference(Y: np.ndarray):
    """log_softmax(Y) and softmax(Y) = exp(log_softmax(Y)), the full-precision side of kl_per_token."""
    lp = log_softmax(Y)
    return lp, np.exp(lp)


# ---------------------------------------------------------------------------
# SBA search
# ---------------------------------------------------------------------------
@dataclass
class SBAResult:
    kl: np.ndarray          # [P] mean KL per candidate p
    p_star: int
    bits: np.ndarray        # [k]
    margin: float           # (second best - best) / best, inf if P == 1


def sba_candidates(k: int) -> int:
    """Number of candidates: p = 0 .. floor(k/2). p = 0 is uniform precision.

    [P1 组件一 SBA]: the search range is [0, k/2]; for LLaMA-7B (k = 32) that
    is 16 promote/demote moves after the uniform start.
    """
    return k // 2 + 1


def mse_per_token(Y: np.ndarray, Yq: np.ndarray) -> np.ndarray:
    """Mean over the output features of (yq_t - y_t)^2 for every token t (row).

    The objective SBA's KL is compared against in the method's ablation
    [P2 Measured effects: KL divergence rather than MSE as the SBA objective].
    """
    D = np.asarray(Yq, dtype=np.float64) - np.asarray(Y, dtype=np.float64)
    return np.mean(D * D, axis=1)


def sba_search(W: np.ndarray, X: ArrayOrChunks, order: Sequence[int], group: int, avg_bits: int,
               reassociate: bool = False, objective: str = "kl") -> SBAResult:
    """Pick p* = argmin_p mean_t KL(softmax(x_t W^T) || softmax(x_t W_p^T)).

    [P1 组件一 SBA], [P2 Approach]: candidates are the balanced allocations
    that promote the p most salient groups and demote the p least salient.
    Every p in [0, k/2] is scored (the double-pointer walk visits them all), and
    the smallest p reaching the least KL wins.

    `objective="mse"` scores a candidate by mse_per_token instead (the ablation
    of [P2 Measured effects]). `order` may be any permutation of the groups:
    the salience order is the method; position order (head-tail) and a random
    permutation are the allocations of the ablation [P1 Fig. 5 caption].

    `reassociate=True` computes X W_p^T as X W_{p-1}^T plus the product of the
    two changed column groups, which is the same sum regrouped.
    """
    if objective not in ("kl", "mse"):
        raise ValueError("objective must be 'kl' or 'mse'")
    W = np.asarray(W, dtype=np.float64)
    k = W.shape[1] // group
    P = sba_candidates(k)
    allocs = [allocation(order, avg_bits, p) for p in range(P)]

    def dequant(p):
        # a candidate's quantized weights, made when used: all P of them at
        # once would not fit in host memory for the larger layers
        return rtn_dequant(W, allocs[p], group)

    kl_sum = np.zeros(P)
    ntok = 0
    for x in _as_chunks(X):
        x = np.asarray(x, dtype=np.float64)
        Y = x @ W.T
        ntok += x.shape[0]
        if not reassociate:
            for p in range(P):
                Yq = x @ dequant(p).T
                kl_sum[p] += (kl_per_token(Y, Yq) if objective == "kl" else mse_per_token(Y, Yq)).sum()
        else:
            ref = kl_reference(Y) if objective == "kl" else None   # the same for every candidate of this chunk
            score = (lambda Yq: kl_per_token(Y, Yq, ref)) if objective == "kl" else (lambda Yq: mse_per_token(Y, Yq))
            Yq = x @ dequant(0).T
            kl_sum[0] += score(Yq).sum()
            for p in range(1, P):
                for c in (order[p - 1], order[k - p]):
                    # candidates p-1 and p differ only on group c; the quantizer
                    # is per group, so its block quantized at either bit width is
                    # what the whole-matrix dequantization would hold there
                    cols = slice(c * group, (c + 1) * group)
                    blk = W[:, cols]
                    d = rtn_dequant(blk, [allocs[p][c]], group) - rtn_dequant(blk, [allocs[p - 1][c]], group)
                    Yq = Yq + x[:, cols] @ d.T
                kl_sum[p] += score(Yq).sum()
    kl = kl_sum / ntok
    p_star = int(np.argmin(kl))
    srt = np.sort(kl)
    margin = float((srt[1] - srt[0]) / max(srt[0], 1e-300)) if P > 1 else float("inf")
    return SBAResult(kl=kl, p_star=p_star, bits=allocs[p_star], margin=margin)


# ---------------------------------------------------------------------------
# SQC: salience-weighted quantizer calibration
# ---------------------------------------------------------------------------
def tau_grid(lam: float, n_tau: int) -> np.ndarray:
    """n_tau candidates spread linearly over [1 - lam, 1 + lam], both ends included.

    [P1 组件二 SQC]: tau is taken linearly in [1 - lambda, 1 + lambda] with
    lambda = 0.1 and n = 50. n_tau = 1 means tau = 1 (plain min-max).
    """
    lam = float(lam)
    if n_tau == 1:
        return np.ones(1)
    t = np.arange(n_tau, dtype=np.float64)
    return (1.0 - lam) + 2.0 * lam * t / float(n_tau - 1)


def salient_mask(w: np.ndarray) -> np.ndarray:
    """Rows of a [rows, g] block: w < mu - 3 sigma or w > mu + 3 sigma (strict).

    [P1 组件二 SQC] 3-sigma mask. Reading: sigma is the population standard
    deviation of the group.
    """
    w = np.asarray(w, dtype=np.float64)
    g = w.shape[1]
    mu = w.sum(axis=1) / g
    var = ((w - mu[:, None]) ** 2).sum(axis=1) / g
    sd = np.sqrt(var)
    return (w < (mu - 3.0 * sd)[:, None]) | (w > (mu + 3.0 * sd)[:, None])


def sqc_error(w: np.ndarray, delta: np.ndarray, mask: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """Salience-weighted l2 reconstruction error per row.

    [P1 组件二 SQC] minimise the l2 reconstruction error with salient and
    non-salient weights sharing one quantizer; [P3] weights it by element-wise
    salience, balancing salient information against overall error. Reading:
    E = mean over the masked set of delta e^2 + mean over the rest of delta e^2
    (the first term is absent when the mask is empty).
    """
    e2 = delta * (w - wq) ** 2
    ns = mask.sum(axis=1)
    nu = (~mask).sum(axis=1)
    es = np.where(mask, e2, 0.0).sum(axis=1)
    eu = np.where(mask, 0.0, e2).sum(axis=1)
    out = eu / nu
    has = ns > 0
    out[has] += es[has] / ns[has]
    return out


@dataclass
class SQCResult:
    codes: np.ndarray       # [m, n] integer codes
    scale: np.ndarray       # [m, k] float32
    zero: np.ndarray        # [m, k] float32
    tau_idx: np.ndarray     # [m, k] chosen tau index
    scale64: np.ndarray     # [m, k] float64 (before storage rounding)
    zero64: np.ndarray
    margin: np.ndarray      # [m, k] relative gap best -> second best error (inf if one tau)
    mask_rate: float        # fraction of weights in the 3-sigma masks


def sqc_group(w: np.ndarray, h: np.ndarray, b: int, lam: float, n_tau: int):
    """SQC for one group of columns: w is [rows, g], h the g inverse-Hessian entries.

    Returns (codes [rows, g], s [rows], z [rows], t* [rows], margin [rows],
    masked count). The per-row steps are those of sqc_calibrate below.
    """
    taus = tau_grid(lam, n_tau)
    m = w.shape[0]
    delta = element_salience(w, h)
    mask = salient_mask(w)
    lo, hi, s0, z0, deg = minmax_params(w, b)
    errs = np.empty((m, n_tau))
    for t, tau in enumerate(taus):
        s = tau * s0
        _, wq = fake_quant(w, s, z0, b)
        errs[:, t] = sqc_error(w, delta, mask, wq)
    best = np.argmin(errs, axis=1)
    best[deg] = 0
    s_best = taus[best] * s0
    s_best[deg] = 1.0
    q, _ = fake_quant(w, s_best, z0, b)
    q[deg] = 0.0
    margin = np.full(m, np.inf)
    if n_tau > 1:
        srt = np.sort(errs, axis=1)
        gap = (srt[:, 1] - srt[:, 0]) / np.maximum(srt[:, 0], 1e-300)
        gap[deg] = np.inf
        margin = gap
    return q.astype(np.int64), s_best, np.asarray(z0, dtype=np.float64), best, margin, int(mask.sum())


def sqc_calibrate(W: np.ndarray, h: np.ndarray, bits: Sequence[int], group: int, lam: float,
                  n_tau: int) -> SQCResult:
    """Per (row, group): 3-sigma mask, then the tau with least weighted error.

    [P1 组件二 SQC]: scale/zero candidates are the min-max quantizer with tau
    applied; reading (clipping): the range becomes [tau lo, tau hi], so
    s = tau s0 and the zero-point stays z0 = -lo / s0. The first tau (lowest
    index) with the least error wins. Degenerate rows (all equal) take tau
    index 0 with scale 1, zero -lo, codes 0.
    """
    W = np.asarray(W, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    m, n = W.shape
    k = n // group
    codes = np.zeros((m, n), dtype=np.int64)
    scale64 = np.zeros((m, k))
    zero64 = np.zeros((m, k))
    tidx = np.zeros((m, k), dtype=np.int64)
    margin = np.full((m, k), np.inf)
    masked = 0
    for c in range(k):
        cols = slice(c * group, (c + 1) * group)
        q, s_best, z0, best, mg, nm = sqc_group(W[:, cols], h[cols], int(bits[c]), lam, n_tau)
        masked += nm
        codes[:, cols] = q
        scale64[:, c] = s_best
        zero64[:, c] = z0
        tidx[:, c] = best
        margin[:, c] = mg
    return SQCResult(codes=codes, scale=scale64.astype(np.float32), zero=zero64.astype(np.float32),
                     tau_idx=tidx, scale64=scale64, zero64=zero64, margin=margin,
                     mask_rate=masked / float(m * n))


def dequant_codes(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray, group: int) -> np.ndarray:
    """w_hat = scale (q - zero) with the stored per-(row, group) scale and zero."""
    s = np.repeat(np.asarray(scale, dtype=np.float64), group, axis=1)
    z = np.repeat(np.asarray(zero, dtype=np.float64), group, axis=1)
    return s * (np.asarray(codes, dtype=np.float64) - z)


# ---------------------------------------------------------------------------
# GPTQ backbone: column-by-column quantization with error compensation
# ---------------------------------------------------------------------------
def gptq_factor(H: np.ndarray, alpha: float = DAMP_ALPHA):
    """U upper triangular with H_d^-1 = U^T U (the Cholesky factor of the damped
    inverse Hessian), and the diagonal of H_d^-1.

    GPTQ's compensation uses the rows of U; H_d is the damped Hessian of the
    rest of the path (dead columns set to 1, then alpha * mean diagonal).
    """
    Hd = damped(H, alpha)
    try:
        Hinv = np.linalg.inv(Hd)
        U = np.linalg.cholesky(Hinv).T
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e)) from e
    return U, np.diagonal(Hinv).copy()


@dataclass
class GPTQResult:
    codes: np.ndarray       # [m, n] integer codes
    scale: np.ndarray       # [m, k] float32
    zero: np.ndarray        # [m, k] float32
    tau_idx: np.ndarray     # [m, k] chosen tau index
    scale64: np.ndarray
    zero64: np.ndarray
    margin: np.ndarray      # [m, k] SQC's relative gap best -> second best error
    Wq: np.ndarray          # [m, n] float64 dequantized weights
    h: np.ndarray           # [n] diag of the damped inverse Hessian
    snapshot: Optional[np.ndarray] = None


def gptq_quantize(W: np.ndarray, H: np.ndarray, bits: Sequence[int], group: int, lam: float, n_tau: int,
                  alpha: float = DAMP_ALPHA, snapshot_after: Optional[int] = None) -> GPTQResult:
    """SliM-LLM inside the GPTQ layer loop [P1 核心设计: the GPTQ layer-wise
    quantization skeleton with the two salience-driven components inserted; P1
    FAQ]: columns are quantized in order; when a group's first column is
    reached, SQC calibrates the group's quantizer (bits from SBA, 3-sigma mask,
    tau search) on the group's weights as the earlier columns' compensation has
    left them; each column is then rounded with its group's quantizer and its
    error, divided by U_jj, is spread over the later columns along row j of U.

    Readings (the pages name GPTQ but do not restate it): columns in their
    natural order (no reordering by activation size); a group's scale and zero
    are fixed when its first column is reached; the element salience inside SQC
    uses the current weights and diag(H_d^-1); dead columns only get H_jj = 1.
    `snapshot_after=j` also returns the working weights right after column j.
    """
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    k = n // group
    U, hd = gptq_factor(H, alpha)
    Wk = W.copy()
    codes = np.zeros((m, n), dtype=np.int64)
    Wq = np.zeros((m, n))
    scale64 = np.zeros((m, k))
    zero64 = np.zeros((m, k))
    tidx = np.zeros((m, k), dtype=np.int64)
    margin = np.full((m, k), np.inf)
    snap = None
    for j in range(n):
        c = j // group
        b = int(bits[c])
        if j % group == 0:
            cols = slice(c * group, (c + 1) * group)
            _, s_c, z_c, t_c, mg, _ = sqc_group(Wk[:, cols], hd[cols], b, lam, n_tau)
            scale64[:, c], zero64[:, c], tidx[:, c], margin[:, c] = s_c, z_c, t_c, mg
        q, wq = fake_quant(Wk[:, j:j + 1], scale64[:, c], zero64[:, c], b)
        codes[:, j] = q[:, 0].astype(np.int64)
        Wq[:, j] = wq[:, 0]
        err = (Wk[:, j] - wq[:, 0]) / U[j, j]
        Wk[:, j + 1:] -= np.outer(err, U[j, j + 1:])
        if snapshot_after == j:
            snap = Wk.copy()
    return GPTQResult(codes=codes, scale=scale64.astype(np.float32), zero=zero64.astype(np.float32), tau_idx=tidx,
                      scale64=scale64, zero64=zero64, margin=margin, Wq=Wq, h=hd, snapshot=snap)


# ---------------------------------------------------------------------------
# Packed storage
# ---------------------------------------------------------------------------
def row_words(n: int, avg_bits: int) -> int:
    return n * avg_bits // 32


def pack_codes(codes: np.ndarray, bits: Sequence[int], group: int, avg_bits: int) -> np.ndarray:
    """Group-structured bitstream, no bitmap or index [P1 FAQ].

    Layout (the pages leave it open): each row is a little-endian bit stream of
    n * avg_bits bits; group c contributes its g codes of bits_c bits each, in
    column order, least significant bit first, after the groups before it. The
    stream is cut into uint32 words. Since sum(bits) = k * avg_bits, every row
    has the same n * avg_bits / 32 words.
    """
    codes = np.asarray(codes, dtype=np.int64)
    m, n = codes.shape
    rw = row_words(n, avg_bits)
    out = np.zeros((m, rw), dtype=np.uint64)
    for i in range(m):
        pos = 0
        for c, b in enumerate(bits):
            for j in range(c * group, (c + 1) * group):
                v = int(codes[i, j])
                for bit in range(int(b)):
                    if (v >> bit) & 1:
                        out[i, pos // 32] |= np.uint64(1 << (pos % 32))
                    pos += 1
        assert pos == rw * 32
    return out.astype(np.uint32)


def unpack_codes(words: np.ndarray, bits: Sequence[int], group: int, n: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint32)
    m = words.shape[0]
    out = np.zeros((m, n), dtype=np.int64)
    for i in range(m):
        pos = 0
        for c, b in enumerate(bits):
            for j in range(c * group, (c + 1) * group):
                v = 0
                for bit in range(int(b)):
                    if (int(words[i, pos // 32]) >> (pos % 32)) & 1:
                        v |= 1 << bit
                    pos += 1
                out[i, j] = v
    return out


def pack_codes_fast(codes: np.ndarray, bits: Sequence[int], group: int, avg_bits: int) -> np.ndarray:
    """The same layout as pack_codes, vectorised over rows (for large layers)."""
    codes = np.asarray(codes, dtype=np.uint64)
    m, n = codes.shape
    rw = row_words(n, avg_bits)
    out = np.zeros((m, rw + 1), dtype=np.uint64)
    pos = 0
    for c, b in enumerate(bits):
        for j in range(c * group, (c + 1) * group):
            w, s = divmod(pos, 32)
            v = codes[:, j] << np.uint64(s)
            out[:, w] |= v & np.uint64(0xFFFFFFFF)
            out[:, w + 1] |= v >> np.uint64(32)
            pos += int(b)
    return out[:, :rw].astype(np.uint32)


def dequant_matmul(words: np.ndarray, bits: Sequence[int], scale: np.ndarray, zero: np.ndarray, group: int,
                   x: np.ndarray) -> np.ndarray:
    """y = x W_hat^T for the packed layer: the inference product on the stored
    codes (unpacked with the layout of pack_codes), w_hat = scale (q - zero).

    The pages measure this product at inference: mixed 1/2/3-bit groups cost
    token rate against uniform-width GPTQ on current GPU kernels [P1 局限性;
    P2 Limitations: 61.2 vs 83.9 tokens/s]. x is [batch, n]; float64 result.
    """
    words = np.asarray(words, dtype=np.uint32)
    n = np.asarray(x).shape[-1]
    codes = unpack_codes(words, bits, group, n)
    Wq = dequant_codes(codes, scale, zero, group)
    return np.asarray(x, dtype=np.float64) @ Wq.T


# ---------------------------------------------------------------------------
# The whole layer
# ---------------------------------------------------------------------------
@dataclass
class LayerResult:
    H: np.ndarray
    h: np.ndarray
    S: np.ndarray
    order: np.ndarray
    order_margin: np.ndarray     # relative gap between consecutive sorted S
    sba: SBAResult
    sqc: SQCResult
    words: np.ndarray
    kl_final: Optional[float] = None


def quantize_layer(W: np.ndarray, X: Union[np.ndarray, Sequence[np.ndarray]], group: int, avg_bits: int,
                   lam: float = 0.1, n_tau: int = 50, alpha: float = DAMP_ALPHA, reassociate: bool = False,
                   final_kl: bool = False) -> LayerResult:
    """hessian -> hinv_diag -> salience -> sba_search -> sqc_calibrate -> pack.

    The order follows [P1 核心设计]: SBA allocates bits between groups, then
    SQC calibrates each group's quantizer. `X` may be a list of token chunks.
    """
    chunks = [X] if isinstance(X, np.ndarray) else list(X)
    H = hessian(chunks)
    h = hinv_diag(H, alpha)
    S = group_salience(W, h, group)
    order = salience_order(S)
    srt = S[order]
    om = np.abs(srt[:-1] - srt[1:]) / np.maximum(np.abs(srt[:-1]), 1e-300)
    sba = sba_search(W, chunks, order, group, avg_bits, reassociate=reassociate)
    sqc = sqc_calibrate(W, h, sba.bits, group, lam, n_tau)
    words = pack_codes_fast(sqc.codes, sba.bits, group, avg_bits)
    res = LayerResult(H=H, h=h, S=S, order=order, order_margin=om, sba=sba, sqc=sqc, words=words)
    if final_kl:
        Wq = dequant_codes(sqc.codes, sqc.scale64, sqc.zero64, group)
        W64 = np.asarray(W, dtype=np.float64)
        tot, cnt = 0.0, 0
        for x in chunks:
            x = np.asarray(x, dtype=np.float64)
            tot += kl_per_token(x @ W64.T, x @ Wq.T).sum()
            cnt += x.shape[0]
        res.kl_final = tot / cnt
    return res
