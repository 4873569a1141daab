"""GPU parity of the GPTQ backbone (slim_gptq and the layer path with gptq=1)
against the oracle's column-by-column gptq_quantize, through the C ABI.

rkmt.cn write-up, section 核心设计 (GPTQ layer-wise skeleton with SliM-LLM's
components inserted) and FAQ. Both sides run fp64; the GPU applies each
128-column block's errors to the later columns at once (the same sums
regrouped) and derives U from a factorization of the reversed Hessian, so the
working weights differ from the oracle's in the last bits. A code decided at a
rounding tie could then differ and its error would be compensated differently
in the rest of the row; the tests require every code, scale, zero and tau
index to agree except in groups where the oracle's own tau choice is a near
tie (relative gap below 1e-9).
"""
import numpy as np
import pytest
import torch

from oracle import slim_oracle as O
from post_weight_quantization_hessian_b200 import slim
from post_weight_quantization_hessian_b200 import synthetic as syn
from parity_util import balanced_bits, device_inputs, x_f64

pytestmark = pytest.mark.gpu


def compare_gptq(codes_gpu, scale_gpu, zero_gpu, tau_gpu, ref: O.GPTQResult, bits, group, avg_bits):
    m, n = ref.codes.shape
    tau_gpu = np.asarray(tau_gpu).astype(np.int64)
    tmis = tau_gpu != ref.tau_idx
    if tmis.any():
        assert ref.margin[tmis].max() < 1e-9, f"{int(tmis.sum())} tau mismatches, oracle margin {ref.margin[tmis].max():.2e}"
    # rows with a near-tie tau difference are compared up to that group only
    first_bad = np.where(tmis.any(axis=1), np.argmax(tmis, axis=1) * group, n)
    codes = O.unpack_codes(np.asarray(codes_gpu).view(np.uint32), bits, group, n)
    ok = np.arange(n)[None, :] < first_bad[:, None]
    agree = float((codes == ref.codes)[ok].mean())
    okg = np.arange(n // group)[None, :] < (first_bad // group)[:, None]
    np.testing.assert_allclose(np.asarray(scale_gpu)[okg], ref.scale[okg], rtol=1e-6)
    np.testing.assert_allclose(np.asarray(zero_gpu)[okg], ref.zero[okg], rtol=1e-6, atol=1e-30)
    return agree, int(tmis.sum())


CASES = [
    dict(m=96, n=256, group=128, avg_bits=2),
    dict(m=130, n=160, group=32, avg_bits=2),     # a 128-column block and a 32-column tail block
    dict(m=64, n=384, group=64, avg_bits=3),
    dict(m=200, n=512, group=32, avg_bits=2),
]


@pytest.mark.parametrize("kw", CASES)
def test_gptq_stage(kw):
    s = syn.LayerSpec(name="g", N=2000, x_dtype="f32", seed=31, n_w_salient=4, w_scale=6.0, n_x_outliers=2,
                      x_scale=20.0, **kw)
    W = syn.make_weight(s)
    X = x_f64(s, syn.make_activations(s))
    # correlated channels, so the compensation has work to do
    X[:, 1:] = 0.5 * X[:, 1:] + 0.5 * X[:, :-1]
    H = O.hessian(X)
    bits = balanced_bits(s.k, s.avg_bits, s.k // 3, seed=5)
    codes, scale, zero, tau = slim.slim_gptq(torch.from_numpy(W).cuda(), torch.from_numpy(H).cuda(),
                                             torch.from_numpy(bits).cuda(), s.group, s.avg_bits, s.lam, s.n_tau)
    ref = O.gptq_quantize(W, H, bits, s.group, s.lam, s.n_tau)
    agree, tmis = compare_gptq(codes.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), tau.cpu().numpy(), ref,
                               bits, s.group, s.avg_bits)
    print(f"gptq {kw}: code agreement {agree:.6f}, near-tie tau differences {tmis}")
    assert agree == 1.0 or (tmis > 0 and agree >= 0.999)
    # the compensation did something: the codes differ from plain SQC's somewhere
    r = O.sqc_calibrate(W, ref.h, bits, s.group, s.lam, s.n_tau)
    assert (r.codes != ref.codes).any()


def test_gptq_layer_path():
    """slim_quantize_layer_opts with gptq=1: the GPU's own H and bits, then GPTQ's codes
    against the oracle's GPTQ on those."""
    s = syn.LayerSpec(name="gl", m=256, n=512, N=3000, x_dtype="bf16", group=64, avg_bits=2, seed=41,
                      n_w_salient=6, w_scale=6.0, n_x_outliers=3, x_scale=25.0)
    W, Xh, Wd, Xd = device_inputs(s)
    d = slim.slim_quantize_layer_opts(Wd, Xd, s.group, s.avg_bits, s.lam, s.n_tau, gptq=True)
    g = {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    ref = O.gptq_quantize(W, g["H"], g["bits"], s.group, s.lam, s.n_tau)
    agree, tmis = compare_gptq(g["codes"], g["scale"], g["zero"], g["tau_idx"], ref, g["bits"], s.group, s.avg_bits)
    print(f"gptq layer: code agreement {agree:.6f}, near-tie tau differences {tmis}")
    assert agree == 1.0 or (tmis > 0 and agree >= 0.999)
    # error compensation lowers the layer's output error against SQC alone
    X = x_f64(s, Xh)
    sq = O.sqc_calibrate(W, g["h"], g["bits"], s.group, s.lam, s.n_tau)
    Wg = O.dequant_codes(O.unpack_codes(g["codes"].view(np.uint32), g["bits"], s.group, s.n), g["scale"], g["zero"],
                         s.group)
    Ws = O.dequant_codes(sq.codes, sq.scale, sq.zero, s.group)
    eg = np.sum((X @ (Wg - W).T) ** 2)
    es = np.sum((X @ (Ws - W).T) ** 2)
    print(f"gptq layer: output error {eg:.4e} vs SQC alone {es:.4e}")
    assert eg < es
