"""The 7B sweep's layers: inputs drawn on the device by synthetic.device_layer
(per-layer seed 1000 block + layer), quantized by the whole path, checked against
the oracle on sampled layers of each shape with a reduced token count (the full
262144-token versions of these shapes are the full-size tests of the q_proj and
down_proj workloads).
"""
import numpy as np
import pytest
import torch

from oracle import slim_oracle as O
from post_weight_quantization_hessian_b200 import slim
from post_weight_quantization_hessian_b200 import synthetic as syn
from parity_util import KL_ATOL, compare_sqc, order_ok, pstar_ok

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("block, layer", [(0, 0), (7, 4), (31, 6)])
def test_sweep_layer(block, layer):
    spec = syn.sweep_spec(block, layer, N=4096)
    Wd, Xd = syn.device_layer(spec, "cuda")
    W = Wd.cpu().numpy()
    X = Xd.float().cpu().numpy().astype(np.float64)
    # the recipe: outlier channels inside the weight clusters, x25; cluster columns x6
    ocols = syn.outlier_columns(spec)
    assert np.abs(X[:, ocols]).mean() > 10 * np.abs(np.delete(X, ocols, axis=1)).mean()
    d = slim.slim_quantize_layer_ex(Wd, Xd, spec.group, spec.avg_bits, spec.lam, spec.n_tau)
    g = {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    np.testing.assert_allclose(g["h"], O.hinv_diag(g["H"]), rtol=1e-9)
    S_chain = O.group_salience(W, g["h"], spec.group)
    np.testing.assert_allclose(g["S"], S_chain, rtol=1e-12)
    assert order_ok(g["order"], S_chain, rel=1e-12) == 0
    sba = O.sba_search(W, X, g["order"], spec.group, spec.avg_bits, reassociate=True)
    dev = np.abs(g["kl"] - sba.kl).max()
    print(f"sweep block {block} layer {spec.name}: max |dKL| {dev:.2e}, p* {g['p_star']} / {sba.p_star}")
    assert dev <= KL_ATOL
    if pstar_ok(g["p_star"], sba.kl, g["kl"]):
        assert np.array_equal(g["bits"], sba.bits.astype(np.uint8))
    rows = np.sort(np.random.default_rng(block).choice(spec.m, 256, replace=False))
    sq = O.sqc_calibrate(W[rows], g["h"], g["bits"], spec.group, spec.lam, spec.n_tau)
    agree, tmis = compare_sqc(g["codes"][rows], g["scale"][rows], g["zero"][rows], g["tau_idx"][rows], sq, g["bits"],
                              spec.group, spec.avg_bits)
    assert agree >= 0.9999 and tmis == 0
