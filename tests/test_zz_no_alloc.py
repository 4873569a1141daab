"""The allocation-free salience entry point gives slim_salience's results.

slim_salience_noalloc exists for callers that may not allocate device memory:
code inside an engine that owns all device memory through its own pool, code
on a path where cudaMalloc's implicit synchronization is not allowed, or code
whose memory budget is fixed in advance. It keeps its scratch in a fixed array
inside the library instead.

The test calls it through the C ABI twice in a row, with different shapes,
and checks each result against slim_salience with the salience tests'
tolerance (S within 1e-12 relative, identical order). The second call also
shows that nothing from the first call's use of the shared scratch leaks into
its result. It passes alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from post_weight_quantization_hessian_b200 import slim
from post_weight_quantization_hessian_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _inputs(m, n, group, seed):
    spec = syn.LayerSpec(name="noalloc", m=m, n=n, N=1, group=group, seed=seed, n_w_salient=5, w_scale=6.0)
    W = torch.from_numpy(syn.make_weight(spec)).cuda()
    h = torch.from_numpy(np.random.default_rng(seed).uniform(0.2, 2.0, n)).cuda()
    return W, h


def test_noalloc_matches_salience_on_two_calls_in_a_row():
    lib = slim._lib()
    stream = torch.cuda.current_stream().cuda_stream
    for m, n, group, seed in ((4096, 4096, 128, 1), (300, 640, 32, 2)):
        W, h = _inputs(m, n, group, seed)
        k = n // group
        S = torch.full((k,), float("nan"), dtype=torch.float64, device="cuda")
        order = torch.full((k,), -1, dtype=torch.int32, device="cuda")
        rc = lib.slim_salience_noalloc(W.data_ptr(), m, n, h.data_ptr(), group, S.data_ptr(), order.data_ptr(),
                                       stream)
        assert rc == 0, slim.STATUS.get(rc)
        S_ref, order_ref = slim.slim_salience(W, h, group)
        np.testing.assert_allclose(S.cpu().numpy(), S_ref.cpu().numpy(), rtol=1e-12)
        assert np.array_equal(order.cpu().numpy(), order_ref.cpu().numpy())


def test_noalloc_rejects_layers_wider_than_its_scratch():
    lib = slim._lib()
    n = 32768 + 128
    rc = lib.slim_salience_noalloc(0x1000, 64, n, 0x2000, 128, 0x3000, 0x4000, None)
    assert rc == 1   # SLIM_EINVAL: more input columns than the fixed scratch holds
