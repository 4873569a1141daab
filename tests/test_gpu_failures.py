"""Failure detection on the GPU, in forms that fault, trap or hang nothing:
host-side injection (SLIM_FAULT=<stage>), a device-side range check turned into
SLIM_ERANGE, one bounded device wait made to run out (a test-only limit on the
scoring kernel's wait for its accumulator) returning SLIM_ETIMEOUT with the
device still usable, and the library's memory pool leaving the device's default
pool untouched."""
import os

import numpy as np
import pytest
import torch

from post_weight_quantization_hessian_b200 import slim
from post_weight_quantization_hessian_b200 import synthetic as syn
from parity_util import device_inputs

pytestmark = pytest.mark.gpu

EINVAL, ETIMEOUT, EINJECTED, ERANGE = 1, 4, 7, 8


def small():
    return syn.LayerSpec(name="f", m=256, n=512, N=1024, x_dtype="bf16", group=128, avg_bits=2, seed=3,
                         n_w_salient=4, w_scale=6.0, n_x_outliers=2, x_scale=25.0)


@pytest.fixture
def env():
    saved = {k: os.environ.get(k) for k in ("SLIM_FAULT", "SLIM_TEST_ACC_WAIT_NS")}
    yield os.environ
    for k, v in saved.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v


@pytest.mark.parametrize("stage", ["hessian", "hinv_diag", "salience", "sba_search", "sqc"])
def test_injected_stage_failure(env, stage):
    s = small()
    W, Xh, Wd, Xd = device_inputs(s)
    env["SLIM_FAULT"] = stage
    with pytest.raises(slim.SlimError) as e:
        slim.slim_quantize_layer(Wd, Xd, s.group, s.avg_bits)
    assert e.value.status == EINJECTED
    del env["SLIM_FAULT"]
    codes, scale, zero, bits = slim.slim_quantize_layer(Wd, Xd, s.group, s.avg_bits)   # usable afterwards
    assert int(bits.cpu().numpy().astype(int).sum()) == s.k * s.avg_bits


def test_injected_failure_of_a_stage_entry_point(env):
    s = small()
    W, Xh, Wd, Xd = device_inputs(s)
    env["SLIM_FAULT"] = "hessian"
    with pytest.raises(slim.SlimError) as e:
        slim.slim_hessian(Xd)
    assert e.value.status == EINJECTED


def test_activation_out_of_fp16_range(env):
    s = small()
    W, Xh, Wd, Xd = device_inputs(s)
    Xbad = Xd.clone()
    Xbad[5, 17] = 70000.0                      # representable in bf16, not in fp16
    with pytest.raises(slim.SlimError) as e:
        slim.slim_quantize_layer(Wd, Xbad, s.group, s.avg_bits)
    assert e.value.status == ERANGE
    slim.slim_quantize_layer(Wd, Xd, s.group, s.avg_bits)


def test_weight_out_of_fp16_operand_range(env):
    s = small()
    W, Xh, Wd, Xd = device_inputs(s)
    Wbad = Wd.clone()
    Wbad[3, 9] = 300.0                         # 300 * 2^8 > 65504
    order = torch.arange(s.k, dtype=torch.int32, device="cuda")
    with pytest.raises(slim.SlimError) as e:
        slim.slim_sba_search(Wbad, Xd, s.group, s.avg_bits, order)
    assert e.value.status == ERANGE


def test_a_device_wait_that_runs_out(env):
    """The scoring kernel's epilogue waits for its first accumulator with a 1 ns
    limit: the wait gives up, the CTA unwinds (its copies and MMAs drained, tensor
    memory freed), the call returns SLIM_ETIMEOUT naming the wait, and the next
    call with the normal limit gives the same result as before."""
    s = syn.LayerSpec(name="w", m=256, n=4096, N=512, x_dtype="bf16", group=128, avg_bits=2, seed=4,
                      n_w_salient=4, w_scale=6.0, n_x_outliers=2, x_scale=25.0)
    W, Xh, Wd, Xd = device_inputs(s)
    order = torch.arange(s.k, dtype=torch.int32, device="cuda")
    kl0, p0, b0 = slim.slim_sba_search(Wd, Xd, s.group, s.avg_bits, order)
    env["SLIM_TEST_ACC_WAIT_NS"] = "1"
    with pytest.raises(slim.SlimError) as e:
        slim.slim_sba_search(Wd, Xd, s.group, s.avg_bits, order)
    assert e.value.status == ETIMEOUT
    assert e.value.device_detail in (240, 241)
    del env["SLIM_TEST_ACC_WAIT_NS"]
    kl1, p1, b1 = slim.slim_sba_search(Wd, Xd, s.group, s.avg_bits, order)
    assert np.array_equal(kl0.cpu().numpy(), kl1.cpu().numpy())
    assert torch.equal(b0, b1)


def test_library_pool_leaves_the_default_pool_alone():
    from cuda.bindings import runtime as rt
    dev = torch.cuda.current_device()
    err, pool = rt.cudaDeviceGetDefaultMemPool(dev)
    assert err == rt.cudaError_t.cudaSuccess
    err, before = rt.cudaMemPoolGetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrReleaseThreshold)
    s = small()
    W, Xh, Wd, Xd = device_inputs(s)
    slim.slim_quantize_layer(Wd, Xd, s.group, s.avg_bits)          # ws = NULL: the library allocates
    err, after = rt.cudaMemPoolGetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrReleaseThreshold)
    assert int(after) == int(before)
