"""GPU parity of slim_dequant_gemv (y = x W_hat^T on the packed layout) against
the oracle's dequant_matmul, through the C ABI.

The inference product is the pages' stated cost of mixed 1/2/3-bit groups
(rkmt.cn write-up, section 局限性; atlas.scime.ai summary, Limitations).

Tolerance: the kernel forms, per (row, group), A = sum_j x_j f_j with
f_j = 1 + q_j 2^-b in [1, 2) and xs = sum_j x_j in fp32 (g terms each), then
2^b (A - xs). Each fp32 sum carries at most about g 2^-24 sum_j |x_j| f_j of
rounding error, and 2^b scales it next to |w_hat| ~ scale 2^b / 2, so per
output |dy| <= ~g 2^-22 sum_j |x_j w_hat_ij| (3e-5 at g = 128) plus the last
fp32 sums over groups; 4e-5 of that abs-sum is the bar.
"""
import numpy as np
import pytest
import torch

from oracle import slim_oracle as O
from post_weight_quantization_hessian_b200 import slim
from post_weight_quantization_hessian_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def quantized_layer(m, n, group, avg_bits, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((m, n)) * 0.02).astype(np.float32)
    W[:, rng.choice(n, 4, replace=False)] *= 6.0
    k = n // group
    bits = O.allocation(rng.permutation(k), avg_bits, k // 3).astype(np.uint8)
    r = O.sqc_calibrate(W, rng.uniform(0.1, 1.0, n), bits, group, 0.1, 50)
    words = O.pack_codes_fast(r.codes, bits, group, avg_bits)
    return words, bits, r.scale, r.zero


@pytest.mark.parametrize("m, n, group, avg_bits, batch, xdt", [
    (300, 512, 128, 2, 1, "f32"),
    (4096, 1024, 64, 2, 3, "bf16"),
    (257, 384, 32, 2, 8, "f32"),       # ragged rows, 1/2/3-bit groups of 32
    (200, 512, 64, 3, 2, "bf16"),      # 2/3/4-bit groups
    (130, 256, 32, 7, 1, "f32"),       # 6/7/8-bit groups (codes straddle words)
])
def test_dequant_gemv(m, n, group, avg_bits, batch, xdt):
    words, bits, scale, zero = quantized_layer(m, n, group, avg_bits, seed=m + n)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((batch, n)).astype(np.float32)
    x[:, 3] *= 20.0
    if xdt == "bf16":
        xb = syn.f32_to_bf16_bits(x)
        x = syn.bf16_bits_to_f32(xb)
        xd = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    else:
        xd = torch.from_numpy(x).cuda()
    y = slim.slim_dequant_gemv(torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(bits).cuda(),
                               torch.from_numpy(scale).cuda(), torch.from_numpy(zero).cuda(), group, avg_bits,
                               xd).cpu().numpy()
    ref = O.dequant_matmul(words, bits, scale, zero, group, x)
    codes = O.unpack_codes(words, bits, group, n)
    Wq = O.dequant_codes(codes, scale, zero, group)
    bound = 4e-5 * (np.abs(x.astype(np.float64)) @ np.abs(Wq).T) + 1e-30
    err = np.abs(y - ref)
    print(f"gemv m={m} n={n} g={group} b={avg_bits} B={batch}: max |dy|/abs-sum {(err / bound).max() * 4e-5:.2e}")
    assert np.all(err <= bound)


def test_dequant_gemv_is_asynchronous_and_repeatable():
    """The call only enqueues: issued back to back on one stream with one workspace, every
    result equals the first (same inputs, fixed-order sums)."""
    words, bits, scale, zero = quantized_layer(512, 1024, 128, 2, seed=9)
    dev = [torch.from_numpy(a).cuda() for a in (words.view(np.int32), bits, scale, zero)]
    x = torch.randn((2, 1024), device="cuda")
    ws = torch.empty(max(256, slim._lib().slim_dequant_gemv_workspace_bytes(512, 1024, 128, 2, 2)), dtype=torch.uint8,
                     device="cuda")
    ys = [slim.slim_dequant_gemv(*dev, 128, 2, x, ws=ws) for _ in range(5)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
