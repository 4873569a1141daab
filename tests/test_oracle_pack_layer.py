"""Pins for the packed layout and the whole-layer invariants of the oracle."""
import numpy as np

from oracle import slim_oracle as O
from post_weight_quantization_hessian_b200 import synthetic as syn


def test_pack_hand_example():
    # two groups of 32 at bits [1, 3], average 2 -> 64 * 2 / 32 = 4 words per row
    codes = np.zeros((1, 64), dtype=np.int64)
    codes[0, :32] = 1                 # stream bits 0..31 all set -> word 0 = 0xFFFFFFFF
    codes[0, 32] = 5                  # stream bits 32..34 = 1,0,1 -> word 1 bits 0..2 = 0b101
    codes[0, 42] = 7                  # stream bits 62,63,64 -> word 1 bits 30,31 and word 2 bit 0
    words = O.pack_codes(codes, [1, 3], 32, 2)
    assert words.tolist() == [[0xFFFFFFFF, 0xC0000005, 0x1, 0x0]]
    assert np.array_equal(O.unpack_codes(words, [1, 3], 32, 64), codes)


def test_pack_roundtrip_and_fast_path():
    rng = np.random.default_rng(0)
    bits = [3, 1, 2, 2, 1, 3]
    g = 32
    codes = np.concatenate([rng.integers(0, 2 ** b, size=(5, g)) for b in bits], axis=1)
    w1 = O.pack_codes(codes, bits, g, 2)
    assert w1.shape == (5, 6 * 32 * 2 // 32)
    assert np.array_equal(O.pack_codes_fast(codes, bits, g, 2), w1)
    assert np.array_equal(O.unpack_codes(w1, bits, g, 6 * g), codes)


def test_tiny_layer_invariants():
    spec = syn.TINY
    W = syn.make_weight(spec)
    X = syn.activations_f64(spec)
    r = O.quantize_layer(W, X, spec.group, spec.avg_bits, spec.lam, spec.n_tau, final_kl=True)
    k = spec.k
    assert sorted(r.order.tolist()) == list(range(k))
    assert r.sba.bits.sum() == k * spec.avg_bits
    assert (r.sba.bits == 3).sum() == (r.sba.bits == 1).sum() == r.sba.p_star
    assert np.all(r.h > 0)
    # every dequantized value sits on its group's grid
    for c, b in enumerate(r.sba.bits):
        q = r.sqc.codes[:, c * spec.group:(c + 1) * spec.group]
        assert q.min() >= 0 and q.max() <= 2 ** b - 1
    assert np.array_equal(O.unpack_codes(r.words, r.sba.bits, spec.group, spec.n), r.sqc.codes)
    # the seeded salient columns' groups outrank the rest
    sal = syn.salient_columns(spec) // spec.group
    assert set(r.order[:1].tolist()) <= set(sal.tolist())
    assert r.kl_final is not None and r.kl_final >= 0


def test_dequant_matmul_hand_example():
    """Two output rows, one group of 32 columns at 2 bits (32 codes x 2 bits = 2 words per
    row), codes written out by hand: y = x (scale (q - zero))^T."""
    q = np.zeros((2, 32), dtype=np.int64)
    q[0, :4] = [3, 0, 1, 2]
    q[1, 30:] = [1, 3]
    words = O.pack_codes(q, [2], 32, 2)
    # row 0: q0..q3 = 3, 0, 1, 2 at bits 0-1, 2-3, 4-5, 6-7 -> 0b10_01_00_11 = 0x93 in the first word
    assert int(words[0, 0]) == 0x93 and int(words[0, 1]) == 0
    # row 1: q30 = 1 at bits 28-29 of word 1, q31 = 3 at bits 30-31 -> 0xD0000000
    assert int(words[1, 1]) == 0xD0000000
    scale = np.array([[0.5], [2.0]])
    zero = np.array([[1.0], [0.25]])
    x = np.zeros((1, 32))
    x[0, 0], x[0, 2], x[0, 31] = 2.0, -1.0, 4.0
    y = O.dequant_matmul(words, [2], scale, zero, 32, x)
    # row 0: w_hat = 0.5 (q - 1): cols 0, 2 -> 1.0, 0.0; col 31 -> -0.5
    # row 1: w_hat = 2 (q - 0.25): cols 0, 2 -> -0.5, -0.5; col 31 -> 5.5
    assert y[0, 0] == 2.0 * 1.0 + (-1.0) * 0.0 + 4.0 * (-0.5)
    assert y[0, 1] == 2.0 * -0.5 + (-1.0) * -0.5 + 4.0 * 5.5


def test_dequant_matmul_is_the_plain_product_on_a_quantized_layer():
    """On a whole quantized layer (mixed 1/2/3-bit groups from a balanced allocation)
    the product equals x W_hat^T formed from the codes the quantizer returned, before
    packing: packing, unpacking and dequantization lose nothing."""
    rng = np.random.default_rng(3)
    W = rng.standard_normal((40, 256)) * 0.02
    bits = O.allocation(np.array([1, 0, 3, 2, 6, 5, 4, 7]), 2, 3)
    r = O.sqc_calibrate(W, np.ones(256), bits, 32, 0.1, 50)
    words = O.pack_codes_fast(r.codes, bits, 32, 2)
    x = rng.standard_normal((3, 256))
    ref = x @ (r.scale64.repeat(32, axis=1) * (r.codes - r.zero64.repeat(32, axis=1))).T
    y = O.dequant_matmul(words, bits, r.scale64, r.zero64, 32, x)
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-15)
