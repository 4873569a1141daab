"""Per-stage GPU parity through the C ABI: each stage gets the same inputs as the
oracle step it is compared with. Sizes span several tiles with ragged tails."""
import numpy as np
import pytest
import torch

from oracle import slim_oracle as O
from post_weight_quantization_hessian_b200 import slim
from post_weight_quantization_hessian_b200 import synthetic as syn
from parity_util import (KL_ATOL, balanced_bits, compare_sqc, device_inputs, hessian_bound, order_ok, pstar_ok,
                         x_f64)

pytestmark = pytest.mark.gpu


def spec(**kw):
    base = dict(name="t", m=300, n=640, N=1000, x_dtype="bf16", group=128, avg_bits=2, seed=5,
                n_w_salient=6, w_scale=6.0, n_x_outliers=3, x_scale=25.0)
    base.update(kw)
    return syn.LayerSpec(**base)


# ---------------------------------------------------------------- hessian
@pytest.mark.parametrize("n, N", [(320, 20000), (96, 300), (512, 129), (256, 64)])
def test_hessian_bf16(n, N):
    s = spec(n=n, N=N, group=32)
    W, Xh, Wd, Xd = device_inputs(s)
    H = slim.slim_hessian(Xd).cpu().numpy()
    X = x_f64(s, Xh)
    ref = O.hessian(X)
    scale = 2.0 * (np.abs(X).T @ np.abs(X))
    err = np.abs(H - ref)
    assert np.all(err <= hessian_bound(N) * scale + 1e-300), float((err / np.maximum(scale, 1e-300)).max())
    assert np.array_equal(H, H.T)
    print(f"hessian n={n} N={N}: max |dH|/scale = {(err / np.maximum(scale, 1e-300)).max():.2e}")


def test_hessian_f32():
    s = spec(n=320, N=3000, x_dtype="f32", group=32)
    W, Xh, Wd, Xd = device_inputs(s)
    H = slim.slim_hessian(Xd).cpu().numpy()
    np.testing.assert_allclose(H, O.hessian(x_f64(s, Xh)), rtol=1e-12, atol=1e-9)


# ---------------------------------------------------------------- hinv_diag
@pytest.mark.parametrize("n", [320, 96, 1056, 200, 1000])   # 200, 1000: padded to a multiple of 32 internally
def test_hinv_diag(n):
    rng = np.random.default_rng(n)
    X = rng.standard_normal((4 * n, n))
    X[:, 3] *= 25.0
    X[:, n // 2] = 0.0                                    # a dead column
    H = O.hessian(X)
    h = slim.slim_hinv_diag(torch.from_numpy(H).cuda(), 0.01).cpu().numpy()
    np.testing.assert_allclose(h, O.hinv_diag(H, 0.01), rtol=1e-9)


def test_hinv_diag_beside_a_busy_gpu():
    """The factorization must not depend on its CTAs being resident together.

    GEMMs on another stream hold most SMs' shared memory while the inverse is
    computed, so the CTAs of one launch start at different times; a CTA that
    wrote a block other CTAs of its launch still had to read would show here.
    """
    n = 2048
    rng = np.random.default_rng(7)
    X = rng.standard_normal((2 * n, n))
    X[:, 11] *= 30.0
    H = O.hessian(X)
    ref = O.hinv_diag(H, 0.01)
    Hd = torch.from_numpy(H).cuda()
    a = torch.randn(8192, 8192, dtype=torch.bfloat16, device="cuda")
    busy, work = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for _ in range(3):
        with torch.cuda.stream(busy):
            for _ in range(24):
                a = (a @ a).clamp_(-1.0, 1.0)
        h = slim.slim_hinv_diag(Hd, 0.01, stream=work).cpu().numpy()
        np.testing.assert_allclose(h, ref, rtol=1e-9)
    torch.cuda.synchronize()


def test_hinv_not_positive_definite():
    H = -np.eye(64)
    with pytest.raises(slim.SlimError) as e:
        slim.slim_hinv_diag(torch.from_numpy(H).cuda(), 0.0)
    assert e.value.status == 5
    assert e.value.device_detail == 0          # the first pivot fails


def test_hinv_not_positive_definite_reports_the_pivot():
    """A positive definite matrix with one bad pivot deep inside (column 150 of 320:
    block 2, sub-block 1): the reported index is that column."""
    n, bad = 320, 150
    rng = np.random.default_rng(4)
    X = rng.standard_normal((4 * n, n))
    H = O.hessian(X)
    H[bad, :] = 0.0
    H[:, bad] = 0.0
    H[bad, bad] = -1.0          # a negative diagonal entry with its row and column cleared
    with pytest.raises(slim.SlimError) as e:
        slim.slim_hinv_diag(torch.from_numpy(H).cuda(), 0.0)
    assert e.value.status == 5
    assert e.value.device_detail == bad
    ok = slim.slim_hinv_diag(torch.from_numpy(O.hessian(X)).cuda(), 0.01)   # the next call succeeds
    assert torch.isfinite(ok).all()


# ---------------------------------------------------------------- salience
@pytest.mark.parametrize("group", [128, 64, 32])
def test_salience(group):
    s = spec(group=group)
    W = syn.make_weight(s)
    h = np.random.default_rng(group).uniform(0.2, 2.0, s.n)
    S, order = slim.slim_salience(torch.from_numpy(W).cuda(), torch.from_numpy(h).cuda(), group)
    S_ref = O.group_salience(W, h, group)
    np.testing.assert_allclose(S.cpu().numpy(), S_ref, rtol=1e-12)
    assert order_ok(order.cpu().numpy(), S_ref, rel=1e-12) == 0


# ---------------------------------------------------------------- sqc
@pytest.mark.parametrize("group, avg_bits, p", [(128, 2, 1), (64, 3, 3), (32, 2, 4), (128, 7, 1), (32, 4, 0)])
def test_sqc(group, avg_bits, p):
    s = spec(m=96, n=384, group=group, avg_bits=avg_bits)
    W = syn.make_weight(s)
    W[5, :group] = 0.125                                   # a degenerate group
    h = np.random.default_rng(7).uniform(0.05, 1.0, s.n)
    bits = balanced_bits(s.k, avg_bits, p, seed=group + p)
    codes, scale, zero, tau = slim.slim_sqc(torch.from_numpy(W).cuda(), torch.from_numpy(h).cuda(),
                                            torch.from_numpy(bits).cuda(), group, avg_bits, 0.1, 50)
    ref = O.sqc_calibrate(W, h, bits, group, 0.1, 50)
    agree, tmis = compare_sqc(codes.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), tau.cpu().numpy(),
                              ref, bits, group, avg_bits)
    assert agree >= 0.9999 and tmis == 0, (agree, tmis)
    words_ref = O.pack_codes(ref.codes, bits, group, avg_bits)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), words_ref)


# ---------------------------------------------------------------- sba_search
SBA_CASES = [
    dict(),                                                          # 3 output tiles (last ragged), 8 token tiles
    dict(m=256, n=384, N=700, group=32),                             # k = 12, half-box groups
    dict(m=200, n=512, N=513, group=64, avg_bits=3),
    dict(m=130, n=96, N=300, group=32),                              # n not a multiple of 64
    dict(m=256, n=512, N=2048, x_dtype="f32", group=128, n_w_salient=4, w_scale=8.0, x_scale=20.0),
]


@pytest.mark.parametrize("kw", SBA_CASES)
def test_sba_search(kw):
    s = spec(**kw)
    W, Xh, Wd, Xd = device_inputs(s)
    X = x_f64(s, Xh)
    h = O.hinv_diag(O.hessian(X))
    order = O.salience_order(O.group_salience(W, h, s.group))
    kl, p_star, bits = slim.slim_sba_search(Wd, Xd, s.group, s.avg_bits,
                                            torch.from_numpy(order.astype(np.int32)).cuda())
    ref = O.sba_search(W, X, order, s.group, s.avg_bits)
    kl = kl.cpu().numpy()
    dev = np.abs(kl - ref.kl).max()
    print(f"sba {kw}: KL {kl} ref {ref.kl} max|dKL| {dev:.2e} p* {int(p_star.item())}/{ref.p_star}")
    assert dev <= KL_ATOL
    if pstar_ok(int(p_star.item()), ref.kl, kl):
        assert np.array_equal(bits.cpu().numpy(), ref.bits.astype(np.uint8))
    b = bits.cpu().numpy().astype(int)
    assert b.sum() == s.k * s.avg_bits


SPLIT_CASES = [(kw, 256) for kw in SBA_CASES] + [
    (dict(m=384, n=512, N=5000, group=64), 512),     # 40 token tiles: chunks of 2 pairs, ragged last tile
    (dict(m=128, n=128, N=600, group=128), 256),     # k = 1: phase A only, no candidate step
    (dict(m=130, n=256, N=3000, group=32, avg_bits=3), 1024),
]


@pytest.mark.parametrize("kw, chunk", SPLIT_CASES)
def test_sba_search_split_matches_one_pass(kw, chunk):
    """Phase A per token chunk, its TMEM state stored, the candidate steps resumed
    from it: the same KL, p* and bits as the one-pass search, bit for bit."""
    s = spec(**kw)
    W, Xh, Wd, Xd = device_inputs(s)
    order = torch.from_numpy(np.random.default_rng(s.seed).permutation(s.k).astype(np.int32)).cuda()
    kl1, p1, b1 = slim.slim_sba_search(Wd, Xd, s.group, s.avg_bits, order)
    kl2, p2, b2 = slim.slim_sba_search_split(Wd, Xd, s.group, s.avg_bits, order, chunk)
    assert np.array_equal(kl1.cpu().numpy().view(np.uint64), kl2.cpu().numpy().view(np.uint64))
    assert int(p1.item()) == int(p2.item())
    assert np.array_equal(b1.cpu().numpy(), b2.cpu().numpy())


def test_sba_search_split_rejects_unaligned_chunks():
    s = spec()
    W, Xh, Wd, Xd = device_inputs(s)
    order = torch.arange(s.k, dtype=torch.int32, device="cuda")
    with pytest.raises(slim.SlimError) as e:
        slim.slim_sba_search_split(Wd, Xd, s.group, s.avg_bits, order, 384)
    assert e.value.status == 1


def test_sqc_larger_layer():
    """1M weights x 50 candidates: every quotient of the calibration loop exercised."""
    s = spec(m=1024, n=1024, group=64, avg_bits=3, seed=21)
    W = syn.make_weight(s)
    h = np.random.default_rng(21).uniform(0.05, 1.0, s.n)
    bits = balanced_bits(s.k, s.avg_bits, 5, seed=21)
    codes, scale, zero, tau = slim.slim_sqc(torch.from_numpy(W).cuda(), torch.from_numpy(h).cuda(),
                                            torch.from_numpy(bits).cuda(), s.group, s.avg_bits, 0.1, 50)
    ref = O.sqc_calibrate(W, h, bits, s.group, 0.1, 50)
    agree, tmis = compare_sqc(codes.cpu().numpy(), scale.cpu().numpy(), zero.cpu().numpy(), tau.cpu().numpy(),
                              ref, bits, s.group, s.avg_bits)
    assert agree >= 0.9999 and tmis == 0, (agree, tmis)
