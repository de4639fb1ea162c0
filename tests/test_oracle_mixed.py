"""Pins of the outlier-channel split (oracle/mixed.py).

Source: TurboQuant review (Jump2Paper), experiment settings table ("KV bit settings",
"outlier handling") and the closing note on outlier channels. The split is two
independent TurboQuant quantizers on complementary channel groups; the pins check the
bookkeeping exactly, the special case that reduces to the plain quantizer, additivity of
the estimate, and (statistically) unbiasedness and the distortion of each group.
"""
import math

import numpy as np
import pytest

import synth
from conftest import load_golden
from oracle import mixed as M
from oracle import quantizer as Q
from oracle import rotation as rot


def test_effective_width_of_the_stated_split():
    g = load_golden("paper_values.json")["outlier_split"]
    m, d = g["outlier_channels"], g["d"]
    w = M.effective_bits([(m, g["outlier_bits"]), (d - m, g["rest_bits"])])
    # the printed expression evaluates to 288 / 128 = 2.25, not the printed 2.5
    assert w == (32 * 3 + 96 * 2) / 128 == 2.25
    assert w != g["printed_effective_bits"]
    # splits of 128 channels that do give the two printed settings
    assert M.effective_bits([(32, 4), (96, 2)]) == 2.5
    assert M.effective_bits([(64, 4), (64, 3)]) == 3.5
    assert M.effective_bits([(128, 3)]) == 3.0


def test_split_merge_roundtrip_any_channel_order():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((9, 40))
    for ch in ([0, 5, 39], list(rng.permutation(40)[:17]), []):
        a, b = M.split(x, ch)
        assert a.shape == (9, len(ch)) and b.shape == (9, 40 - len(ch))
        np.testing.assert_array_equal(M.merge(a, b, ch, 40), x)
        rest = M.rest_channels(ch, 40)
        assert sorted(list(ch) + list(rest)) == list(range(40)) and np.all(np.diff(rest) > 0)


def test_outlier_channels_finds_the_heavy_ones():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((500, 64))
    heavy = [3, 17, 40, 41, 63]
    x[:, heavy] *= 10.0
    np.testing.assert_array_equal(M.outlier_channels(x, 5), heavy)


def _prod_state(d, b, seed):
    Pi = rot.haar_from_gaussian(synth.gaussian_matrix(d, seed))
    S = synth.gaussian_matrix(d, seed + 1000)
    cb = Q.make_codebook(d, b - 1) if b > 1 else None
    return Pi, S, cb


def _prod_roundtrip(x, st):
    Pi, S, cb = st
    codes, z, nu, rho, _, _ = Q.encode_prod(x, Pi, S, cb)
    return Q.decode_prod(codes, z, nu, rho, Pi, S, cb)


def test_empty_outlier_group_is_the_plain_quantizer():
    d = 32
    x = synth.gaussian_vectors(50, d, seed=3)
    st = _prod_state(d, 3, 7)
    a, b = M.split(x, [])
    assert a.shape[1] == 0
    # equal up to the BLAS's summation order on a copied array
    np.testing.assert_allclose(M.merge(np.zeros((50, 0)), _prod_roundtrip(b, st), [], d), _prod_roundtrip(x, st),
                               rtol=1e-12, atol=1e-12)


def test_estimate_is_the_sum_of_the_group_estimates():
    d, ch = 24, [1, 4, 9, 10, 22]
    x = synth.gaussian_vectors(30, d, seed=4)
    q = synth.gaussian_vectors(6, d, seed=5)
    so, sr = _prod_state(len(ch), 3, 11), _prod_state(d - len(ch), 2, 13)
    xo, xr = M.split(x, ch)
    to, tr = _prod_roundtrip(xo, so), _prod_roundtrip(xr, sr)
    qo, qr = M.split(q, ch)
    np.testing.assert_allclose(Q.estimate(q, M.merge(to, tr, ch, d)),
                               Q.estimate(qo, to) + Q.estimate(qr, tr), rtol=1e-12, atol=1e-12)


def test_split_prod_estimate_is_unbiased():
    # E over the random state of <q, x~> equals <q, x> (Theorem 2 per group, summed).
    d, ch = 16, [0, 5, 6, 11]
    rng = np.random.default_rng(8)
    x = rng.standard_normal((1, d))
    x[:, ch] *= 6.0
    q = rng.standard_normal((1, d))
    true = float((q @ x.T)[0, 0])
    xo, xr = M.split(x, ch)
    qo, qr = M.split(q, ch)
    errs = []
    for t in range(3000):
        so, sr = _prod_state(len(ch), 3, 100 + 2 * t), _prod_state(d - len(ch), 2, 101 + 2 * t)
        est = float((qo @ _prod_roundtrip(xo, so).T)[0, 0] + (qr @ _prod_roundtrip(xr, sr).T)[0, 0])
        errs.append(est - true)
    errs = np.array(errs)
    assert abs(errs.mean()) < 4 * errs.std() / math.sqrt(len(errs))


def test_split_mse_distortion_is_the_sum_of_group_distortions():
    # E||x - x~||^2 = ||x_O||^2 D(m, b_O) + ||x_R||^2 D(d-m, b_R) (Theorem 1 per group).
    d, m = 128, 32
    ch = np.arange(0, d, d // m)
    x = synth.unit_vectors(8192, d, seed=21, dtype=np.float64)
    x[:, ch] *= 4.0
    xo, xr = M.split(x, ch)
    cbo, cbr = Q.make_codebook(m, 3), Q.make_codebook(d - m, 2)
    Po = rot.haar_from_gaussian(synth.gaussian_matrix(m, 31))
    Pr = rot.haar_from_gaussian(synth.gaussian_matrix(d - m, 32))
    co, no, _ = Q.encode_mse(xo, Po, cbo)
    cr, nr, _ = Q.encode_mse(xr, Pr, cbr)
    xt = M.merge(Q.decode_mse(co, no, Po, cbo), Q.decode_mse(cr, nr, Pr, cbr), ch, d)
    err = np.sum((xt - x) ** 2, axis=1)
    want = np.sum(xo ** 2, axis=1) * cbo.dmse + np.sum(xr ** 2, axis=1) * cbr.dmse
    assert abs(err.mean() / want.mean() - 1) < 0.03
