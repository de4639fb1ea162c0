"""Pins of the oracle's rotations against the pages and the mathematics.

Sources: TurboQuant review (Jump2Paper), Lemma 1 and the figure of the first coordinate
at d=1000 (Beta law, Gaussian N(0,1/d) at large d); AI Trends summary of the TurboQuant
video, chapter "L2 normalize + RHT matrix" (the RHT's inverse is its transpose); the
Reddit critique on the damoang.net RotorQuant post (a global rotation spreads a one-hot
vector over all 128 dimensions).
"""
import math

import numpy as np
import pytest
import scipy.linalg
from scipy import stats

import synth
from oracle import rotation as rot


def test_haar_qr_is_orthogonal_and_unique():
    for d in (8, 128, 256):
        g = synth.gaussian_matrix(d, seed=0)
        P = rot.haar_from_gaussian(g)
        np.testing.assert_allclose(P.T @ P, np.eye(d), atol=1e-12)
        assert abs(abs(np.linalg.det(P)) - 1) < 1e-9
        # Pi^T G is upper triangular with a positive diagonal: the unique QR with R_ii > 0.
        R = P.T @ g
        assert np.max(np.abs(np.tril(R, -1))) < 1e-10
        assert np.all(np.diag(R) > 0)


def test_rht_is_orthogonal_and_sylvester():
    for d in (2, 8, 128, 256):
        eps = synth.rht_signs(d, seed=0)
        P = rot.rht_matrix(eps)
        np.testing.assert_allclose(P.T @ P, np.eye(d), atol=1e-13)   # inverse = transpose
        i = np.arange(d)
        pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
        np.testing.assert_array_equal(P * math.sqrt(d) * eps[None, :], (-1.0) ** pc)


def test_one_hot_is_spread_evenly(paper):
    d = paper["one_hot_spread"]["d"]
    P = rot.rht_matrix(synth.rht_signs(d, seed=3))
    for j in (0, 5, d - 1):
        e = np.zeros(d)
        e[j] = 1
        np.testing.assert_allclose(np.abs(P @ e), np.full(d, 1 / math.sqrt(d)), rtol=1e-14)


def test_rotated_coordinates_follow_lemma1():
    # A fixed worst-case input (one-hot) rotated by many independent Haar matrices:
    # each coordinate of y = Pi x follows f_X (KS test against the library Beta law).
    d = 32
    a = (d - 1) / 2
    ys = []
    for s in range(400):
        P = rot.haar_from_gaussian(synth.gaussian_matrix(d, seed=100 + s))
        ys.append(P[:, 0])              # Pi e_1
    y = np.concatenate(ys)
    assert stats.kstest((y + 1) / 2, stats.beta(a, a).cdf).pvalue > 1e-3
    # The same data is far from the law of a different dimension: the test has power.
    assert stats.kstest((y + 1) / 2, stats.beta(a + 6, a + 6).cdf).pvalue < 1e-6
    assert abs(np.var(y) * d - 1) < 0.05


def test_uniform_inputs_fixed_rotation_follow_lemma1_and_gaussian_limit():
    for d in (128, 1536):
        a = (d - 1) / 2
        P = rot.haar_from_gaussian(synth.gaussian_matrix(d, seed=0)) if d == 128 else None
        x = synth.unit_vectors(4000 if d == 128 else 600, d, seed=9, dtype=np.float64)
        y = (x @ P.T) if P is not None else x
        v = y[:, :16].ravel()
        assert stats.kstest((v + 1) / 2, stats.beta(a, a).cdf).pvalue > 1e-3
        if d == 1536:
            # Large d: the Beta law is close to N(0, 1/d).
            assert stats.kstest(v * math.sqrt(d), stats.norm.cdf).pvalue > 1e-3


def test_paley_hadamard12_is_a_skew_hadamard_matrix():
    # Paley I (q = 11): H H^T = 12 I, entries +-1, and H - I is skew-symmetric.
    H = rot.paley_hadamard12()
    assert H.shape == (12, 12) and set(np.unique(H)) == {-1.0, 1.0}
    np.testing.assert_array_equal(H @ H.T, 12 * np.eye(12))
    np.testing.assert_array_equal((H - np.eye(12)).T, -(H - np.eye(12)))
    # the quadratic residues of GF(11) are 1, 3, 4, 5, 9: row 1 of Q, shifted by the border
    np.testing.assert_array_equal(H[1, 2:], [1, -1, 1, 1, 1, -1, -1, -1, 1, -1])


@pytest.mark.parametrize("d", [96, 192, 384, 1536])
def test_kronecker_rht_is_orthogonal(d):
    eps = synth.rht_signs(d, seed=2)
    P = rot.rht_matrix(eps)
    np.testing.assert_allclose(P @ P.T, np.eye(d), atol=1e-12)
    # structure: entry (i, j) = H12[i / m][j / m] * H_m[i % m][j % m] * eps_j / sqrt(d), m = d / 12
    m = d // 12
    H12, Hm = rot.paley_hadamard12(), scipy.linalg.hadamard(m)
    i, j = 5 * m + 3, 7 * m + 1
    assert P[i, j] == H12[5, 7] * Hm[3, 1] * eps[j] / np.sqrt(d)
    # a rotated one-hot vector spreads evenly: every |coordinate| = 1/sqrt(d)
    np.testing.assert_allclose(np.abs(P[:, 17]), 1 / np.sqrt(d), rtol=1e-12)
