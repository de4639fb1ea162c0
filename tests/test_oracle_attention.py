"""Pins of the oracle's decode attention and top-k against brute force and limits.

Sources: PolarQuant review (mdooai, attention over a quantized KV cache: softmax of
scaled query-key products weighting the values); TurboQuant review (Jump2Paper,
KV-cache and nearest-neighbour applications).
"""
import math

import numpy as np

import synth
from oracle import attention as A
from oracle import quantizer as Q
from oracle import rotation as rot


def _loops_attention(q, K, V, scale):
    H, T, d = K.shape
    out = [[0.0] * d for _ in range(H)]
    for h in range(H):
        s = [sum(q[h][j] * K[h][t][j] for j in range(d)) * scale for t in range(T)]
        m = max(s)
        w = [math.exp(v - m) for v in s]
        tot = sum(w)
        for t in range(T):
            for j in range(d):
                out[h][j] += w[t] / tot * V[h][t][j]
    return np.array(out)


def test_attention_equals_loops():
    rng = np.random.default_rng(3)
    H, T, d = 2, 9, 4
    q, K, V = rng.standard_normal((H, d)), rng.standard_normal((H, T, d)), rng.standard_normal((H, T, d))
    np.testing.assert_allclose(A.decode_attention(q, K, V, 0.5), _loops_attention(q, K, V, 0.5),
                               atol=1e-13)


def test_attention_softmax_extremes():
    # A dominant key returns its value; equal keys return the mean of the values.
    d = 4
    K = np.zeros((1, 3, d))
    K[0, 1, 0] = 1e3
    V = np.arange(12.0).reshape(1, 3, d)
    out = A.decode_attention(np.array([[1.0, 0, 0, 0]]), K, V, 1.0)
    np.testing.assert_allclose(out[0], V[0, 1])
    out = A.decode_attention(np.array([[0.0, 0, 0, 0]]), K, V, 1.0)
    np.testing.assert_allclose(out[0], V[0].mean(axis=0))


def test_compressed_attention_tends_to_exact():
    # With more bits, attention over reconstructed K and V approaches exact attention.
    d, T = 64, 256
    P = rot.haar_from_gaussian(synth.gaussian_matrix(d, 0))
    S = synth.gaussian_matrix(d, 1)
    K = synth.unit_vectors(T, d, seed=60, dtype=np.float64)
    V = synth.unit_vectors(T, d, seed=61, dtype=np.float64)
    q = synth.gaussian_vectors(1, d, seed=62) * 3
    exact = A.decode_attention(q, K[None], V[None], 1 / math.sqrt(d))
    errs = []
    for b in (2, 3, 4, 5, 6):
        cbk, cbv = Q.make_codebook(d, b - 1), Q.make_codebook(d, b)
        c, z, nu, rho, _, _ = Q.encode_prod(K, P, S, cbk)
        kt = Q.decode_prod(c, z, nu, rho, P, S, cbk)
        cv, nv, _ = Q.encode_mse(V, P, cbv)
        vt = Q.decode_mse(cv, nv, P, cbv)
        errs.append(np.max(np.abs(A.decode_attention(q, kt[None], vt[None], 1 / math.sqrt(d)) - exact)))
    assert all(e2 < e1 for e1, e2 in zip(errs, errs[1:]))
    assert errs[-1] < 2e-3


def test_topk_matches_python_sort_with_ties():
    rng = np.random.default_rng(4)
    est = np.round(rng.standard_normal((5, 200)), 1)        # many ties
    idx, vals = A.topk(est, 10)
    for i in range(5):
        want = sorted(range(200), key=lambda k: (-est[i, k], k))[:10]
        assert list(idx[i]) == want
        np.testing.assert_array_equal(vals[i], est[i, want])
