"""Embedding-search shape at full size: 1,000,000 vectors, d = 1536 (Gaussian mixture, bf16),
TurboQuant_prod b = 2 with dense Pi and S (bf16) on the tensor core, 1000 queries, top-10.

The whole database is encoded and searched on the GPU in the launch configuration of a user
call. The oracle then re-encodes the whole database block by block: every block's planes are
checked under the band rule, and the estimates of all 1000 queries against all 10^6 keys give
the oracle's own top-10 of every query, which the library's top-10 must match (a swap at the
cut counts as a match when the two estimates are within the score tolerance; a key whose
planes differ from the oracle's in-band is checked against the oracle's estimate from the library's
planes).
"""
import numpy as np
import pytest

import synth
from oracle import attention as OA
from oracle import quantizer as OQ
from parity import ABS_SCORE, Pair, check_codes, unpack

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
tq = pytest.importorskip("vector_quantization_tq_b200")

N, D, NQ, K, BLK = 1_000_000, 1536, 1000, 10, 32768


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _merge_topk(best_i, best_v, blk_i, blk_v):
    """Top-K of the union of two candidate lists per query (ties to the lower index)."""
    ci = np.concatenate([best_i, blk_i], axis=1)
    cv = np.concatenate([best_v, blk_v], axis=1)
    order = np.lexsort((ci, -cv), axis=1)[:, :K]
    return np.take_along_axis(ci, order, axis=1), np.take_along_axis(cv, order, axis=1)


def test_c5_full_encode_and_search():
    pair = Pair(tq, D, 2, tq.PROD, tq.ROT_DENSE, tq.BF16)
    bits, _ = synth.mixture_vectors(N, D)
    x = _bf16_dev(bits)
    codes, qjl, norms, rnorms = pair.st.empty_planes(N)
    tq.quantize_prod(pair.st, x, codes, qjl, norms, rnorms)
    del x
    qbits, _ = synth.mixture_vectors(NQ, D, seed=synth.SEED_DATA + 9, centre_seed=synth.SEED_DATA)
    idx = torch.empty((NQ, K), dtype=torch.int64, device="cuda")
    vals = torch.empty((NQ, K), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.search_workspace(pair.st, NQ, N, K), dtype=torch.uint8, device="cuda")
    tq.search_topk(pair.st, _bf16_dev(qbits), codes, qjl, norms, rnorms, K, idx, vals, ws)
    torch.cuda.synchronize()
    tq.device_status(0)
    gi, gv = idx.cpu().numpy(), vals.cpu().numpy()
    assert np.all(np.diff(gv, axis=1) <= 0)
    assert np.all((gi >= 0) & (gi < N))
    assert all(len(set(row)) == K for row in gi)
    g = dict(codes=codes.cpu().numpy(), qjl=qjl.cpu().numpy(), norms=norms.cpu().numpy(),
             rnorms=rnorms.cpu().numpy())
    del codes, qjl, norms, rnorms
    qv = synth.bf16_from_bits(qbits)

    best_i = np.zeros((NQ, 0), np.int64)
    best_v = np.zeros((NQ, 0))
    ref = np.full((NQ, K), np.nan)        # oracle estimate of every returned key
    bad_all = np.zeros(N, bool)
    for r0 in range(0, N, BLK):
        r1 = min(N, r0 + BLK)
        enc = pair.encode(synth.bf16_from_bits(bits[r0:r1]))
        bad = check_codes(pair, {k: v[r0:r1] for k, v in g.items()}, enc)
        bad_all[r0:r1] = bad
        est = OQ.estimate(qv, pair.decode(enc))
        blk_i = np.broadcast_to(np.arange(r0, r1), est.shape)
        top = np.argpartition(-est, K - 1, axis=1)[:, :K]
        best_i, best_v = _merge_topk(best_i, best_v, np.take_along_axis(blk_i, top, 1),
                                     np.take_along_axis(est, top, 1))
        inb = (gi >= r0) & (gi < r1)
        qi, kj = np.nonzero(inb)
        ref[qi, kj] = est[qi, gi[qi, kj] - r0]
    assert not np.isnan(ref).any()
    assert bad_all.mean() < 0.01

    # keys whose planes differ in-band: the oracle's estimate from the library's planes
    qi, kj = np.nonzero(bad_all[gi])
    for i, j in zip(qi, kj):
        k = gi[i, j]
        codes_k = unpack(g["codes"][k:k + 1], pair.b_mse, D)
        z_k = unpack(g["qjl"][k:k + 1], 1, D)
        xt = OQ.decode_prod(codes_k, z_k, g["norms"][k:k + 1].astype(np.float64),
                            g["rnorms"][k:k + 1].astype(np.float64), pair.Pi, pair.S, pair.cb)
        ref[i, j] = OQ.estimate(qv[i:i + 1], xt)[0, 0]

    # every returned estimate is the oracle's
    np.testing.assert_allclose(gv, ref, atol=ABS_SCORE)
    # the oracle's top-10 (ties to the lower index, as OA.topk) against the library's
    oi, ov = best_i, best_v
    np.testing.assert_array_equal(OA.topk(ov, K)[0], np.tile(np.arange(K), (NQ, 1)))
    for i in range(NQ):
        got, want = set(gi[i].tolist()), set(oi[i].tolist())
        for j, k in enumerate(gi[i]):
            if k not in want:        # a swap at the cut: no worse than the oracle's 10th
                assert ref[i, j] >= ov[i, -1] - ABS_SCORE, (i, k)
        for j, k in enumerate(oi[i]):
            if k not in got and not bad_all[k]:   # left out: no better than the returned 10th
                assert ov[i, j] <= gv[i, -1] + ABS_SCORE, (i, k)
