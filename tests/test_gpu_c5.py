"""Embedding-search shape at full size: 1,000,000 vectors, d = 1536 (Gaussian mixture, bf16),
TurboQuant_prod b = 2 with dense Pi and S (bf16) on the tensor core, 1000 queries, top-10.

The whole database is encoded and searched on the GPU in the launch configuration of a user
call. The oracle re-encodes two sampled blocks of 65536 vectors and checks their planes under
the band rule; for sampled queries it recomputes the estimates of the returned keys, and
checks that no key of the sampled blocks beats the returned 10th estimate.
"""
import numpy as np
import pytest

import synth
from oracle import quantizer as OQ
from parity import ABS_SCORE, Pair, check_codes

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
tq = pytest.importorskip("vector_quantization_tq_b200")

N, D, NQ, K, BLK = 1_000_000, 1536, 1000, 10, 65536


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


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
    assert np.all(np.diff(gv, axis=1) <= ABS_SCORE)
    qv = synth.bf16_from_bits(qbits)

    sample_q = [0, 417, 999]
    for blk in (3, 12):
        r0, r1 = blk * BLK, (blk + 1) * BLK
        enc = pair.encode(synth.bf16_from_bits(bits[r0:r1]))
        gpu = dict(codes=codes[r0:r1].cpu().numpy(), qjl=qjl[r0:r1].cpu().numpy(),
                   norms=norms[r0:r1].cpu().numpy(), rnorms=rnorms[r0:r1].cpu().numpy())
        bad = check_codes(pair, gpu, enc)
        est = OQ.estimate(qv[sample_q], pair.decode(enc))
        for row, i in enumerate(sample_q):
            # no key of the sampled block outside the returned ten beats the 10th estimate
            ok = ~bad
            ok[[k - r0 for k in gi[i] if r0 <= k < r1]] = False
            assert np.max(est[row][ok]) <= gv[i, -1] + ABS_SCORE
    # the returned keys' estimates, recomputed by the oracle
    for i in sample_q:
        keys = gi[i]
        enc = pair.encode(synth.bf16_from_bits(bits[keys]))
        est = OQ.estimate(qv[i:i + 1], pair.decode(enc))[0]
        np.testing.assert_allclose(gv[i], est, atol=ABS_SCORE)
