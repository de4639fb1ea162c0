"""Parity at full workload sizes, in the launch configuration the bench uses.

* Keys [1, 32, 32768, 128] bf16, TurboQuant_prod b=3 with RHT and S bf16: the whole batch is
  encoded in one call (as in bench.py); two heads are regenerated on the host and checked
  against the oracle under the band rule, together with their decode scores.
* Decode attention over 32 heads x 131072 tokens (K prod b=4, V mse b=4, dense Pi): the whole
  cache is encoded and attended on the GPU; for two heads the oracle's planes replace the
  library's, and those heads' outputs are checked against the oracle's attention.
  All heads are checked for finiteness and for |out| <= max_t |v~_t|.
"""
import math

import numpy as np
import pytest

import synth
from oracle import attention as OA
from oracle import quantizer as OQ
from parity import ABS_SCORE, Pair, check_codes

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
tq = pytest.importorskip("vector_quantization_tq_b200")


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def test_c2_full_batch_sampled_heads():
    H, T, d = 32, 32768, 128
    pair = Pair(tq, d, 3, tq.PROD, tq.ROT_RHT, tq.BF16)
    bits = synth.kv_prefill_batch(H, T, d).reshape(H * T, d)
    x = _bf16_dev(bits)
    codes, qjl, norms, rnorms = pair.st.empty_planes(H * T)
    tq.quantize_prod(pair.st, x, codes, qjl, norms, rnorms)
    qb = synth.decode_queries(H, d)
    scores = torch.empty((H, 1, T), dtype=torch.float32, device="cuda")
    tq.score(pair.st, _bf16_dev(qb), codes, qjl, norms, rnorms, scores, groups=H, nq=1, n=T)
    torch.cuda.synchronize()
    tq.device_status(0)
    qv = synth.bf16_from_bits(qb)
    for h in (0, 19):
        sl = slice(h * T, (h + 1) * T)
        hb = synth.kv_prefill_batch(H, T, d, head_range=(h, h + 1))[0]
        np.testing.assert_array_equal(hb, bits[sl])
        enc = pair.encode(synth.bf16_from_bits(hb))
        gpu = dict(codes=codes[sl].cpu().numpy(), qjl=qjl[sl].cpu().numpy(), norms=norms[sl].cpu().numpy(),
                   rnorms=rnorms[sl].cpu().numpy())
        bad = check_codes(pair, gpu, enc)
        est = OQ.estimate(qv[h:h + 1], pair.decode(enc))[0]
        got = scores[h, 0].cpu().numpy()
        assert np.max(np.abs(got - est)[~bad]) <= ABS_SCORE


def test_c3_full_cache_attention():
    H, T, d = 32, 131072, 128
    kp = Pair(tq, d, 4, tq.PROD, tq.ROT_DENSE, tq.F32)
    vp = Pair(tq, d, 4, tq.MSE, tq.ROT_DENSE, tq.F32)
    kc, kz, kn, kr = kp.st.empty_planes(H * T)
    vc, _, vn, _ = vp.st.empty_planes(H * T)
    for h in range(H):                        # encode head by head (bounded host memory)
        K = torch.from_numpy(synth.unit_vectors(T, d, seed=synth.SEED_DATA, stream=h)).cuda()
        V = torch.from_numpy(synth.unit_vectors(T, d, seed=synth.SEED_DATA + 5, stream=h)).cuda()
        sl = slice(h * T, (h + 1) * T)
        tq.quantize_prod(kp.st, K, kc[sl], kz[sl], kn[sl], kr[sl])
        tq.quantize_mse(vp.st, V, vc[sl], vn[sl])
    checked = (3, 28)
    want = {}
    for h in checked:                         # the oracle's planes for the checked heads
        K = synth.unit_vectors(T, d, seed=synth.SEED_DATA, stream=h).astype(np.float64)
        V = synth.unit_vectors(T, d, seed=synth.SEED_DATA + 5, stream=h).astype(np.float64)
        ke, ve = kp.encode(K), vp.encode(V)
        kpk, vpk = kp.packed(ke), vp.packed(ve)
        sl = slice(h * T, (h + 1) * T)
        kc[sl] = torch.from_numpy(kpk["codes"]).cuda()
        kz[sl] = torch.from_numpy(kpk["qjl"]).cuda()
        kn[sl] = torch.from_numpy(kpk["norms"]).cuda()
        kr[sl] = torch.from_numpy(kpk["rnorms"]).cuda()
        vc[sl] = torch.from_numpy(vpk["codes"]).cuda()
        vn[sl] = torch.from_numpy(vpk["norms"]).cuda()
        want[h] = (kp.decode(ke), vp.decode(ve))
    qb = synth.decode_queries(H, d)
    qv = synth.bf16_from_bits(qb)
    out = torch.empty((H, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.attend_workspace(kp.st, vp.st, H, T), dtype=torch.uint8, device="cuda")
    scale = 1.0 / math.sqrt(d)
    tq.attend_decode(kp.st, vp.st, _bf16_dev(qb), kc, kz, kn, kr, vc, vn, scale, out, ws, H=H, T=T)
    torch.cuda.synchronize()
    tq.device_status(0)
    o = out.cpu().numpy()
    assert np.all(np.isfinite(o))
    for h in checked:
        kt, vt = want[h]
        ref = OA.decode_attention(qv[h:h + 1], kt[None], vt[None], scale)[0]
        assert np.max(np.abs(o[h] - ref)) <= ABS_SCORE
        assert np.linalg.norm(o[h]) <= np.max(np.linalg.norm(vt, axis=1)) * (1 + 1e-5)
