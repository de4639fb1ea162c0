"""Outlier-channel split on the GPU against the oracle.

TurboQuant review (Jump2Paper), experiment settings ("KV bit settings", "outlier handling"):
the outlier channels and the rest are two independent quantizers at their own bit widths.
The oracle side is oracle/mixed.py (split / merge / outlier choice) around the plain
quantizer of each group; the comparison rules are those of parity.py, applied per group.
"""
import numpy as np
import pytest

import synth
from oracle import mixed as OM
from oracle import quantizer as OQ
from parity import ABS_SCORE, REL_L2, Pair, check_codes, rel_l2, unpack

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
tq = pytest.importorskip("vector_quantization_tq_b200")

# (d, outlier channels m, outlier bits, other bits, mode, rotation, matrix dtype): the stated
# 32@3 + 96@2 split (dense and with the groups' Hadamard transforms, orders 32 and 12 x 8),
# a 2.5-bit split, an MSE split, and a wider head.
CASES = [(128, 32, 3, 2, 1, 0, 0), (128, 32, 3, 2, 1, 1, 1), (128, 32, 4, 2, 1, 0, 0), (128, 32, 3, 2, 0, 0, 0),
         (256, 64, 4, 3, 1, 0, 0)]
# Splits of 128 bf16 channels whose groups are Hadamard-rotated at 1 or 2 code bits run on the
# tensor-core encoder: the 32@3 + 96@2 split over several tiles per SM, a 64 + 64 MSE split,
# and a 96-channel outer group.
TC_CASES = [(128, 32, 3, 2, 1, 1, 1, 148 * 128 * 3 + 5), (128, 64, 2, 1, 0, 1, 1, 20000),
            (128, 96, 2, 3, 1, 1, 1, 9001)]


def _host(planes):
    codes, qjl, norms, rnorms = planes
    out = dict(codes=codes.cpu().numpy(), norms=norms.cpu().numpy())
    if qjl is not None:
        out.update(qjl=qjl.cpu().numpy(), rnorms=rnorms.cpu().numpy())
    return out


@pytest.mark.parametrize("d,m,bo,br,mode,rot,md", CASES)
@pytest.mark.parametrize("n", [3001])
def test_split_encode_dequant_score(d, m, bo, br, mode, rot, md, n):
    _split_case(d, m, bo, br, mode, rot, md, n)


@pytest.mark.parametrize("d,m,bo,br,mode,rot,md,n", TC_CASES)
def test_split_tensor_core_encoder(d, m, bo, br, mode, rot, md, n):
    _split_case(d, m, bo, br, mode, rot, md, n)


def _split_case(d, m, bo, br, mode, rot, md, n):
    bits = synth.kv_prefill_batch(1, n, d, seed=51)[0]
    x = synth.bf16_from_bits(bits).astype(np.float64)
    ch = OM.outlier_channels(x, m)
    po = Pair(tq, m, bo, mode, rot, md, seed_pi=20, seed_s=21)
    pr = Pair(tq, d - m, br, mode, rot, md, seed_pi=22, seed_s=23)
    sp = tq.Split(po.st, pr.st, ch)
    x_dev = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    pl_o, pl_r = sp.empty_planes(n)
    tq.split_quantize(sp, x_dev, pl_o, pl_r)
    torch.cuda.synchronize()
    tq.device_status(0)

    xo, xr = OM.split(x, ch)
    enc_o, enc_r = po.encode(xo), pr.encode(xr)
    bad = check_codes(po, _host(pl_o), enc_o) | check_codes(pr, _host(pl_r), enc_r)
    assert bad.mean() < 0.01

    want = OM.merge(po.decode(enc_o), pr.decode(enc_r), ch, d)
    out = torch.empty((n, d), dtype=torch.float32, device="cuda")
    tq.split_dequant(sp, pl_o, pl_r, out)
    got = out.cpu().numpy()
    assert np.max(rel_l2(got[~bad], want[~bad])) <= REL_L2

    nq = 5
    q = synth.gaussian_vectors(nq, d, seed=52).astype(np.float32)
    scores = torch.empty((nq, n), dtype=torch.float32, device="cuda")
    tq.split_score(sp, torch.from_numpy(q).cuda(), pl_o, pl_r, scores)
    est = OQ.estimate(q.astype(np.float64), want)
    assert np.max(np.abs(scores.cpu().numpy() - est)[:, ~bad]) <= ABS_SCORE
    sp.close()


def test_split_rejects_bad_channel_lists():
    po = Pair(tq, 32, 3, tq.PROD, tq.ROT_DENSE, tq.F32)
    pr = Pair(tq, 96, 2, tq.PROD, tq.ROT_DENSE, tq.F32)
    pm = Pair(tq, 96, 2, tq.MSE, tq.ROT_DENSE, tq.F32)
    good = np.arange(0, 128, 4)
    tq.Split(po.st, pr.st, good).close()
    for ch in (good[::-1], np.r_[good[:-1], good[-2]], np.r_[good[:-1], 128], good[:-1]):
        with pytest.raises(tq.TQError):
            tq.Split(po.st, pr.st, ch)
    with pytest.raises(tq.TQError):   # modes differ
        tq.Split(po.st, pm.st, good)


@pytest.mark.parametrize("H,T,dv_out", [(3, 1000, 32), (2, 300, 64)])
def test_split_decode_attention(H, T, dv_out):
    # K: 32 outlier channels at prod b=4, 96 at prod b=3; V: dv_out channels at mse b=4, the
    # rest at mse b=3, with their own outlier list.
    from oracle import attention as OA
    d, mk = 128, 32
    rng = np.random.default_rng(60)
    k = rng.standard_normal((H * T, d))
    v = rng.standard_normal((H * T, d))
    k[:, [3, 70]] *= 8.0
    v[:, [5, 90, 100]] *= 6.0
    kch, vch = OM.outlier_channels(k, mk), OM.outlier_channels(v, dv_out)
    ko = Pair(tq, mk, 4, tq.PROD, tq.ROT_DENSE, tq.F32, seed_pi=30, seed_s=31)
    ki = Pair(tq, d - mk, 3, tq.PROD, tq.ROT_DENSE, tq.F32, seed_pi=32, seed_s=33)
    vo = Pair(tq, dv_out, 4, tq.MSE, tq.ROT_DENSE, tq.F32, seed_pi=34)
    vi = Pair(tq, d - dv_out, 3, tq.MSE, tq.ROT_DENSE, tq.F32, seed_pi=35)
    ks, vs = tq.Split(ko.st, ki.st, kch), tq.Split(vo.st, vi.st, vch)
    kpl, vpl = ks.empty_planes(H * T), vs.empty_planes(H * T)
    tq.split_quantize(ks, torch.from_numpy(k.astype(np.float32)).cuda(), *kpl)
    tq.split_quantize(vs, torch.from_numpy(v.astype(np.float32)).cuda(), *vpl)
    q = rng.standard_normal((H, d)).astype(np.float32)
    out = torch.empty((H, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.split_attend_workspace(ks, vs, H, T), dtype=torch.uint8, device="cuda")
    scale = 1.0 / np.sqrt(d)
    tq.split_attend_decode(ks, vs, torch.from_numpy(q).cuda(), kpl, vpl, scale, out, ws, H=H, T=T)
    torch.cuda.synchronize()
    tq.device_status(0)
    # the oracle from the library's own planes (encode parity is covered above), decoded per group
    def dec(pair, pl):
        g = _host(pl)
        codes = unpack_planes(pair, g)
        if pair.mode == tq.MSE:
            return OQ.decode_mse(codes, g["norms"].astype(np.float64), pair.Pi, pair.cb)
        z = unpack(g["qjl"], 1, pair.d)
        return OQ.decode_prod(codes, z, g["norms"].astype(np.float64), g["rnorms"].astype(np.float64), pair.Pi,
                              pair.S, pair.cb)
    kt = OM.merge(dec(ko, kpl[0]), dec(ki, kpl[1]), kch, d).reshape(H, T, d)
    vt = OM.merge(dec(vo, vpl[0]), dec(vi, vpl[1]), vch, d).reshape(H, T, d)
    want = OA.decode_attention(q, kt, vt, scale)
    assert np.max(np.abs(out.cpu().numpy() - want)) <= ABS_SCORE
    ks.close()
    vs.close()


def unpack_planes(pair, g):
    from parity import unpack as _unpack
    return _unpack(g["codes"], pair.b_mse, pair.d) if pair.b_mse > 0 else np.zeros((len(g["norms"]), pair.d),
                                                                                     np.int64)
