"""Decode attention with grouped queries over a cache with room to grow, and the streaming
(append-then-attend) decode step, on the GPU against the oracle.

TurboQuant review (Jump2Paper): the method is online (each new KV vector is quantized as it
arrives, no data-dependent tuning); the attention form is the PolarQuant review's. The
oracle reconstructs K and V from the library's planes (encode parity is covered by the
parity tests) and runs decode_attention with query head h reading KV head h / G.
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

D = 128


def _states(kb=4, vb=4):
    kp = Pair(tq, D, kb, tq.PROD, tq.ROT_DENSE, tq.F32, seed_pi=40, seed_s=41)
    vp = Pair(tq, D, vb, tq.MSE, tq.ROT_DENSE, tq.F32, seed_pi=42)
    return kp, vp


def _decode_rows(pair, planes, rows):
    codes, qjl, norms, rnorms = [None if t is None else t.cpu().numpy() for t in planes]
    c = unpack(codes[rows], pair.b_mse, D) if pair.b_mse > 0 else np.zeros((len(rows), D), np.int64)
    nu = norms[rows].astype(np.float64)
    if pair.mode == tq.MSE:
        return OQ.decode_mse(c, nu, pair.Pi, pair.cb)
    z = unpack(qjl[rows], 1, D)
    return OQ.decode_prod(c, z, nu, rnorms[rows].astype(np.float64), pair.Pi, pair.S, pair.cb)


def _cache(kp, vp, Hkv, T, Tcap, seed):
    """Planes [Hkv][Tcap] with the first T rows of every head encoded from unit vectors."""
    kpl, vpl = kp.st.empty_planes(Hkv * Tcap), vp.st.empty_planes(Hkv * Tcap)
    k = synth.unit_vectors(Hkv * T, D, seed=seed).reshape(Hkv, T, D)
    v = synth.unit_vectors(Hkv * T, D, seed=seed + 1).reshape(Hkv, T, D)
    for g in range(Hkv):
        sl = slice(g * Tcap, g * Tcap + T)
        kc, kz, kn, kr = kpl
        tq.quantize_prod(kp.st, torch.from_numpy(k[g]).cuda(), kc[sl], kz[sl], kn[sl], kr[sl])
        vc, _, vn, _ = vpl
        tq.quantize_mse(vp.st, torch.from_numpy(v[g]).cuda(), vc[sl], vn[sl])
    return kpl, vpl


def _oracle(kp, vp, kpl, vpl, q, G, T, Tcap, scale):
    H = q.shape[0]
    Hkv = H // G
    kt = np.stack([_decode_rows(kp, kpl, np.arange(g * Tcap, g * Tcap + T)) for g in range(Hkv)])
    vt = np.stack([_decode_rows(vp, vpl, np.arange(g * Tcap, g * Tcap + T)) for g in range(Hkv)])
    return OA.decode_attention(q, np.repeat(kt, G, axis=0), np.repeat(vt, G, axis=0), scale)


@pytest.mark.parametrize("H,G,T,Tcap", [(8, 4, 700, 1000), (6, 3, 257, 300), (4, 1, 513, 516)])
def test_grouped_decode(H, G, T, Tcap):
    kp, vp = _states()
    kpl, vpl = _cache(kp, vp, H // G, T, Tcap, seed=70)
    q = synth.gaussian_vectors(H, D, seed=71).astype(np.float32)
    out = torch.empty((H, D), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.attend_workspace(kp.st, vp.st, H, T), dtype=torch.uint8, device="cuda")
    scale = 1.0 / np.sqrt(D)
    tq.attend_decode_grouped(kp.st, vp.st, torch.from_numpy(q).cuda(), G, T, Tcap, kpl[0], kpl[1], kpl[2], kpl[3],
                             vpl[0], vpl[2], scale, out, ws)
    torch.cuda.synchronize()
    tq.device_status(0)
    want = _oracle(kp, vp, kpl, vpl, q, G, T, Tcap, scale)
    assert np.max(np.abs(out.cpu().numpy() - want)) <= ABS_SCORE


def test_append_then_attend_over_steps():
    H, G, T0, Tcap, steps = 8, 2, 300, 320, 3
    Hkv = H // G
    kp, vp = _states()
    kpl, vpl = _cache(kp, vp, Hkv, T0, Tcap, seed=80)
    scale = 1.0 / np.sqrt(D)
    for step in range(steps):
        T = T0 + step
        q = synth.gaussian_vectors(H, D, seed=90 + step).astype(np.float32)
        kn = synth.unit_vectors(Hkv, D, seed=100 + step)
        vn = synth.unit_vectors(Hkv, D, seed=200 + step)
        out = torch.empty((H, D), dtype=torch.float32, device="cuda")
        ws = torch.empty(tq.attend_workspace(kp.st, vp.st, H, T + 1), dtype=torch.uint8, device="cuda")
        tq.attend_append_decode(kp.st, vp.st, torch.from_numpy(q).cuda(), G, torch.from_numpy(kn).cuda(),
                                torch.from_numpy(vn).cuda(), T, Tcap, kpl[0], kpl[1], kpl[2], kpl[3], vpl[0],
                                vpl[2], scale, out, ws)
        torch.cuda.synchronize()
        tq.device_status(0)
        # the appended rows are the encodings of the new vectors
        rows = np.arange(Hkv) * Tcap + T
        enc_k, enc_v = kp.encode(kn.astype(np.float64)), vp.encode(vn.astype(np.float64))
        gk = dict(codes=kpl[0].cpu().numpy()[rows], qjl=kpl[1].cpu().numpy()[rows],
                  norms=kpl[2].cpu().numpy()[rows], rnorms=kpl[3].cpu().numpy()[rows])
        gv = dict(codes=vpl[0].cpu().numpy()[rows], norms=vpl[2].cpu().numpy()[rows])
        check_codes(kp, gk, enc_k)
        check_codes(vp, gv, enc_v)
        want = _oracle(kp, vp, kpl, vpl, q, G, T + 1, Tcap, scale)
        assert np.max(np.abs(out.cpu().numpy() - want)) <= ABS_SCORE


def test_grouped_rejects_bad_shapes():
    kp, vp = _states()
    kpl, vpl = _cache(kp, vp, 2, 10, 16, seed=5)
    q = torch.zeros((6, D), dtype=torch.float32, device="cuda")
    out = torch.empty((6, D), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.attend_workspace(kp.st, vp.st, 6, 10) + 256, dtype=torch.uint8, device="cuda")
    for G, T, Tcap in ((4, 10, 16), (3, 17, 16), (0, 10, 16)):   # H % G, T > Tcap, G = 0
        with pytest.raises(tq.TQError):
            tq.attend_decode_grouped(kp.st, vp.st, q, G, T, Tcap, kpl[0], kpl[1], kpl[2], kpl[3], vpl[0], vpl[2],
                                     0.1, out, ws)
