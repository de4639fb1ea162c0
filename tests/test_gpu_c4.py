"""Distortion / bias sweep on the GPU (2^20 uniform unit vectors, d = 128 and 256, b = 1..4,
MSE and prod, 1024 unit queries), and parity of the statistics kernel with the oracle.

Checks follow the TurboQuant review (Jump2Paper): Theorem 1 (D_mse = d C(f_X, b), between
the lower bound 4^-b and sqrt(3) pi / 2 4^-b), the 1-bit 2/pi bias and the slope 1 - D_mse
of the MSE quantizer, Theorem 2 (the prod estimate is unbiased).
If TQ_C4_REPORT is set, the sweep's numbers are written there as JSON.
"""
import json
import math
import os

import numpy as np
import pytest

import synth
from oracle import quantizer as OQ
from parity import Pair

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
tq = pytest.importorskip("vector_quantization_tq_b200")


def _encode_decode(pair, x_dev):
    n = x_dev.shape[0]
    codes, qjl, norms, rnorms = pair.st.empty_planes(n)
    if pair.mode == tq.MSE:
        tq.quantize_mse(pair.st, x_dev, codes, norms)
    else:
        tq.quantize_prod(pair.st, x_dev, codes, qjl, norms, rnorms)
    xt = torch.empty_like(x_dev)
    tq.dequant(pair.st, codes, qjl, norms, rnorms, xt)
    return xt


def _stats(x, xt, q):
    out = torch.zeros(6, dtype=torch.float64, device="cuda")
    tq.ip_stats(x, xt, q, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_stats_kernel_matches_oracle():
    d, n, nq = 128, 4096, 64
    pair = Pair(tq, d, 3, tq.PROD, tq.ROT_DENSE, tq.F32)
    x = synth.unit_vectors(n, d, seed=70)
    q = synth.unit_vectors(nq, d, seed=71)
    enc = pair.encode(x.astype(np.float64))
    xt_o = pair.decode(enc)
    # the GPU statistics of the oracle's reconstruction, against the same sums in fp64
    got = _stats(torch.from_numpy(x).cuda(), torch.from_numpy(xt_o.astype(np.float32)).cuda(),
                 torch.from_numpy(q).cuda())
    xf, tf, qf = x.astype(np.float64), xt_o.astype(np.float32).astype(np.float64), q.astype(np.float64)
    a, b = qf @ xf.T, qf @ tf.T
    want = [np.sum((xf - tf) ** 2), np.sum(xf ** 2), np.sum(b - a), np.sum((b - a) ** 2), np.sum(a * b),
            np.sum(a * a)]
    np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("d", [128, 256])
def test_distortion_bias_sweep(d):
    n, nq = 1 << 20, 1024
    x = torch.from_numpy(synth.unit_vectors(n, d, seed=80 + d)).cuda()
    q = torch.from_numpy(synth.unit_vectors(nq, d, seed=81 + d)).cuda()
    report = []
    for mode in (tq.MSE, tq.PROD):
        for b in (1, 2, 3, 4):
            pair = Pair(tq, d, b, mode, tq.ROT_DENSE, tq.F32)
            xt = _encode_decode(pair, x)
            s = _stats(x, xt, q)
            tq.device_status(0)
            D = s[0] / n
            slope = s[4] / s[5]
            mean_e = s[2] / (n * nq)
            sd_e = math.sqrt(s[3] / (n * nq) - mean_e ** 2)
            row = dict(d=d, b=b, mode="mse" if mode == tq.MSE else "prod", D=D, slope=slope, mean_err=mean_e,
                       sd_err=sd_e)
            report.append(row)
            if mode == tq.MSE:
                Da = pair.cb.dmse
                assert abs(D / Da - 1) < 0.01, row                        # Theorem 1
                assert 4.0 ** (-b) <= D <= math.sqrt(3) * math.pi / 2 * 4.0 ** (-b), row
                assert abs(slope - (1 - Da)) < 0.01, row                   # bias 1 - D_mse
                if b == 1:
                    assert abs(slope - 2 / math.pi) < 0.005, row           # the printed 2/pi
            else:
                # unbiased: the mean error over pairs is within 3 standard errors counted per vector
                assert abs(mean_e) < 3 * sd_e / math.sqrt(n), row          # Theorem 2
                assert abs(slope - 1) < 0.01, row
                Dm1 = pair.cb.dmse if pair.cb is not None else 1.0
                assert sd_e ** 2 <= math.pi / (2 * d) * Dm1 * 1.05, row    # D_prod bound
    path = os.environ.get("TQ_C4_REPORT")
    if path:
        old = json.load(open(path)) if os.path.exists(path) else []
        json.dump(old + report, open(path, "w"), indent=1)
