"""Prefix coding of the codebook indices on the GPU against the oracle (oracle/entropy.py).

TurboQuant review (Jump2Paper), limitations: an optimal prefix code on the b = 4 indices
averages about 3.8 bits. Integer work, so the check is bit-exact: the stream bytes and the
offsets equal the oracle's for the same codes, and decoding returns the codes. At a size the
pure-Python oracle cannot walk (more than 1024 blocks, so the scan of block totals takes
several passes), the offsets are checked against vectorised length sums and the round trip
is exact.
"""
import numpy as np
import pytest

import synth
from oracle import entropy as EN
from parity import unpack

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
tq = pytest.importorskip("vector_quantization_tq_b200")

D = 128


def _codes_planes(st, n, seed):
    """Codes of n unit vectors encoded by the library (MSE state)."""
    x = torch.from_numpy(synth.unit_vectors(n, D, seed=seed)).cuda()
    codes, _, norms, _ = st.empty_planes(n)
    tq.quantize_mse(st, x, codes, norms)
    return codes


def _run(st, codes):
    n = codes.shape[0]
    offsets = torch.empty(n + 1, dtype=torch.int64, device="cuda")
    stream = torch.empty(tq.entropy_max_bytes(st, n), dtype=torch.uint8, device="cuda")
    ws = torch.empty(tq.entropy_workspace(st, n), dtype=torch.uint8, device="cuda")
    tq.entropy_encode(st, codes, offsets, stream, ws)
    back = torch.empty_like(codes)
    tq.entropy_decode(st, stream, offsets, back)
    torch.cuda.synchronize()
    tq.device_status(0)
    return offsets.cpu().numpy(), stream.cpu().numpy(), back


@pytest.mark.parametrize("b,n", [(4, 5000), (3, 1), (2, 1500), (4, 1025)])
def test_stream_matches_oracle(b, n):
    st = tq.State(D, b, tq.MSE, tq.ROT_RHT, tq.F32, signs=synth.rht_signs(D))
    codes = _codes_planes(st, n, seed=300 + b)
    off, stream, back = _run(st, codes)
    ln, w, _ = tq.entropy_table(st)
    c = unpack(codes.cpu().numpy(), b, D)
    o_stream, o_off = EN.encode(c, ln, w)
    np.testing.assert_array_equal(off, o_off)
    np.testing.assert_array_equal(stream[:len(o_stream)], o_stream)
    assert not stream[len(o_stream):].any()
    assert torch.equal(back, codes)
    st.close()


def test_large_batch_offsets_and_round_trip():
    b, n = 4, 1_100_000            # 1075 blocks of 1024 vectors: the totals scan wraps
    st = tq.State(D, b, tq.MSE, tq.ROT_RHT, tq.F32, signs=synth.rht_signs(D))
    codes = _codes_planes(st, n, seed=310)
    off, stream, back = _run(st, codes)
    ln, _, mean = tq.entropy_table(st)
    lengths = np.asarray(ln)[unpack(codes.cpu().numpy(), b, D)].sum(axis=1)
    np.testing.assert_array_equal(np.diff(off), lengths)
    assert off[0] == 0 and off[-1] == lengths.sum()
    assert torch.equal(back, codes)
    # the measured width is the law's mean within sampling noise, about 4.5 % under 4 bits
    assert abs(off[-1] / (n * D) - mean) < 0.01
    st.close()
