"""The decode-attention entry point that allocates nothing (tq_attend_decode_noalloc).

Some callers cannot allocate device memory: runtimes whose own pool allocator owns all
device memory, and latency-critical decode loops where an allocation is not acceptable.
For them the library keeps the split partials in a fixed device array. This test calls
that entry point through the C ABI twice in a row and checks each result against the
workspace-taking tq_attend_decode on the same inputs, within the parity tolerance.
It lives in a file of its own so that it is collected last.
"""
import math

import numpy as np
import pytest

import synth
from parity import ABS_SCORE, Pair

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

tq = pytest.importorskip("vector_quantization_tq_b200")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_noalloc_matches_workspace_entry_point_twice():
    d, H, T = 128, 4, 2000
    kp = Pair(tq, d, 4, tq.PROD, tq.ROT_DENSE, tq.F32)
    vp = Pair(tq, d, 4, tq.MSE, tq.ROT_DENSE, tq.F32)
    K = synth.unit_vectors(H * T, d, seed=synth.SEED_DATA + 20)
    V = synth.unit_vectors(H * T, d, seed=synth.SEED_DATA + 21)
    kpk, vpk = kp.packed(kp.encode(K.astype(np.float64))), vp.packed(vp.encode(V.astype(np.float64)))
    kc, kz, kn, kr = (_dev(kpk[k]) for k in ("codes", "qjl", "norms", "rnorms"))
    vc, vn = _dev(vpk["codes"]), _dev(vpk["norms"])
    qb = synth.decode_queries(H, d)
    q = _dev(qb.view(np.int16)).view(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)

    ref = torch.empty((H, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.attend_workspace(kp.st, vp.st, H, T), dtype=torch.uint8, device="cuda")
    tq.attend_decode(kp.st, vp.st, q, kc, kz, kn, kr, vc, vn, scale, ref, ws, H=H, T=T)
    torch.cuda.synchronize()
    want = ref.cpu().numpy()

    for _ in range(2):   # the second call reuses the fixed scratch left by the first
        out = torch.full((H, d), float("nan"), dtype=torch.float32, device="cuda")
        tq.attend_decode_noalloc(kp.st, vp.st, q, kc, kz, kn, kr, vc, vn, scale, out, H=H, T=T)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - want)) <= ABS_SCORE


@pytest.mark.parametrize("d,kmode,rot", [(64, tq.PROD, tq.ROT_DENSE), (256, tq.MSE, tq.ROT_RHT)])
def test_noalloc_general_kernel_twice(d, kmode, rot):
    # d != 128 runs the general attention kernel: the fixed array then holds only partials
    H, T = 3, 1500
    kp = Pair(tq, d, 3, kmode, rot, tq.F32)
    vp = Pair(tq, d, 3, tq.MSE, rot, tq.F32)
    K = synth.unit_vectors(H * T, d, seed=synth.SEED_DATA + 22)
    V = synth.unit_vectors(H * T, d, seed=synth.SEED_DATA + 23)
    kpk, vpk = kp.packed(kp.encode(K.astype(np.float64))), vp.packed(vp.encode(V.astype(np.float64)))
    kc, kn = _dev(kpk["codes"]), _dev(kpk["norms"])
    kz = _dev(kpk["qjl"]) if kmode == tq.PROD else None
    kr = _dev(kpk["rnorms"]) if kmode == tq.PROD else None
    vc, vn = _dev(vpk["codes"]), _dev(vpk["norms"])
    q = _dev(synth.gaussian_vectors(H, d, seed=24).astype(np.float32))
    scale = 1.0 / math.sqrt(d)
    ref = torch.empty((H, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.attend_workspace(kp.st, vp.st, H, T), dtype=torch.uint8, device="cuda")
    tq.attend_decode(kp.st, vp.st, q, kc, kz, kn, kr, vc, vn, scale, ref, ws, H=H, T=T)
    torch.cuda.synchronize()
    want = ref.cpu().numpy()
    for _ in range(2):
        out = torch.full((H, d), float("nan"), dtype=torch.float32, device="cuda")
        tq.attend_decode_noalloc(kp.st, vp.st, q, kc, kz, kn, kr, vc, vn, scale, out, H=H, T=T)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - want)) <= ABS_SCORE


def test_noalloc_rejects_shapes_beyond_the_fixed_array():
    # the limit is tq_attend_workspace(ks, vs, H, T) <= 4 MiB; above it nothing is launched
    d, T = 128, 1000
    kp = Pair(tq, d, 4, tq.PROD, tq.ROT_DENSE, tq.F32)
    vp = Pair(tq, d, 4, tq.MSE, tq.ROT_DENSE, tq.F32)
    H = 8
    while tq.attend_workspace(kp.st, vp.st, H, T) <= (4 << 20):
        H *= 2
    kc, kz, kn, kr = kp.st.empty_planes(H * T)
    vc, _, vn, _ = vp.st.empty_planes(H * T)
    q = torch.zeros((H, d), dtype=torch.float32, device="cuda")
    out = torch.zeros((H, d), dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.attend_decode_noalloc(kp.st, vp.st, q, kc, kz, kn, kr, vc, vn, 0.1, out, H=H, T=T)
    assert e.value.status == 2
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
