"""The boundary's ownership rule: after a state (or split) exists, no call allocates device memory.

Every call that needs scratch space takes a caller workspace sized by its *_workspace query.
Each case below allocates all buffers and workspaces with torch first, makes one warm-up
call (the first launch of a kernel may load its module, which takes device memory once per
process), then checks that a second call leaves the device's free memory exactly where it
was (cudaMemGetInfo through torch), so no allocation was made or kept by the library.
"""
import numpy as np
import pytest

import synth
from parity import Pair

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
tq = pytest.importorskip("vector_quantization_tq_b200")


def _no_alloc(call):
    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    tq.device_status(0)
    assert free1 == free0, f"device free memory moved by {free0 - free1} bytes"


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _u8(nbytes):
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("rot", [tq.ROT_DENSE, tq.ROT_RHT])
def test_wide_encoder_works_in_the_caller_workspace(rot):
    # d = 1536 prod: the two-pass tensor-core encoders keep the residual in the workspace
    d, n = 1536, 3000
    pair = Pair(tq, d, 2, tq.PROD, rot, tq.BF16)
    x = _bf16(synth.mixture_vectors(n, d)[0])
    planes = pair.st.empty_planes(n)
    need = tq.quantize_workspace(pair.st, n, tq.BF16)
    assert need > 0
    ws = _u8(need)
    _no_alloc(lambda: tq.quantize_prod(pair.st, x, *planes, workspace=ws))
    # a workspace for fewer vectors than n still works (more passes), same planes
    small = _u8(tq.quantize_workspace(pair.st, 200, tq.BF16))
    planes2 = pair.st.empty_planes(n)
    tq.quantize_prod(pair.st, x, *planes2, workspace=small)
    torch.cuda.synchronize()
    for a, b in zip(planes, planes2):
        assert torch.equal(a, b)
    # below the minimum (128 vectors): TQ_ENOMEM before any launch
    with pytest.raises(tq.TQError) as e:
        tq.quantize_prod(pair.st, x, *planes2, workspace=_u8(tq.quantize_workspace(pair.st, 64, tq.BF16)))
    assert e.value.status == 3


def test_table_scorer_and_attention_work_in_the_caller_workspace():
    d, H, T = 128, 4, 3000
    kp = Pair(tq, d, 3, tq.PROD, tq.ROT_RHT, tq.BF16)
    vp = Pair(tq, d, 3, tq.MSE, tq.ROT_RHT, tq.BF16)
    kx = _bf16(synth.kv_prefill_batch(H, T, d).reshape(H * T, d))
    kpl, vpl = kp.st.empty_planes(H * T), vp.st.empty_planes(H * T)
    tq.quantize_prod(kp.st, kx, *kpl)
    tq.quantize_mse(vp.st, kx, vpl[0], vpl[2])
    q = _bf16(synth.decode_queries(H, d))
    scores = torch.empty((H, 1, T), dtype=torch.float32, device="cuda")
    ws = _u8(tq.score_workspace(kp.st, H, 1))
    _no_alloc(lambda: tq.score(kp.st, q, *kpl, scores, groups=H, nq=1, n=T, workspace=ws))
    out = torch.empty((H, d), dtype=torch.float32, device="cuda")
    aws = _u8(tq.attend_workspace(kp.st, vp.st, H, T))
    _no_alloc(lambda: tq.attend_decode(kp.st, vp.st, q, kpl[0], kpl[1], kpl[2], kpl[3], vpl[0], vpl[2],
                                       d ** -0.5, out, aws, H=H, T=T))
    with pytest.raises(tq.TQError) as e:
        tq.score(kp.st, q, *kpl, scores, groups=H, nq=1, n=T, workspace=_u8(256))
    assert e.value.status == 3


def test_split_score_and_search_work_in_the_caller_workspace():
    d, n = 128, 2000
    po = Pair(tq, 32, 3, tq.PROD, tq.ROT_DENSE, tq.F32, seed_pi=30, seed_s=31)
    pi = Pair(tq, 96, 2, tq.PROD, tq.ROT_DENSE, tq.F32, seed_pi=32, seed_s=33)
    sp = tq.Split(po.st, pi.st, np.arange(0, 128, 4))
    x = torch.from_numpy(synth.gaussian_vectors(n, d, seed=5).astype(np.float32)).cuda()
    pl_o, pl_i = sp.empty_planes(n)
    tq.split_quantize(sp, x, pl_o, pl_i)
    q = torch.from_numpy(synth.gaussian_vectors(3, d, seed=6).astype(np.float32)).cuda()
    scores = torch.empty((3, n), dtype=torch.float32, device="cuda")
    ws = _u8(tq.split_score_workspace(sp, tq.F32, 1, 3))
    _no_alloc(lambda: tq.split_score(sp, q, pl_o, pl_i, scores, workspace=ws))
    sp.close()

    st = Pair(tq, 256, 2, tq.PROD, tq.ROT_DENSE, tq.BF16)
    xb = _bf16(synth.mixture_vectors(n, 256, centres=16)[0])
    planes = st.st.empty_planes(n)
    tq.quantize_prod(st.st, xb, *planes)
    qb = _bf16(synth.mixture_vectors(5, 256, seed=91, centres=16, centre_seed=synth.SEED_DATA)[0])
    idx = torch.empty((5, 10), dtype=torch.int64, device="cuda")
    vals = torch.empty((5, 10), dtype=torch.float32, device="cuda")
    sws = _u8(tq.search_workspace(st.st, 5, n, 10))
    _no_alloc(lambda: tq.search_topk(st.st, qb, *planes, 10, idx, vals, sws))
