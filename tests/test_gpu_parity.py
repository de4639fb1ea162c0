"""GPU parity: libtq kernels (through the C ABI) against the fp64 oracle, same seeded inputs.

Sizes span several tiles with ragged tails; the bar is the one stated in tests/parity.py.
"""
import math

import numpy as np
import pytest

import synth
from oracle import attention as OA
from oracle import quantizer as OQ
from parity import ABS_SCORE, REL_L2, Pair, check_codes, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

tq = pytest.importorskip("vector_quantization_tq_b200")


def dev_f32(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host(t):
    return None if t is None else t.cpu().numpy()


def gpu_encode(pair, x_dev, n=None):
    n = x_dev.shape[0] if n is None else n
    codes, qjl, norms, rnorms = pair.st.empty_planes(n)
    if pair.mode == tq.MSE:
        tq.quantize_mse(pair.st, x_dev, codes, norms)
    else:
        tq.quantize_prod(pair.st, x_dev, codes, qjl, norms, rnorms)
    torch.cuda.synchronize()
    return dict(codes=host(codes), qjl=host(qjl), norms=host(norms), rnorms=host(rnorms)), \
        (codes, qjl, norms, rnorms)


def planes_to_dev(pk):
    def t(a, dt):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t(pk["codes"], None), t(pk.get("qjl"), None), t(pk["norms"], None), t(pk.get("rnorms"), None)


def gpu_dequant(pair, planes, n):
    out = torch.empty((n, pair.d), dtype=torch.float32, device="cuda")
    tq.dequant(pair.st, *planes, out)
    torch.cuda.synchronize()
    return host(out)


def gpu_score(pair, q_dev, planes, groups=1):
    codes, qjl, norms, rnorms = planes
    n = norms.shape[0] // groups
    nq = q_dev.shape[0] // groups
    out = torch.empty((groups, nq, n), dtype=torch.float32, device="cuda")
    tq.score(pair.st, q_dev, codes, qjl, norms, rnorms, out, groups=groups, nq=nq, n=n)
    torch.cuda.synchronize()
    return host(out)


# --------------------------------------------------------------------------------------
# Config 1: TurboQuant_mse b=3, d=128, 4096 unit vectors, dense Haar Pi (seed 0),
# encode + decode + 64 queries x 4096 estimates.
# --------------------------------------------------------------------------------------
def test_c1_mse_encode_decode_score():
    pair = Pair(tq, 128, 3, tq.MSE, tq.ROT_DENSE, tq.F32)
    x = synth.unit_vectors(4096, 128, seed=synth.SEED_DATA)
    q = synth.unit_vectors(64, 128, seed=synth.SEED_DATA + 1)
    enc = pair.encode(x.astype(np.float64))
    gpu, gplanes = gpu_encode(pair, dev_f32(x))
    bad = check_codes(pair, gpu, enc)
    # decode of the oracle's planes
    pk = pair.packed(enc)
    oplanes = planes_to_dev(pk)
    xt_o = pair.decode(enc)
    xt_g = gpu_dequant(pair, oplanes, 4096)
    assert np.max(rel_l2(xt_g, xt_o)) <= REL_L2
    # decode of the library's own planes (vectors without an in-band code flip)
    xt_gg = gpu_dequant(pair, gplanes, 4096)
    assert np.max(rel_l2(xt_gg[~bad], xt_o[~bad])) <= REL_L2
    # scores from the oracle's planes against <q, x~>
    est = OQ.estimate(q, xt_o)
    sg = gpu_score(pair, dev_f32(q), oplanes)[0]
    assert np.max(np.abs(sg - est)) <= ABS_SCORE
    sgg = gpu_score(pair, dev_f32(q), gplanes)[0]
    assert np.max(np.abs(sgg[:, ~bad] - est[:, ~bad])) <= ABS_SCORE


# --------------------------------------------------------------------------------------
# Config 2 (reduced heads/tokens): TurboQuant_prod b=3, RHT, S bf16, KV-shaped bf16 keys.
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("tokens", [3000, 257])
def test_c2_prod_rht_kv_keys(tokens):
    H, d = 2, 128
    pair = Pair(tq, d, 3, tq.PROD, tq.ROT_RHT, tq.BF16)
    bits = synth.kv_prefill_batch(H, tokens, d).reshape(H * tokens, d)
    x = synth.bf16_from_bits(bits)
    enc = pair.encode(x)
    gpu, gplanes = gpu_encode(pair, dev_bf16(bits))
    bad = check_codes(pair, gpu, enc)
    pk = pair.packed(enc)
    oplanes = planes_to_dev(pk)
    xt_o = pair.decode(enc)
    assert np.max(rel_l2(gpu_dequant(pair, oplanes, H * tokens), xt_o)) <= REL_L2
    # one decode query per head against that head's keys
    qb = synth.decode_queries(H, d)
    qv = synth.bf16_from_bits(qb)
    est = np.stack([qv[h] @ xt_o[h * tokens:(h + 1) * tokens].T for h in range(H)])
    sg = gpu_score(pair, dev_bf16(qb), oplanes, groups=H)[:, 0, :]
    assert np.max(np.abs(sg - est)) <= ABS_SCORE
    sgg = gpu_score(pair, dev_bf16(qb), gplanes, groups=H)[:, 0, :]
    okk = ~bad.reshape(H, tokens)
    assert np.max(np.abs(sgg - est)[okk]) <= ABS_SCORE


# --------------------------------------------------------------------------------------
# Config 3 (reduced): fused decode attention, K prod b=4, V mse b=4, dense Pi.
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("H,T,d,rot", [(3, 1000, 128, tq.ROT_DENSE), (2, 300, 128, tq.ROT_DENSE),
                                       (2, 300, 96, tq.ROT_RHT), (2, 257, 192, tq.ROT_RHT),
                                       (2, 300, 160, tq.ROT_DENSE)])
def test_c3_decode_attention(H, T, d, rot):
    # d = 128 runs the table kernel; the other shapes the general kernel (96 and 192 with the
    # order-12 Kronecker Hadamard rotation, 160 a width that does not divide the block)
    kp = Pair(tq, d, 4, tq.PROD, rot, tq.F32)
    vp = Pair(tq, d, 4, tq.MSE, rot, tq.F32)
    K = synth.unit_vectors(H * T, d, seed=synth.SEED_DATA)
    V = synth.unit_vectors(H * T, d, seed=synth.SEED_DATA + 5)
    qb = synth.decode_queries(H, d)
    qv = synth.bf16_from_bits(qb)
    ke, ve = kp.encode(K.astype(np.float64)), vp.encode(V.astype(np.float64))
    kt, vt = kp.decode(ke), vp.decode(ve)
    scale = 1.0 / math.sqrt(d)
    want = OA.decode_attention(qv, kt.reshape(H, T, d), vt.reshape(H, T, d), scale)
    kpl, vpl = planes_to_dev(kp.packed(ke)), planes_to_dev(vp.packed(ve))
    out = torch.empty((H, d), dtype=torch.float32, device="cuda")
    wsb = tq.attend_workspace(kp.st, vp.st, H, T)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    tq.attend_decode(kp.st, vp.st, dev_bf16(qb), kpl[0], kpl[1], kpl[2], kpl[3], vpl[0], vpl[2], scale, out, ws,
                     H=H, T=T)
    torch.cuda.synchronize()
    assert np.max(np.abs(host(out) - want)) <= ABS_SCORE


def test_attention_rejects_small_workspace():
    d, H, T = 128, 2, 600
    kp = Pair(tq, d, 3, tq.MSE, tq.ROT_DENSE, tq.F32)
    vp = Pair(tq, d, 3, tq.MSE, tq.ROT_DENSE, tq.F32)
    need = tq.attend_workspace(kp.st, vp.st, H, T)
    assert need > 0
    codes = torch.zeros((H * T, kp.st.code_bytes), dtype=torch.uint8, device="cuda")
    norms = torch.ones(H * T, dtype=torch.float32, device="cuda")
    q = torch.zeros((H, d), dtype=torch.float32, device="cuda")
    out = torch.empty((H, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(need - 256 if need > 256 else 0, dtype=torch.uint8, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.attend_decode(kp.st, vp.st, q, codes, None, norms, None, codes, norms, 0.1, out, ws,
                         ws_bytes=need - 1, H=H, T=T)
    assert e.value.status == 3


# --------------------------------------------------------------------------------------
# Other dimensions and modes through the general kernels (ragged n, fp32/bf16, ld > d).
# --------------------------------------------------------------------------------------
CASES = [
    (32, 2, tq.MSE, tq.ROT_RHT, tq.F32), (64, 4, tq.PROD, tq.ROT_DENSE, tq.F32),
    (256, 1, tq.MSE, tq.ROT_DENSE, tq.F32), (256, 2, tq.PROD, tq.ROT_RHT, tq.F32),
    (256, 4, tq.PROD, tq.ROT_DENSE, tq.F32), (512, 3, tq.MSE, tq.ROT_RHT, tq.F32),
    (1536, 2, tq.PROD, tq.ROT_DENSE, tq.BF16), (128, 1, tq.PROD, tq.ROT_DENSE, tq.F32),
    (128, 6, tq.MSE, tq.ROT_DENSE, tq.F32), (2048, 1, tq.PROD, tq.ROT_RHT, tq.BF16),
    (512, 2, tq.PROD, tq.ROT_DENSE, tq.BF16), (1536, 3, tq.MSE, tq.ROT_DENSE, tq.BF16),
    (1024, 4, tq.PROD, tq.ROT_DENSE, tq.BF16),
    # Hadamard orders 12 * 2^k (Paley H_12 Kronecker Sylvester) and widths 32 k up to 256
    (96, 3, tq.PROD, tq.ROT_RHT, tq.F32), (192, 2, tq.MSE, tq.ROT_RHT, tq.F32),
    (1536, 2, tq.PROD, tq.ROT_RHT, tq.BF16), (160, 2, tq.PROD, tq.ROT_DENSE, tq.F32),
    (224, 3, tq.MSE, tq.ROT_DENSE, tq.F32),
    # d = 128 with a dense rotation and 1- to 4-bit MSE codes: the tiled CUDA-core encoder
    (128, 1, tq.MSE, tq.ROT_DENSE, tq.F32), (128, 2, tq.PROD, tq.ROT_DENSE, tq.F32),
    (128, 3, tq.MSE, tq.ROT_DENSE, tq.BF16), (128, 5, tq.PROD, tq.ROT_DENSE, tq.BF16),
    # d = 256 with a dense fp32 rotation: the streamed-matrix CUDA-core encoder
    (256, 2, tq.MSE, tq.ROT_DENSE, tq.F32), (256, 4, tq.MSE, tq.ROT_DENSE, tq.F32),
    (256, 1, tq.PROD, tq.ROT_DENSE, tq.F32), (256, 3, tq.PROD, tq.ROT_DENSE, tq.F32),
    (256, 5, tq.PROD, tq.ROT_DENSE, tq.F32),
]


@pytest.mark.parametrize("d,b,mode,rot,md", CASES)
@pytest.mark.parametrize("bf16_in", [False, True])
def test_general_paths(d, b, mode, rot, md, bf16_in):
    n = 301
    pair = Pair(tq, d, b, mode, rot, md)
    xf = synth.gaussian_vectors(n, d, seed=40 + d).astype(np.float32) * 3
    xf[7] = 0.0                                              # a zero vector
    if bf16_in:
        bits = synth.bf16_bits(xf)
        x = synth.bf16_from_bits(bits)
        pad = np.zeros((n, d + 8), np.uint16)
        pad[:, :d] = bits
        xd = dev_bf16(pad)[:, :d]                            # row stride d + 8
    else:
        x = xf.astype(np.float64)
        pad = np.zeros((n, d + 4), np.float32)
        pad[:, :d] = xf
        xd = dev_f32(pad)[:, :d]                             # row stride d + 4
    enc = pair.encode(x)
    gpu, gplanes = gpu_encode(pair, xd, n)
    bad = check_codes(pair, gpu, enc)
    assert gpu["norms"][7] == 0.0
    if mode == tq.PROD:
        assert gpu["rnorms"][7] == 0.0 and np.all(gpu["qjl"][7] == 255)
    xt_o = pair.decode(enc)
    oplanes = planes_to_dev(pair.packed(enc))
    xt_g = gpu_dequant(pair, oplanes, n)
    ok = np.ones(n, bool)
    ok[7] = False
    assert np.max(rel_l2(xt_g[ok], xt_o[ok])) <= REL_L2
    assert np.all(xt_g[7] == 0)
    q = synth.gaussian_vectors(11, d, seed=77)
    sg = gpu_score(pair, dev_f32(q), oplanes)[0]
    est = OQ.estimate(q, xt_o)
    assert np.max(np.abs(sg - est)) <= ABS_SCORE


@pytest.mark.parametrize("d,b,mode", [(128, 2, tq.MSE), (128, 4, tq.PROD), (256, 3, tq.MSE), (256, 2, tq.PROD)])
def test_dense_tiled_encoder_many_tiles(d, b, mode):
    # more tiles (128 vectors at d = 128, 64 at d = 256) than SMs, so every persistent block of
    # the tiled encoder and dequantizer walks several, plus a ragged tail
    n = 148 * 128 * 2 + 77
    pair = Pair(tq, d, b, mode, tq.ROT_DENSE, tq.F32)
    x = synth.unit_vectors(n, d, seed=321).astype(np.float32)
    enc = pair.encode(x.astype(np.float64))
    gpu, _ = gpu_encode(pair, dev_f32(x), n)
    check_codes(pair, gpu, enc)
    # the tiled dequantizer over the same tiles: the oracle's planes back to vectors
    xt_g = gpu_dequant(pair, planes_to_dev(pair.packed(enc)), n)
    assert np.max(rel_l2(xt_g, pair.decode(enc))) <= REL_L2


@pytest.mark.parametrize("b,mode", [(2, tq.PROD), (3, tq.PROD), (4, tq.MSE)])
def test_dense_gemm_encoder_many_tiles(b, mode):
    # d = 512 on the tensor-core encoder: 297 row tiles of 128 (the last one ragged) x 2 column
    # tiles over at most one persistent block per SM, so every block takes several tiles and
    # reuses both accumulators and every ring stage more than once
    d, n = 512, 148 * 128 * 2 + 77
    pair = Pair(tq, d, b, mode, tq.ROT_DENSE, tq.BF16)
    bits = synth.bf16_bits(synth.unit_vectors(n, d, seed=322).astype(np.float32))
    enc = pair.encode(synth.bf16_from_bits(bits))
    gpu, _ = gpu_encode(pair, dev_bf16(bits), n)
    check_codes(pair, gpu, enc)


def test_empty_inputs_are_noops():
    pair = Pair(tq, 128, 3, tq.MSE, tq.ROT_DENSE, tq.F32)
    x = torch.empty((0, 128), dtype=torch.float32, device="cuda")
    tq.quantize_mse(pair.st, x, None, None, n=0, ld=128)
    tq.dequant(pair.st, None, None, torch.empty(0, device="cuda"), None, None, n=0)


def test_misaligned_input_is_rejected():
    pair = Pair(tq, 128, 3, tq.MSE, tq.ROT_DENSE, tq.F32)
    buf = torch.zeros(129 * 4, dtype=torch.float32, device="cuda")
    codes, _, norms, _ = pair.st.empty_planes(4)
    with pytest.raises(tq.TQError) as e:
        tq.quantize_mse(pair.st, buf.data_ptr() + 4, codes, norms, n=4, ld=128, dtype=tq.F32)
    assert e.value.status == 1
    with pytest.raises(tq.TQError):
        tq.quantize_mse(pair.st, buf.data_ptr(), codes, norms, n=4, ld=129, dtype=tq.F32)


def test_state_export_import_and_seeded_state():
    st = tq.State(128, 3, tq.PROD, tq.ROT_DENSE, tq.F32, seed_pi=11, seed_s=12)   # Philox draws
    P = st.copy(tq.FIELD_PI)
    np.testing.assert_allclose(P @ P.T, np.eye(128), atol=1e-5)
    st2 = tq.State.from_bytes(st.export())
    np.testing.assert_array_equal(st2.copy(tq.FIELD_S), st.copy(tq.FIELD_S))
    x = dev_f32(synth.gaussian_vectors(100, 128, seed=3))
    outs = []
    for s in (st, st2):
        codes, qjl, norms, rnorms = s.empty_planes(100)
        tq.quantize_prod(s, x, codes, qjl, norms, rnorms)
        outs.append([host(t) for t in (codes, qjl, norms, rnorms)])
    for a, b in zip(*outs):
        np.testing.assert_array_equal(a, b)


def test_search_topk_small():
    d, n, nq, k = 256, 5000, 9, 10
    pair = Pair(tq, d, 2, tq.PROD, tq.ROT_DENSE, tq.BF16)
    bits, _ = synth.mixture_vectors(n, d, centres=16)
    x = synth.bf16_from_bits(bits)
    enc = pair.encode(x)
    xt = pair.decode(enc)
    qbits, _ = synth.mixture_vectors(nq, d, seed=91, centres=16, centre_seed=synth.SEED_DATA)
    qv = synth.bf16_from_bits(qbits)
    est = OQ.estimate(qv, xt)
    oidx, ovals = OA.topk(est, k)
    planes = planes_to_dev(pair.packed(enc))
    idx = torch.empty((nq, k), dtype=torch.int64, device="cuda")
    vals = torch.empty((nq, k), dtype=torch.float32, device="cuda")
    wsb = tq.search_workspace(pair.st, nq, n, k)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    tq.search_topk(pair.st, dev_bf16(qbits), *planes, k, idx, vals, ws)
    torch.cuda.synchronize()
    gi, gv = host(idx), host(vals)
    for i in range(nq):
        kth = ovals[i, -1]
        for j in range(k):
            if gi[i, j] not in oidx[i]:
                assert est[i, gi[i, j]] >= kth - ABS_SCORE   # a swap at the cut is allowed
        np.testing.assert_allclose(gv[i], est[i, gi[i]], atol=ABS_SCORE)
        assert np.all(np.diff(gv[i]) <= 0)


# --------------------------------------------------------------------------------------
# The tensor-core encoder (d = 128, RHT, bf16 input): tails of every size, strided rows.
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("b,mode", [(2, 1), (3, 1), (4, 1), (1, 0), (2, 0), (3, 0), (4, 0)])
@pytest.mark.parametrize("n,pad", [(1, 0), (127, 8), (129, 0), (5000, 8)])
def test_tc_encoder(b, mode, n, pad):
    d = 128
    pair = Pair(tq, d, b, mode, tq.ROT_RHT, tq.BF16)
    bits = synth.kv_prefill_batch(1, n, d, seed=31 + n)[0]
    buf = np.zeros((n, d + pad), np.uint16)
    buf[:, :d] = bits
    xd = dev_bf16(buf)[:, :d]
    enc = pair.encode(synth.bf16_from_bits(bits))
    gpu, gplanes = gpu_encode(pair, xd, n)
    tq.device_status(0)
    bad = check_codes(pair, gpu, enc)
    xt_o = pair.decode(enc)
    xt_g = gpu_dequant(pair, gplanes, n)
    assert np.max(rel_l2(xt_g[~bad], xt_o[~bad]), initial=0) <= REL_L2


# The two-team encoder (b_mse 1 and 2) with several tiles per CTA: each team refills its two
# TMA stages and reuses its TMEM columns across tiles, and the last tile is ragged.
@pytest.mark.parametrize("b,mode", [(2, 1), (3, 1), (1, 0), (2, 0)])
def test_tc_encoder_many_tiles(b, mode):
    d, n = 128, 148 * 128 * 5 + 77
    pair = Pair(tq, d, b, mode, tq.ROT_RHT, tq.BF16)
    bits = synth.kv_prefill_batch(1, n, d, seed=41)[0]
    enc = pair.encode(synth.bf16_from_bits(bits))
    gpu, gplanes = gpu_encode(pair, dev_bf16(bits), n)
    tq.device_status(0)
    bad = check_codes(pair, gpu, enc)
    xt_o = pair.decode(enc)
    xt_g = gpu_dequant(pair, gplanes, n)
    assert np.max(rel_l2(xt_g[~bad], xt_o[~bad]), initial=0) <= REL_L2


# --------------------------------------------------------------------------------------
# The dense tensor-core encoder (d >= 512, Pi and S bf16, bf16 input): several M tiles and
# a ragged tail, more than one pass of its internal chunking.
# --------------------------------------------------------------------------------------
# Prod encode with the randomized Hadamard rotation at d >= 512 (bf16 in, bf16 S): residual
# pass on the CUDA cores, S r and its signs on the tensor core; more than one internal chunk.
@pytest.mark.parametrize("d,b,n", [(1536, 2, 5000), (512, 3, 70000), (2048, 2, 700)])
def test_rht_encoder_with_tensor_core_signs(d, b, n):
    pair = Pair(tq, d, b, tq.PROD, tq.ROT_RHT, tq.BF16)
    bits, _ = synth.mixture_vectors(n, d, seed=63, centres=16)
    bits[3] = 0                                             # a zero vector
    enc = pair.encode(synth.bf16_from_bits(bits))
    gpu, gplanes = gpu_encode(pair, dev_bf16(bits), n)
    tq.device_status(0)
    bad = check_codes(pair, gpu, enc)
    assert gpu["norms"][3] == 0.0 and gpu["rnorms"][3] == 0.0 and np.all(gpu["qjl"][3] == 255)
    xt_o = pair.decode(enc)
    xt_g = gpu_dequant(pair, gplanes, n)
    ok = ~bad
    ok[3] = False
    assert np.max(rel_l2(xt_g[ok], xt_o[ok])) <= REL_L2


@pytest.mark.parametrize("d,b,mode,n", [(1536, 2, 1, 5000), (512, 3, 1, 70000), (1536, 1, 0, 300)])
def test_dense_gemm_encoder(d, b, mode, n):
    pair = Pair(tq, d, b, mode, tq.ROT_DENSE, tq.BF16)
    bits, _ = synth.mixture_vectors(n, d, seed=57)
    enc = pair.encode(synth.bf16_from_bits(bits))
    gpu, gplanes = gpu_encode(pair, dev_bf16(bits), n)
    tq.device_status(0)
    bad = check_codes(pair, gpu, enc)
    xt_o = pair.decode(enc)
    xt_g = gpu_dequant(pair, gplanes, n)
    assert np.max(rel_l2(xt_g[~bad], xt_o[~bad]), initial=0) <= REL_L2


# --------------------------------------------------------------------------------------
# Tensor-core search (1-bit prod codes, dense Pi and S bf16): several query tiles and key
# tiles with ragged tails; top-k against the oracle's estimates.
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("d,n,nq,k,qf32,rot", [(512, 10000, 200, 10, False, tq.ROT_DENSE),
                                                (1536, 5000, 37, 16, True, tq.ROT_DENSE),
                                                (512, 300, 5, 7, False, tq.ROT_DENSE),
                                                (1536, 5000, 37, 10, False, tq.ROT_RHT),
                                                (1024, 3000, 9, 5, True, tq.ROT_RHT)])
def test_search_topk_tensor_core(d, n, nq, k, qf32, rot):
    pair = Pair(tq, d, 2, tq.PROD, rot, tq.BF16)
    bits, _ = synth.mixture_vectors(n, d, seed=61, centres=32)
    enc = pair.encode(synth.bf16_from_bits(bits))
    xt = pair.decode(enc)
    qbits, _ = synth.mixture_vectors(nq, d, seed=62, centres=32, centre_seed=61)
    qv = synth.bf16_from_bits(qbits)
    est = OQ.estimate(qv, xt)
    oidx, ovals = OA.topk(est, k)
    planes = planes_to_dev(pair.packed(enc))
    qd = dev_f32(qv) if qf32 else dev_bf16(qbits)
    idx = torch.empty((nq, k), dtype=torch.int64, device="cuda")
    vals = torch.empty((nq, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.search_workspace(pair.st, nq, n, k), dtype=torch.uint8, device="cuda")
    tq.search_topk(pair.st, qd, *planes, k, idx, vals, ws)
    torch.cuda.synchronize()
    tq.device_status(0)
    gi, gv = host(idx), host(vals)
    for i in range(nq):
        assert len(set(gi[i].tolist())) == k
        np.testing.assert_allclose(gv[i], est[i, gi[i]], atol=ABS_SCORE)
        assert np.all(np.diff(gv[i]) <= ABS_SCORE)
        kth = ovals[i, -1]
        for j in range(k):
            if gi[i, j] not in oidx[i]:
                assert est[i, gi[i, j]] >= kth - ABS_SCORE
