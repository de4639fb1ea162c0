"""Helpers for the GPU-vs-oracle parity tests.

Builds a library state and the matching oracle quantities from the same seeded draws,
and implements the comparison rules:
  * packed codes bit-exact, except coordinates within 1e-5 of a decision boundary
    (rotated value vs boundary; QJL: |(S r)_j| vs 0); such mismatches must stay below
    1e-4 of the coordinates;
  * reconstructions within 1e-3 relative L2; scores and attention outputs within 2e-3
    absolute.
Unpacking of the library's bytes is done here with numpy (no oracle code touches the
library's outputs).
"""
from __future__ import annotations

import numpy as np

import synth
from oracle import quantizer as OQ
from oracle import rotation as OR

BAND = 1e-5
MISMATCH_RATE = 1e-4
REL_L2 = 1e-3
ABS_SCORE = 2e-3


class Pair:
    """A libtq state and its oracle twin (same draws, same stored precision)."""

    def __init__(self, tq, d, b, mode, rot, mat_dtype, seed_pi=synth.SEED_PI, seed_s=synth.SEED_S, device=0):
        self.d, self.b, self.mode, self.rot = d, b, mode, rot
        G = synth.gaussian_matrix(d, seed_pi) if rot == tq.ROT_DENSE else None
        eps = synth.rht_signs(d, seed_pi) if rot == tq.ROT_RHT else None
        S = synth.gaussian_matrix(d, seed_s) if mode == tq.PROD else None
        self.st = tq.State(d, b, mode, rot, mat_dtype, device=device, gauss_pi=G, signs=eps, s=S)
        rnd = OR.round_f32 if mat_dtype == tq.F32 else OR.round_bf16
        self.Pi = rnd(OR.haar_from_gaussian(G)) if G is not None else OR.rht_matrix(eps)
        self.S = rnd(S) if S is not None else None
        self.b_mse = b if mode == tq.MSE else b - 1
        self.cb = OQ.make_codebook(d, self.b_mse) if self.b_mse > 0 else None

    # oracle side -------------------------------------------------------------------
    def encode(self, x):
        if self.mode == 0:
            codes, nu, y = OQ.encode_mse(x, self.Pi, self.cb)
            return dict(codes=codes, nu=nu, y=y)
        codes, z, nu, rho, y, s = OQ.encode_prod(x, self.Pi, self.S, self.cb)
        return dict(codes=codes, z=z, nu=nu, rho=rho, y=y, s=s)

    def decode(self, enc):
        if self.mode == 0:
            return OQ.decode_mse(enc["codes"], enc["nu"], self.Pi, self.cb)
        return OQ.decode_prod(enc["codes"], enc["z"], enc["nu"], enc["rho"], self.Pi, self.S, self.cb)

    def packed(self, enc):
        """Oracle planes as numpy arrays in the library layout."""
        out = dict(codes=OQ.pack_bits(enc["codes"], self.b_mse) if self.b_mse > 0 else
                   np.zeros((len(enc["nu"]), 0), np.uint8),
                   norms=enc["nu"].astype(np.float32))
        if self.mode == 1:
            out["qjl"] = OQ.pack_bits(enc["z"], 1)
            out["rnorms"] = enc["rho"].astype(np.float32)
        return out


def unpack(packed: np.ndarray, b: int, d: int) -> np.ndarray:
    """LSB-first unpack of library planes [n, bytes] into codes [n, d]."""
    n = packed.shape[0]
    if b == 0:
        return np.zeros((n, d), np.int64)
    bits = np.unpackbits(np.ascontiguousarray(packed, np.uint8), axis=1, bitorder="little")[:, : b * d]
    bits = bits.reshape(n, d, b).astype(np.int64)
    return np.sum(bits << np.arange(b)[None, None, :], axis=2)


def band_distance(y: np.ndarray, t32: np.ndarray) -> np.ndarray:
    """Distance of each rotated coordinate to its nearest decision boundary."""
    if len(t32) == 0:
        return np.full(y.shape, np.inf)
    idx = np.searchsorted(t32, y)
    lo = np.abs(y - t32[np.clip(idx - 1, 0, len(t32) - 1)])
    hi = np.abs(y - t32[np.clip(idx, 0, len(t32) - 1)])
    return np.minimum(lo, hi)


def check_codes(pair: Pair, gpu: dict, enc: dict, report: dict | None = None):
    """Compare library planes with the oracle encode under the band rule. Returns mismatch info."""
    d, n = pair.d, len(enc["nu"])
    info = {}
    bad_vec = np.zeros(n, bool)
    if pair.b_mse > 0:
        g = unpack(gpu["codes"], pair.b_mse, d)
        mism = g != enc["codes"]
        dist = band_distance(enc["y"], pair.cb.t32)
        out_band = mism & (dist >= BAND)
        assert not out_band.any(), f"{out_band.sum()} code mismatches outside the {BAND} band"
        info["code_mismatch"] = int(mism.sum())
        assert mism.sum() <= MISMATCH_RATE * mism.size, info
        bad_vec |= mism.any(axis=1)
    if pair.mode == 1:
        gz = unpack(gpu["qjl"], 1, d)
        mism = (gz != enc["z"]) & ~bad_vec[:, None]
        out_band = mism & (np.abs(enc["s"]) >= BAND)
        assert not out_band.any(), f"{out_band.sum()} QJL mismatches outside the band"
        info["qjl_mismatch"] = int(mism.sum())
        assert mism.sum() <= MISMATCH_RATE * mism.size, info
        ok = ~bad_vec
        np.testing.assert_allclose(gpu["rnorms"][ok], enc["rho"][ok], rtol=1e-4, atol=1e-6)
        # an in-band sign flip is allowed, but that vector's estimates then differ: flag it
        bad_vec |= mism.any(axis=1)
    np.testing.assert_allclose(gpu["norms"], enc["nu"], rtol=1e-5, atol=1e-30)
    info["vectors_with_code_mismatch"] = int(bad_vec.sum())
    if report is not None:
        report.update(info)
    return bad_vec


def rel_l2(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    num = np.linalg.norm(a - b, axis=-1)
    den = np.maximum(np.linalg.norm(b, axis=-1), 1e-30)
    return num / den
