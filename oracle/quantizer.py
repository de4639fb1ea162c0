"""TurboQuant_mse / TurboQuant_prod encode, decode and inner-product estimate (fp64, CPU).

Test infrastructure. Follows the TurboQuant review (Jump2Paper, arXiv 2504.19874):
  * Problem statement table: Q maps R^d to B = b*d bits, Q^{-1} reconstructs; inputs
    are assumed unit-norm (the norm is stored and restored, as in the AI Trends
    summary, chapter "L2 normalize + RHT matrix").
  * TurboQuant_mse: rotate y = Pi x, give each coordinate the index of its Lloyd-Max
    cell, reconstruct x~ = Pi^T c[idx] (inverse rotation = transpose).
  * Definition 1 (QJL): Q_qjl(x) = sign(S x), S with i.i.d. N(0,1) entries;
    Q_qjl^{-1}(z) = sqrt(pi/2)/d * S^T z.
  * Theorem 2 (prod): (b-1)-bit TurboQuant_mse, then QJL on the residual, with its
    norm kept: x~ = x~_mse + ||r|| Q_qjl^{-1}(Q_qjl(r)).
  * Unbiasedness requirement: E[<y, Q^{-1}(Q(x))>] = <y, x>; the estimate of <q, x>
    is <q, x~>.

Readings of points the pages leave open (each is also listed in the design notes):
  * The residual is formed in the rotated domain, r = y - c[idx], and S acts on it
    (S Pi is again an i.i.d. Gaussian matrix, and ||r|| is unchanged by Pi).
  * Decisions are taken in fp32 on both sides: a code is #{k : t_k <= fp32(y_j)}
    with fp32-stored boundaries t_k (a value on a boundary goes to the upper cell);
    a QJL bit is [fp32((S r)_j) >= 0] (zero maps to +1).
  * The stored state defines the transform: Pi, S and the centroids are used with the
    values the device holds (fp32 or bf16), converted exactly to fp64.
  * A zero vector stores norm 0, rotated coordinates 0, residual 0 and norm(r) = 0.
  * b = 1 in prod mode is 0-bit MSE: x~_mse = 0 and r = y.
  * Packing: each vector's codes form one LSB-first bit stream, code j in bits
    [j*b, j*b + b); QJL bit j is bit j of its own plane; planes are [n][bytes].
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import codebook as _cb
from .rotation import round_f32

__all__ = [
    "Codebook",
    "make_codebook",
    "quantize_coords",
    "pack_bits",
    "unpack_bits",
    "encode_mse",
    "decode_mse",
    "encode_prod",
    "decode_prod",
    "estimate",
    "QJL_SCALE",
]


def QJL_SCALE(d: int) -> float:
    """sqrt(pi/2)/d, the scale of Q_qjl^{-1} (Definition 1)."""
    return float(np.sqrt(np.pi / 2.0) / d)


@dataclass(frozen=True)
class Codebook:
    d: int
    b: int
    centroids: np.ndarray      # fp64 Lloyd-Max centroids, ascending (2^b)
    bounds: np.ndarray         # fp64 midpoints (2^b - 1)
    c32: np.ndarray            # stored centroids (fp32 values as fp64)
    t32: np.ndarray            # stored boundaries (fp32 values as fp64)
    dmse: float


def make_codebook(d: int, b: int) -> Codebook:
    c, t, D, _ = _cb.lloyd_max(d, b)
    return Codebook(d, b, c, t, round_f32(c), round_f32(t), D)


def quantize_coords(y: np.ndarray, cb: Codebook) -> np.ndarray:
    """idx_j = #{k : t_k <= y_j}, compared in fp32 (upper cell on a tie)."""
    y32 = np.asarray(y, np.float64).astype(np.float32)
    t32 = cb.t32.astype(np.float32)
    return np.searchsorted(t32, y32, side="right").astype(np.int64)


def pack_bits(codes: np.ndarray, b: int) -> np.ndarray:
    """Pack [n, d] codes of b bits into [n, ceil(b*d/8)] bytes, LSB-first per vector."""
    codes = np.asarray(codes, np.int64)
    n, d = codes.shape
    if b == 0:
        return np.zeros((n, 0), np.uint8)
    bits = ((codes[:, :, None] >> np.arange(b)[None, None, :]) & 1).reshape(n, d * b)
    return np.packbits(bits.astype(np.uint8), axis=1, bitorder="little")


def unpack_bits(packed: np.ndarray, b: int, d: int) -> np.ndarray:
    """Inverse of pack_bits."""
    packed = np.asarray(packed, np.uint8)
    n = packed.shape[0]
    if b == 0:
        return np.zeros((n, d), np.int64)
    bits = np.unpackbits(packed, axis=1, bitorder="little")[:, : d * b].reshape(n, d, b)
    return np.sum(bits.astype(np.int64) << np.arange(b)[None, None, :], axis=2)


def _rotate_unit(x: np.ndarray, Pi: np.ndarray):
    x = np.asarray(x, np.float64)
    nu = np.linalg.norm(x, axis=1)
    safe = np.where(nu > 0, nu, 1.0)
    y = (x / safe[:, None]) @ np.asarray(Pi, np.float64).T
    y[nu == 0] = 0.0
    return nu, y


def encode_mse(x: np.ndarray, Pi: np.ndarray, cb: Codebook):
    """TurboQuant_mse encode. Returns (codes[n,d] int, norms[n], y[n,d] rotated unit vectors)."""
    nu, y = _rotate_unit(x, Pi)
    return quantize_coords(y, cb), nu, y


def decode_mse(codes: np.ndarray, norms: np.ndarray, Pi: np.ndarray, cb: Codebook) -> np.ndarray:
    """x~ = ||x|| Pi^T c[idx]."""
    yt = cb.c32[np.asarray(codes, np.int64)]
    return np.asarray(norms, np.float64)[:, None] * (yt @ np.asarray(Pi, np.float64))


def encode_prod(x: np.ndarray, Pi: np.ndarray, S: np.ndarray, cb_m1: Codebook | None):
    """TurboQuant_prod encode with a (b-1)-bit MSE codebook `cb_m1` (None when b = 1).

    Returns (codes[n,d], qjl_bits[n,d] in {0,1}, norms[n], rnorms[n], y, s = S r).
    """
    nu, y = _rotate_unit(x, Pi)
    n, d = y.shape
    if cb_m1 is None:
        codes = np.zeros((n, d), np.int64)
        r = y.copy()
    else:
        codes = quantize_coords(y, cb_m1)
        r = y - cb_m1.c32[codes]
    r[nu == 0] = 0.0
    rho = np.linalg.norm(r, axis=1)
    s = r @ np.asarray(S, np.float64).T
    z = (s.astype(np.float32) >= 0).astype(np.int64)
    return codes, z, nu, rho, y, s


def decode_prod(codes, qjl_bits, norms, rnorms, Pi, S, cb_m1: Codebook | None) -> np.ndarray:
    """x~ = ||x|| Pi^T (c[idx] + ||r|| sqrt(pi/2)/d S^T (2z - 1))."""
    S = np.asarray(S, np.float64)
    d = S.shape[0]
    codes = np.asarray(codes, np.int64)
    yt = np.zeros(codes.shape) if cb_m1 is None else cb_m1.c32[codes]
    sgn = 2.0 * np.asarray(qjl_bits, np.float64) - 1.0
    yt = yt + (np.asarray(rnorms, np.float64) * QJL_SCALE(d))[:, None] * (sgn @ S)
    return np.asarray(norms, np.float64)[:, None] * (yt @ np.asarray(Pi, np.float64))


def estimate(q: np.ndarray, x_tilde: np.ndarray) -> np.ndarray:
    """Inner-product estimates <q_i, x~_k> for queries [nq, d] and reconstructions [n, d]."""
    return np.asarray(q, np.float64) @ np.asarray(x_tilde, np.float64).T
