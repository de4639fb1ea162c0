"""Random rotations Pi (fp64, CPU). Test infrastructure.

* Dense Haar rotation: the TurboQuant review (Jump2Paper) states that Pi maps any
  unit vector to a uniform point on the sphere and that the paper uses a general QR
  rotation (discussion of why a rotation and not a projection). Pi is the Q factor of
  a d x d N(0,1) matrix, with the signs of R's diagonal moved into Q so that the
  factorisation is unique (Q diag(sign(diag R))).
* Randomized Hadamard transform: the AI Trends summary of the TurboQuant video
  (chapter "L2 normalize + RHT matrix") rotates by an RHT, whose inverse is its
  transpose; the Jump2Paper review's future-work paragraph names Hadamard plus random
  signs. Reading used: Pi = H_d diag(eps) / sqrt(d), H_d the Sylvester Hadamard matrix
  (signs applied first, then H, then 1/sqrt(d)).
"""
from __future__ import annotations

import numpy as np
import scipy.linalg

__all__ = ["haar_from_gaussian", "rht_matrix", "round_f32", "round_bf16"]


def haar_from_gaussian(g: np.ndarray) -> np.ndarray:
    """Haar-random orthogonal matrix from a square N(0,1) matrix via QR with the sign fix."""
    q, r = np.linalg.qr(np.asarray(g, dtype=np.float64))
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    return q * s[None, :]


def rht_matrix(signs: np.ndarray) -> np.ndarray:
    """Pi = H_d diag(eps) / sqrt(d) with H_d Sylvester's Hadamard matrix (d a power of two)."""
    eps = np.asarray(signs, dtype=np.float64)
    d = eps.shape[0]
    h = scipy.linalg.hadamard(d).astype(np.float64)
    return h * eps[None, :] / np.sqrt(d)


def round_f32(a: np.ndarray) -> np.ndarray:
    """Values of `a` as stored in fp32 (the stored state defines the transform)."""
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Values of `a` rounded to bf16 (nearest, ties to even), via fp32."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)
