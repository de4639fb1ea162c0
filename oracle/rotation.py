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

__all__ = ["haar_from_gaussian", "paley_hadamard12", "hadamard", "rht_matrix", "round_f32", "round_bf16"]


def haar_from_gaussian(g: np.ndarray) -> np.ndarray:
    """Haar-random orthogonal matrix from a square N(0,1) matrix via QR with the sign fix."""
    q, r = np.linalg.qr(np.asarray(g, dtype=np.float64))
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    return q * s[None, :]


def paley_hadamard12() -> np.ndarray:
    """Paley's Hadamard matrix of order 12 (from GF(11))."""
    q = 11
    residues = {(x * x) % q for x in range(1, q)}
    chi = np.array([0.0] + [1.0 if a in residues else -1.0 for a in range(1, q)])
    Q = np.array([[chi[(j - i) % q] for j in range(q)] for i in range(q)])
    core = np.zeros((q + 1, q + 1))
    core[0, 1:] = 1.0
    core[1:, 0] = -1.0
    core[1:, 1:] = Q
    return np.eye(q + 1) + core


def hadamard(d: int) -> np.ndarray:
    """Hadamard matrix of order d: Sylvester's for d = 2^k, H_12 (x) Sylvester's for 12 * 2^k."""
    if d & (d - 1) == 0:
        return scipy.linalg.hadamard(d).astype(np.float64)
    if d % 12 == 0 and (d // 12) & (d // 12 - 1) == 0:
        return np.kron(paley_hadamard12(), scipy.linalg.hadamard(d // 12).astype(np.float64))
    raise ValueError(f"no Hadamard matrix built for d = {d}")


def rht_matrix(signs: np.ndarray) -> np.ndarray:
    """Pi = H_d diag(eps) / sqrt(d) (see `hadamard` for the orders covered)."""
    eps = np.asarray(signs, dtype=np.float64)
    d = eps.shape[0]
    return hadamard(d) * eps[None, :] / np.sqrt(d)


def round_f32(a: np.ndarray) -> np.ndarray:
    """Values of `a` as stored in fp32 (the stored state defines the transform)."""
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Values of `a` rounded to bf16 (nearest, ties to even), via fp32."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)
