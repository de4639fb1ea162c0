"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle.

This module draws random numbers and shapes them into workloads. It holds none of
the quantizer's arithmetic: no rotation is formed here (a dense rotation is built by
each side from the Gaussian matrix drawn here), no codebook, no quantization.

Every generator is a pure function of its seed (numpy PCG64), so the oracle and the
library see bit-identical inputs. bf16 inputs are produced by rounding fp32 to the
nearest bf16 (ties to even) and are returned both as the 16-bit patterns that are
uploaded to the device and as exact float64 values for the oracle.

Workloads follow the shapes of the TurboQuant review (Jump2Paper, experiment setup
table: d=128 KV heads of Llama-3.1-8B-class models; DBpedia d=1536 search) with
synthetic data standing in for the models and datasets.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rng",
    "bf16_round",
    "bf16_bits",
    "bf16_from_bits",
    "gaussian_matrix",
    "rht_signs",
    "unit_vectors",
    "gaussian_vectors",
    "kv_prefill_batch",
    "decode_queries",
    "mixture_vectors",
    "SEED_PI",
    "SEED_S",
    "SEED_DATA",
]

# Seed plan: 0 draws the rotation (Gaussian matrix or RHT signs), 1 draws the QJL
# matrix S, 2 and above draw data.
SEED_PI = 0
SEED_S = 1
SEED_DATA = 2


def rng(seed: int, stream: int = 0) -> np.random.Generator:
    """PCG64 generator for (seed, stream); streams make per-head data reproducible."""
    return np.random.Generator(np.random.PCG64([int(seed), int(stream)]))


def bf16_bits(a) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return uint16 bits."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_from_bits(bits) -> np.ndarray:
    """Exact float64 values of bf16 bit patterns."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16)).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_round(a) -> np.ndarray:
    """fp64 values of the bf16 numbers nearest to a (through fp32)."""
    return bf16_from_bits(bf16_bits(a))


def gaussian_matrix(d: int, seed: int = SEED_PI, *, bf16: bool = False) -> np.ndarray:
    """d x d matrix of i.i.d. N(0,1) draws (float64; rounded to bf16 values if asked)."""
    g = rng(seed, 0).standard_normal((d, d))
    return bf16_round(g) if bf16 else g


def rht_signs(d: int, seed: int = SEED_PI) -> np.ndarray:
    """d random signs in {-1,+1} (int8), the diagonal of the randomized Hadamard transform."""
    bits = rng(seed, 1).integers(0, 2, size=d)
    return (2 * bits - 1).astype(np.int8)


def gaussian_vectors(n: int, d: int, seed: int, stream: int = 0) -> np.ndarray:
    """n x d i.i.d. N(0,1) float64."""
    return rng(seed, stream).standard_normal((n, d))


def unit_vectors(n: int, d: int, seed: int, stream: int = 0, dtype=np.float32) -> np.ndarray:
    """n unit vectors uniform on the sphere: N(0,1) rows divided by their L2 norm.

    The division happens in float64 and the result is rounded to `dtype` once, so
    the stored rows are unit vectors up to that dtype's rounding.
    """
    g = gaussian_vectors(n, d, seed, stream)
    g /= np.linalg.norm(g, axis=1, keepdims=True)
    return g.astype(dtype)


def kv_prefill_batch(heads: int, tokens: int, d: int, seed: int = SEED_DATA,
                     n_outliers: int = 4, outlier_scale: float = 20.0,
                     lognorm_sigma: float = 0.5, head_range=None) -> np.ndarray:
    """KV-cache-shaped keys [heads, tokens, d] as bf16 bit patterns (uint16).

    Entries N(0,1); per head, `n_outliers` channels (a seeded pick per head) are
    scaled by `outlier_scale`; each token's vector is then rescaled to a norm drawn
    from log-normal(0, lognorm_sigma). Head h is drawn from stream h, so any subset
    of heads can be regenerated alone (`head_range=(h0, h1)`).
    """
    h0, h1 = (0, heads) if head_range is None else head_range
    out = np.empty((h1 - h0, tokens, d), dtype=np.uint16)
    for h in range(h0, h1):
        g = rng(seed, 1000 + h)
        x = g.standard_normal((tokens, d), dtype=np.float32)
        ch = g.choice(d, size=n_outliers, replace=False)
        x[:, ch] *= np.float32(outlier_scale)
        nrm = np.linalg.norm(x, axis=1, keepdims=True)
        target = np.exp(lognorm_sigma * g.standard_normal((tokens, 1), dtype=np.float32))
        x *= target / nrm
        out[h - h0] = bf16_bits(x)
    return out


def decode_queries(heads: int, d: int, seed: int = SEED_DATA + 1) -> np.ndarray:
    """One N(0, I) query per head, as bf16 bit patterns [heads, d]."""
    return bf16_bits(rng(seed, 7).standard_normal((heads, d)))


def mixture_vectors(n: int, d: int, seed: int = SEED_DATA, centres: int = 256,
                    sigma: float = 0.3, row_range=None, centre_seed: int | None = None):
    """Gaussian-mixture embeddings, L2-normalised, as bf16 bit patterns [n, d].

    Centres are uniform on the sphere; a point is centre + sigma * N(0, I)/sqrt(d)
    (so the noise norm is about sigma, comparable to the unit centres), then
    normalised. Rows are drawn in blocks of 65536 from per-block streams, so a
    slice `row_range=(r0, r1)` regenerates exactly those rows.
    Returns (bits, labels).
    """
    cs = seed if centre_seed is None else centre_seed
    mu = rng(cs, 99).standard_normal((centres, d))
    mu /= np.linalg.norm(mu, axis=1, keepdims=True)
    r0, r1 = (0, n) if row_range is None else row_range
    blk = 65536
    bits = np.empty((r1 - r0, d), dtype=np.uint16)
    labels = np.empty(r1 - r0, dtype=np.int64)
    for b0 in range((r0 // blk) * blk, r1, blk):
        b1 = min(b0 + blk, n)
        g = rng(seed, 5000 + b0 // blk)
        lab = g.integers(0, centres, size=b1 - b0)
        x = mu[lab] + sigma * g.standard_normal((b1 - b0, d)) / np.sqrt(d)
        x /= np.linalg.norm(x, axis=1, keepdims=True)
        lo, hi = max(b0, r0), min(b1, r1)
        bits[lo - r0:hi - r0] = bf16_bits(x[lo - b0:hi - b0])
        labels[lo - r0:hi - r0] = lab[lo - b0:hi - b0]
    return bits, labels
