"""Decode attention over a compressed cache, and top-k search (fp64, CPU). Test infrastructure.

* Attention: softmax(K~ q * scale) V~ for one query per head, with K~ and V~ the
  reconstructions of the compressed keys and values. The standard form is the one the
  PolarQuant review (mdooai, attention with quantized KV) writes; the TurboQuant review
  (Jump2Paper, KV-cache application) states that the inner products of KV vectors
  drive the attention scores. Reading used: scale = 1/sqrt(d), softmax with the
  maximum subtracted.
* Search: top-k database vectors by the estimated inner product <q, x~> (Jump2Paper,
  nearest-neighbour search application). Ties go to the lower index.
"""
from __future__ import annotations

import numpy as np

__all__ = ["softmax", "decode_attention", "topk"]


def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    s = np.asarray(s, np.float64)
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def decode_attention(q: np.ndarray, k_tilde: np.ndarray, v_tilde: np.ndarray,
                     scale: float) -> np.ndarray:
    """One decode step: q [H, d], k_tilde/v_tilde [H, T, d] -> out [H, d]."""
    q = np.asarray(q, np.float64)
    s = np.einsum("hd,htd->ht", q, np.asarray(k_tilde, np.float64)) * scale
    p = softmax(s, axis=1)
    return np.einsum("ht,htd->hd", p, np.asarray(v_tilde, np.float64))


def topk(est: np.ndarray, k: int):
    """Per row of est [nq, n]: the k largest values, ties to the lower index.

    Returns (idx [nq, k] int64, vals [nq, k])."""
    est = np.asarray(est, np.float64)
    n = est.shape[1]
    order = np.lexsort((np.broadcast_to(np.arange(n), est.shape), -est), axis=1)[:, :k]
    return order.astype(np.int64), np.take_along_axis(est, order, axis=1)
