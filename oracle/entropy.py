"""Prefix coding of the codebook indices (CPU). Test infrastructure.

TurboQuant review (Jump2Paper), limitations paragraph: an optimal prefix code on the b = 4
codebook indices brings the average width to about 3.8 bits (about 5 % less); the paper
itself leaves the step out.

Readings (also listed in the design notes):
  * The code is the Huffman code of the index law of one coordinate under Lemma 1:
    p_i = F(t_i) - F(t_{i-1}) over the cells of the Lloyd-Max boundaries (t_{-1} = -1,
    t_{L-1} = 1). It is fixed per (d, b), so coding stays data-independent (online).
    The law is even, so p_{L-1-i} is set equal to p_i (computed for i < L/2).
  * Huffman's algorithm repeatedly merges the two least probable nodes; ties go to the
    node with the lower id (leaves 0..L-1, merged nodes numbered L, L+1, ... as created).
  * Canonical codewords: symbols sorted by (length, symbol) get consecutive integers, the
    codeword growing by one and shifting left when the length grows.
  * Stream: a vector's d codes in coordinate order, each codeword written first bit (its
    most significant) first; vectors back to back; bit j of the stream is bit j % 8 of
    byte j // 8 (LSB-first, as the fixed-width planes). offsets[k] is vector k's first bit,
    offsets[n] the total.
"""
from __future__ import annotations

import heapq

import numpy as np

from . import codebook as _cb

__all__ = ["index_probabilities", "huffman_lengths", "canonical_codewords", "encode", "decode"]


def index_probabilities(d: int, bounds) -> np.ndarray:
    """p_i of the 2^b cells of the boundaries under f_X, made exactly symmetric."""
    t = np.asarray(bounds, np.float64)
    L = len(t) + 1
    edges = np.concatenate([[-1.0], t, [1.0]])
    p = np.empty(L)
    for i in range(L // 2):
        p[i] = float(_cb.cdf(edges[i + 1], d) - _cb.cdf(edges[i], d))
        p[L - 1 - i] = p[i]
    return p


def huffman_lengths(p) -> np.ndarray:
    """Codeword lengths of Huffman's code for probabilities p (ties to the lower node id)."""
    p = [float(v) for v in p]
    L = len(p)
    if L == 1:
        return np.array([1])
    heap = [(p[i], i) for i in range(L)]
    heapq.heapify(heap)
    parent = {}
    nxt = L
    while len(heap) > 1:
        pa, a = heapq.heappop(heap)
        pb, b = heapq.heappop(heap)
        parent[a] = parent[b] = nxt
        heapq.heappush(heap, (pa + pb, nxt))
        nxt += 1
    root = heap[0][1]
    lengths = np.zeros(L, np.int64)
    for i in range(L):
        n, depth = i, 0
        while n != root:
            n = parent[n]
            depth += 1
        lengths[i] = depth
    return lengths


def canonical_codewords(lengths) -> np.ndarray:
    """Canonical codewords (integers, `lengths[i]` bits each) for the given lengths."""
    lengths = np.asarray(lengths, np.int64)
    order = sorted(range(len(lengths)), key=lambda i: (lengths[i], i))
    words = np.zeros(len(lengths), np.int64)
    code, prev = 0, int(lengths[order[0]])
    for k, i in enumerate(order):
        if k > 0:
            code = (code + 1) << (int(lengths[i]) - prev)
        prev = int(lengths[i])
        words[i] = code
    return words


def encode(codes: np.ndarray, lengths, words):
    """Stream bytes and offsets [n + 1] for codes [n, d] (see the module notes)."""
    codes = np.asarray(codes, np.int64)
    n, d = codes.shape
    lengths = np.asarray(lengths, np.int64)
    bits = []
    offsets = np.zeros(n + 1, np.int64)
    for k in range(n):
        for c in codes[k]:
            ln, w = int(lengths[c]), int(words[c])
            bits.extend((w >> (ln - 1 - j)) & 1 for j in range(ln))
        offsets[k + 1] = len(bits)
    stream = np.packbits(np.array(bits, np.uint8), bitorder="little") if bits else np.zeros(0, np.uint8)
    return stream, offsets


def decode(stream: np.ndarray, offsets, n: int, d: int, lengths, words) -> np.ndarray:
    """Inverse of encode: codes [n, d]."""
    bits = np.unpackbits(np.asarray(stream, np.uint8), bitorder="little")
    table = {(int(lengths[i]), int(words[i])): i for i in range(len(lengths))}
    out = np.zeros((n, d), np.int64)
    for k in range(n):
        pos = int(offsets[k])
        for j in range(d):
            w, ln = 0, 0
            while (ln, w) not in table:
                w = (w << 1) | int(bits[pos])
                ln += 1
                pos += 1
            out[k, j] = table[(ln, w)]
    return out
