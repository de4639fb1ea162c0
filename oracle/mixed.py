"""Outlier-channel split with two bit widths (fp64, CPU). Test infrastructure.

TurboQuant review (Jump2Paper, arXiv 2504.19874): the experiment-settings table ("KV bit
settings": 2.5 and 3.5 bits with outlier and non-outlier channels separated; "outlier
handling": 32 of 128 channels at 3 bits, 96 at 2 bits) and the closing note on outlier
channels (they take large values, so they get more bits).

Readings of what the pages leave open (each is also listed in the design notes):
  * Each channel group is its own TurboQuant quantizer of the group's dimension: its own
    rotation, its own Lloyd-Max codebook (Lemma 1 at that dimension), its own QJL matrix
    (prod) and its own stored norms.
  * The reconstruction puts each group's reconstruction back into its channels, so the
    inner-product estimate <q, x~> is the sum of the two groups' estimates.
  * The outlier channels are chosen by the caller (the pages do not say how); the tests
    and the bench take the m channels of largest mean square over the batch.
  * Effective width: the pages print (32*3 + 96*2)/128 = 2.5, but that expression equals
    2.25. The split is kept as stated and its width is reported from the formula,
    sum_g m_g b_g / d; a 2.5-bit split is e.g. 32 channels at 4 bits and 96 at 2.
"""
from __future__ import annotations

import numpy as np

__all__ = ["rest_channels", "split", "merge", "effective_bits", "outlier_channels"]


def rest_channels(channels, d: int) -> np.ndarray:
    """The channels not in `channels`, ascending."""
    mask = np.ones(d, bool)
    mask[np.asarray(channels, np.int64)] = False
    return np.nonzero(mask)[0]


def split(x: np.ndarray, channels) -> tuple[np.ndarray, np.ndarray]:
    """(x[:, channels], x[:, rest]) for rows x [n, d]; `channels` in the caller's order."""
    x = np.asarray(x)
    ch = np.asarray(channels, np.int64)
    return x[:, ch], x[:, rest_channels(ch, x.shape[1])]


def merge(x_out: np.ndarray, x_rest: np.ndarray, channels, d: int) -> np.ndarray:
    """Inverse of split: row j of the result holds x_out in `channels`, x_rest elsewhere."""
    ch = np.asarray(channels, np.int64)
    n = x_out.shape[0]
    out = np.zeros((n, d), np.result_type(x_out, x_rest))
    out[:, ch] = x_out
    out[:, rest_channels(ch, d)] = x_rest
    return out


def effective_bits(groups) -> float:
    """Bits per channel of a split, sum_g m_g b_g / sum_g m_g (norms not counted)."""
    groups = [(int(m), float(b)) for m, b in groups]
    return sum(m * b for m, b in groups) / sum(m for m, _ in groups)


def outlier_channels(x: np.ndarray, m: int) -> np.ndarray:
    """The m channels of largest mean square over the rows of x, ascending."""
    ms = np.mean(np.square(np.asarray(x, np.float64)), axis=0)
    top = np.argsort(-ms, kind="stable")[:m]
    return np.sort(top)
