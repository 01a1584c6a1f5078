"""Batched projection over the union of the sequences' kept channels (oracle
side, fp64; test infrastructure only).

What the pages fix (ByteCross README, "Usage: The byte account",
crossover_batch): a batch of sequences reads the projection weights that the
union of its sequences' selections covers, once per step, and the batch
crossover takes the fraction of the weights that union covers (92% at four
sequences in the README's example).  The pages give only this byte model, not
the batched step.

Reading taken (the plainest one the byte model supports): every sequence
keeps its own channels exactly as in the batch-1 step -- its own top-k of
|x_b| -- so its projection is unchanged,

    y_b[j] = sum over c in S_b of x_b[c] * W[c, j],

and the batch's weight traffic is the rows of U = S_1 u ... u S_B, each read
once.  A sequence never uses a channel that only another sequence kept.
"""
from __future__ import annotations

import numpy as np

from .decoder import bf16_to_f64


def union_channels(sels, d_in: int) -> np.ndarray:
    """U = S_1 u ... u S_B, ascending."""
    mark = np.zeros(d_in, dtype=bool)
    for s in sels:
        mark[np.asarray(s, dtype=np.int64)] = True
    return np.flatnonzero(mark)


def union_keep(sels, d_in: int) -> float:
    """|U| / d_in: the fraction of a projection's rows the batch reads."""
    return union_channels(sels, d_in).shape[0] / d_in


def gemv_batch(w_bits: np.ndarray, X: np.ndarray, sels) -> np.ndarray:
    """y[b] = sum over c in S_b of X[b, c] * W[c, :] for an input-channel-major
    bf16 matrix W [d_in][d_out]; one row of y per sequence, fp64."""
    d_in, d_out = w_bits.shape
    X = np.asarray(X, dtype=np.float64)
    y = np.zeros((X.shape[0], d_out))
    for b, s in enumerate(sels):
        s = np.asarray(s, dtype=np.int64)
        y[b] = X[b, s] @ bf16_to_f64(w_bits[s])
    return y


def union_bytes(sels, d_in: int, d_out: int, elem: int = 2) -> int:
    """Weight bytes a batched projection reads: |U| rows of d_out elements."""
    return union_channels(sels, d_in).shape[0] * d_out * elem
