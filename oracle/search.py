"""Exhaustive top-k inner-product search over quantized vectors (oracle).

R, *Validation* / *Results*: the same quantizer serves nearest-neighbour search by
inner product (GloVe d=200, OpenAI3 d=1536/3072), with near-zero indexing time.
Reading: order by estimated score descending, ties by ascending id.
"""
from __future__ import annotations

import numpy as np

__all__ = ["topk"]


def topk(scores: np.ndarray, k: int):
    """Return (ids [nq, k] int64, values [nq, k]) sorted by (-score, id)."""
    scores = np.asarray(scores, dtype=np.float64)
    nq, n = scores.shape
    ids = np.zeros((nq, k), dtype=np.int64)
    vals = np.zeros((nq, k))
    idx = np.arange(n)
    for i in range(nq):
        order = np.lexsort((idx, -scores[i]))[:k]
        ids[i] = order
        vals[i] = scores[i, order]
    return ids, vals
