"""Outlier-channel split: independent TurboQuant instances on channel groups (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

R, *Method* (KV-cache experiments): the channels of a key or value vector are split
into an outlier group and a non-outlier group, and each group is quantized by its own
TurboQuant instance; the 2.5-bit setting is 32 outlier channels at 3 bits plus the
other 96 channels at 2 bits.  LK, Show HN post: the outlier channels are detected
online, with no calibration data; LK, "What's next": precomputed per-model channel
lists.

Readings taken where the pages are silent (all listed in the design notes):

* A group is a list of channel indices.  The groups are disjoint and together cover
  channels 0..d-1.  Group g sees the sub-vector x[:, ch_g] (channels in the listed
  order) and runs TurboQuant-mse (or -prod) of dimension d_g = len(ch_g) with its own
  rotation (d_g x d_g), its own codebook (the Beta marginal for d_g) and its own norm
  ||x[:, ch_g]||.
* Online detection: after a set of vectors has been seen, the k channels with the
  largest mean square over them form the outlier group (a tie goes to the lower
  channel index); both groups list their channels in ascending order.
* Inner products add over the groups: est(q, x) = sum_g est_g(q[ch_g], x_g), the
  reconstruction scatters each group's x_hat_g back to its channels, and attention uses
  these estimates and reconstructions exactly as the single-instance path does.
* Bit width.  The code bits alone average sum_g d_g b_g / d, which is 2.25 for the
  pages' setting, while the pages call that setting 2.5-bit.  The two agree when every
  group also stores one 16-bit norm per vector, (288 + 2 x 16) / 128 = 2.5, so
  :func:`effective_bits` takes the norm width as a parameter (0 = codes only).
"""
from __future__ import annotations

import numpy as np

from . import quantizer as Q

__all__ = ["outlier_channels", "split_groups", "effective_bits", "quantize_split",
           "dequantize_split", "estimate_split"]


def outlier_channels(x_seen, k: int) -> np.ndarray:
    """The k channels with the largest mean square over the rows of x_seen, ascending.

    Ties go to the lower channel index (a stable sort on the negated mean square).
    """
    x = np.asarray(x_seen, dtype=np.float64)
    d = x.shape[1]
    if not 0 <= k <= d:
        raise ValueError("k must lie in 0..d")
    ms = np.mean(x * x, axis=0)
    order = np.argsort(-ms, kind="stable")
    return np.sort(order[:k])


def split_groups(d: int, outliers) -> list[np.ndarray]:
    """[outlier channels, the other channels], each ascending."""
    out = np.unique(np.asarray(outliers, dtype=np.int64))
    if out.size and (out[0] < 0 or out[-1] >= d):
        raise ValueError("channel index out of range")
    rest = np.setdiff1d(np.arange(d), out)
    return [out, rest]


def _check_groups(groups, d: int):
    allc = np.concatenate([np.asarray(g, dtype=np.int64) for g in groups])
    if allc.size != d or not np.array_equal(np.sort(allc), np.arange(d)):
        raise ValueError("groups must be disjoint and cover every channel")


def effective_bits(groups, bits, norm_bits: int = 0) -> float:
    """Average bits per channel: (sum_g d_g b_g + n_groups * norm_bits) / d."""
    sizes = np.array([len(g) for g in groups], dtype=np.float64)
    total = np.dot(sizes, np.asarray(bits, dtype=np.float64)) + len(groups) * norm_bits
    return float(total / sizes.sum())


def quantize_split(x, groups, instances):
    """Quantize every row of x [n, d] group by group.

    ``instances[g]`` is a dict with ``kind`` ("mse" or "prod"), ``rot`` [d_g, d_g],
    ``centroids``, ``boundaries``, ``bits`` and, for prod, ``S`` [m_g, d_g].  Returns one
    record dict per group, as :func:`oracle.quantizer.quantize_mse` / ``quantize_prod``
    return them for the sub-vectors.
    """
    x = np.asarray(x, dtype=np.float64)
    _check_groups(groups, x.shape[1])
    recs = []
    for ch, ins in zip(groups, instances):
        xs = x[:, np.asarray(ch, dtype=np.int64)]
        if ins["kind"] == "mse":
            recs.append(Q.quantize_mse(xs, ins["rot"], ins["centroids"], ins["boundaries"], ins["bits"]))
        elif ins["kind"] == "prod":
            recs.append(Q.quantize_prod(xs, ins["rot"], ins["S"], ins["centroids"], ins["boundaries"], ins["bits"]))
        else:
            raise ValueError("kind must be mse or prod")
    return recs


def dequantize_split(records, groups, instances, d: int) -> np.ndarray:
    """x_hat [n, d]: each group's reconstruction written back to its channels."""
    n = records[0]["norms"].shape[0]
    xh = np.zeros((n, d))
    for rec, ch, ins in zip(records, groups, instances):
        if ins["kind"] == "mse":
            part = Q.dequantize_mse(rec["idx"], rec["norms"], ins["rot"], ins["centroids"])
        else:
            part = Q.dequantize_prod(rec["chat"], rec["s"], rec["norms"], rec["rnorms"], ins["rot"], ins["S"])
        xh[:, np.asarray(ch, dtype=np.int64)] = part
    return xh


def estimate_split(q, records, groups, instances) -> np.ndarray:
    """est(q, x) [nq, n] = sum over groups of the group's estimate on q[:, ch_g]."""
    q = np.asarray(q, dtype=np.float64)
    total = None
    for rec, ch, ins in zip(records, groups, instances):
        qs = q[:, np.asarray(ch, dtype=np.int64)]
        if ins["kind"] == "mse":
            e = Q.estimate_mse(qs, ins["rot"], rec["idx"], rec["norms"], ins["centroids"])
        else:
            e = Q.estimate_prod(qs, ins["rot"], ins["S"], rec["chat"], rec["s"], rec["norms"], rec["rnorms"])
        total = e if total is None else total + e
    return total
