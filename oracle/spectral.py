"""SpectralQuant-style variant, restated plainly in float64 (oracle).

SQ post 4: rotate by the eigenvectors of the K covariance measured in a calibration
pass, so dim 0 carries the largest variance lambda_0.  SQ post 6: allocate bits over
the top signal dims by water-filling ("Shannon-Berger"), e.g. [3,3,3,3] -> [5,3,2,2].
SQ post 5: apply the 1-bit JL correction only to the top 4 signal dims (4 sign bits).

Readings taken where the posts are silent:

* Calibration uses the uncentred second moment M = X^T X / n (equal to the
  covariance for zero-mean data, and no stored mean is needed); eigenpairs from
  ``numpy.linalg.eigh``, sorted by descending eigenvalue, each eigenvector's sign
  flipped so its largest-magnitude component is positive (ties: lowest index).
* "Water-filling" is Shannon reverse water-filling in integer bits: distortion
  lambda_j 4^(-b_j); each of ``budget`` bits goes to argmax_j lambda_j 4^(-b_j)
  (ties: lowest j; dims capped at ``max_bits``).
* Dimension j is quantized with sqrt(lambda_j) times the standard-normal Lloyd-Max
  codebook of b_j bits; there is no per-vector norm.
* QJL on the top-k residual r = z_top - c_hat_top with a k x k Gaussian S_top;
  estimate = sum_j q~_j c_hat_j + sqrt(pi/2)/k * ||r|| * <S_top q~_top, 2s - 1>,
  q~ = rot @ q.

Record layout (the library's contract, restated from its definition): a head of
ceil((sum_{j<k} b_j + k_qjl)/32) words holding the top-k codes LSB-first in dim
order followed by the k_qjl sign bits; then ceil(d * tail_bits / 32) tail words
holding dim j's code at stream bits [j*tail_bits, (j+1)*tail_bits) for j >= k
(fields of dims j < k are 0).  ``rnorms`` holds ||r|| when QJL is on.
"""
from __future__ import annotations

import math

import numpy as np

from .codebook import lloyd_max
from .quantizer import unpack_codes

__all__ = ["calibrate", "waterfill", "build_descriptor", "quantize_spectral",
           "dequantize_spectral", "estimate_spectral", "head_words", "record_words",
           "unpack_spectral"]


def calibrate(X: np.ndarray):
    """Eigen-decomposition of the second-moment matrix (SQ post 4).

    Returns (eigvecs [d, d] with row j = eigenvector j, eigvals [d]) sorted descending.
    """
    X = np.asarray(X, dtype=np.float64)
    M = X.T @ X / X.shape[0]
    w, v = np.linalg.eigh(M)
    order = np.argsort(-w, kind="stable")
    w = w[order]
    v = v[:, order].T.copy()
    for j in range(v.shape[0]):
        k = int(np.argmax(np.abs(v[j])))
        if v[j, k] < 0:
            v[j] = -v[j]
    return v, w


def waterfill(lam, budget: int, max_bits: int = 8):
    """Greedy integer reverse water-filling (SQ post 6)."""
    lam = np.asarray(lam, dtype=np.float64)
    b = np.zeros(lam.shape[0], dtype=np.int64)
    for _ in range(budget):
        gain = np.where(b < max_bits, lam * np.power(4.0, -b), -np.inf)
        j = int(np.argmax(gain))          # first maximum -> lowest index on ties
        if not np.isfinite(gain[j]):
            break
        b[j] += 1
    return b


def build_descriptor(eigvecs, eigvals, k_top: int, budget: int, tail_bits: int,
                     qjl: bool, S_top=None, max_bits: int = 8):
    """Per-dimension bits, scales and codebooks for the spectral quantizer."""
    d = eigvecs.shape[0]
    lam = np.maximum(np.asarray(eigvals, dtype=np.float64), 0.0)
    bits = np.full(d, tail_bits, dtype=np.int64)
    bits[:k_top] = waterfill(lam[:k_top], budget, max_bits)
    sigma = np.sqrt(lam)
    books = {}
    for b in sorted(set(int(v) for v in bits)):
        if b > 0:
            c, t, _ = lloyd_max(b, "gaussian", sigma=1.0)
            books[b] = (c, t)
    return {"rot": np.asarray(eigvecs, dtype=np.float64), "bits": bits, "sigma": sigma,
            "books": books, "k_top": k_top, "tail_bits": tail_bits, "qjl": qjl,
            "S_top": None if S_top is None else np.asarray(S_top, dtype=np.float64)}


def head_words(desc) -> int:
    k = desc["k_top"]
    nb = int(np.sum(desc["bits"][:k])) + (k if desc["qjl"] else 0)
    return (nb + 31) // 32


def record_words(desc) -> int:
    d = desc["bits"].shape[0]
    return head_words(desc) + (d * desc["tail_bits"] + 31) // 32


def _pack_record(idx_row, s_row, desc) -> np.ndarray:
    k = desc["k_top"]
    d = idx_row.shape[0]
    hw = head_words(desc)
    tb = desc["tail_bits"]
    tw = (d * tb + 31) // 32
    head = 0
    pos = 0
    for j in range(k):
        head |= int(idx_row[j]) << pos
        pos += int(desc["bits"][j])
    if desc["qjl"]:
        for i in range(k):
            head |= int(s_row[i]) << pos
            pos += 1
    tail = 0
    for j in range(k, d):
        tail |= int(idx_row[j]) << (j * tb)
    out = np.zeros(hw + tw, dtype=np.uint32)
    for w in range(hw):
        out[w] = (head >> (32 * w)) & 0xFFFFFFFF
    for w in range(tw):
        out[hw + w] = (tail >> (32 * w)) & 0xFFFFFFFF
    return out


def unpack_spectral(codes, desc):
    """Inverse of the record layout: (idx [n, d], s [n, k_top]) from packed records."""
    codes = np.asarray(codes, dtype=np.uint32)
    n = codes.shape[0]
    d = desc["bits"].shape[0]
    k = desc["k_top"]
    hw = head_words(desc)
    tb = desc["tail_bits"]
    # the tail is the plain LSB-first code stream of d fields (fields of dims < k are 0)
    idx = unpack_codes(codes[:, hw:], d, tb)
    idx[:, :k] = 0
    s = np.zeros((n, k), dtype=np.int64)
    for i in range(n):
        head = sum(int(codes[i, w]) << (32 * w) for w in range(hw))
        pos = 0
        for j in range(k):
            b = int(desc["bits"][j])
            idx[i, j] = (head >> pos) & ((1 << b) - 1)
            pos += b
        if desc["qjl"]:
            for j in range(k):
                s[i, j] = (head >> (pos + j)) & 1
    return idx, s


def quantize_spectral(x, desc):
    """z = rot @ x; per-dim nearest centroid of sqrt(lambda_j) * codebook(b_j); QJL on top-k."""
    x = np.asarray(x, dtype=np.float64)
    z = x @ desc["rot"].T
    n, d = z.shape
    idx = np.zeros((n, d), dtype=np.int64)
    chat = np.zeros((n, d))
    for j in range(d):
        b = int(desc["bits"][j])
        if b == 0:
            continue
        c, t = desc["books"][b]
        sj = desc["sigma"][j]
        idx[:, j] = np.sum(z[:, j, None] > sj * t[None, :], axis=1)
        chat[:, j] = sj * c[idx[:, j]]
    k = desc["k_top"]
    out = {"z": z, "idx": idx, "chat": chat}
    if desc["qjl"]:
        r = z[:, :k] - chat[:, :k]
        out["r"] = r
        out["rnorms"] = np.sqrt(np.sum(r * r, axis=1))
        out["proj"] = r @ desc["S_top"].T
        out["s"] = (out["proj"] >= 0).astype(np.int64)
    s = out.get("s", np.zeros((n, k), dtype=np.int64))
    out["codes"] = np.stack([_pack_record(idx[i], s[i], desc) for i in range(n)]) if n else \
        np.zeros((0, record_words(desc)), dtype=np.uint32)
    return out


def dequantize_spectral(chat, desc) -> np.ndarray:
    """x_hat = rot^T c_hat (values; no QJL term)."""
    return np.asarray(chat, dtype=np.float64) @ desc["rot"]


def estimate_spectral(q, desc, chat, s=None, rnorms=None) -> np.ndarray:
    """Inner-product estimate [nq, n] (SQ post 5: QJL on the top-k dims only)."""
    qt = np.asarray(q, dtype=np.float64) @ desc["rot"].T
    est = qt @ np.asarray(chat, dtype=np.float64).T
    if desc["qjl"]:
        k = desc["k_top"]
        uq = qt[:, :k] @ desc["S_top"].T
        corr = uq @ (2.0 * np.asarray(s, dtype=np.float64) - 1.0).T
        est = est + math.sqrt(math.pi / 2.0) / k * np.asarray(rnorms)[None, :] * corr
    return est
