"""TurboQuant-mse and TurboQuant-prod, restated plainly in float64 (oracle).

R, *Method*: rotate by a random rotation Pi, then quantize each coordinate with the
precomputed Lloyd-Max codebook; TurboQuant-prod spends b-1 bits on that MSE stage
and encodes the residual with the 1-bit Quantized-JL transform, which makes the
inner-product estimate unbiased.  R, *Limitations*: the analysis is for unit
vectors and norms are stored separately.  LK, X thread 5/16: "Random rotation ->
scalar Lloyd-Max -> 1-bit QJL residual".

Readings taken where the pages are silent (all listed in the design notes):

* y = Pi @ (x / ||x||) with Pi row-major as given (fp32 values promoted to f64);
  a zero vector quantizes u = 0.
* idx_j = #{k : t_k < y_j}: a value exactly on a boundary takes the lower cell.
* Code numbering ascends with the centroid (0 = most negative).
* QJL: S has i.i.d. N(0,1) rows, m of them; the residual r = y - c[idx] is taken in
  the rotated unit-scale domain; sign bit s_i = 1 iff (S r)_i >= 0.
* Estimator constant sqrt(pi/2)/m: for s ~ N(0, I), E[<s,q'> sign<s,r>] =
  sqrt(2/pi) <q', r> / ||r||, so sqrt(pi/2)/m * ||r|| * sum_i <s_i,q'> sign<s_i,r>
  is unbiased for <q', r>.
* bits = 1 for prod means zero MSE bits (c_hat = 0) and pure QJL.

Packed record format (the library's contract, restated here from its definition):

* ``codes``: per vector W = ceil(d*b/32) little-endian uint32 words; code j occupies
  stream bits [j*b, j*b + b), least-significant bit first.  Unused bits are 0.
* ``signs`` (prod): per vector ceil(m/32) words; bit i%32 of word i//32 is s_i.
* ``norms``: ||x|| as float32; ``rnorms`` (prod): ||r|| as float32.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "rotate", "assign", "pack_codes", "unpack_codes", "pack_signs", "unpack_signs",
    "quantize_mse", "dequantize_mse", "quantize_prod", "dequantize_prod",
    "estimate_mse", "estimate_prod", "words_for",
]


def words_for(count: int, bits: int) -> int:
    """Number of uint32 words that hold ``count`` fields of ``bits`` bits."""
    return (count * bits + 31) // 32


def rotate(x: np.ndarray, rot: np.ndarray):
    """Return (norms, y) with y = rot @ (x / ||x||) per row; zero rows give y = 0."""
    x = np.asarray(x, dtype=np.float64)
    nu = np.sqrt(np.sum(x * x, axis=1))
    u = np.zeros_like(x)
    nz = nu > 0
    u[nz] = x[nz] / nu[nz, None]
    y = u @ np.asarray(rot, dtype=np.float64).T
    return nu, y


def assign(y: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    """idx = #{k : t_k < y} for each entry (nearest centroid; ties to the lower cell)."""
    t = np.asarray(boundaries, dtype=np.float64)
    return np.sum(y[..., None] > t, axis=-1).astype(np.int64)


def pack_codes(idx: np.ndarray, bits: int) -> np.ndarray:
    """Pack integer codes [n, d] into the LSB-first bit stream, uint32 [n, W]."""
    idx = np.asarray(idx, dtype=np.int64)
    n, d = idx.shape
    w = words_for(d, bits)
    if w == 0:
        return np.zeros((n, 0), dtype=np.uint32)
    stream = ((idx[:, :, None] >> np.arange(bits)[None, None, :]) & 1).reshape(n, d * bits)
    padded = np.zeros((n, w * 32), dtype=np.uint64)
    padded[:, : d * bits] = stream
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    words = (padded.reshape(n, w, 32) * weights[None, None, :]).sum(axis=2)
    return words.astype(np.uint32)


def unpack_codes(words: np.ndarray, d: int, bits: int) -> np.ndarray:
    """Inverse of :func:`pack_codes`."""
    words = np.asarray(words, dtype=np.uint64)
    n, w = words.shape
    stream = ((words[:, :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)).reshape(n, w * 32)
    stream = stream[:, : d * bits].reshape(n, d, bits).astype(np.int64)
    return np.sum(stream << np.arange(bits)[None, None, :], axis=2)


def pack_signs(s: np.ndarray) -> np.ndarray:
    """Sign bits [n, m] (0/1) -> uint32 [n, ceil(m/32)], bit i%32 of word i//32."""
    return pack_codes(np.asarray(s, dtype=np.int64), 1)


def unpack_signs(words: np.ndarray, m: int) -> np.ndarray:
    return unpack_codes(words, m, 1)


def quantize_mse(x, rot, centroids, boundaries, bits: int):
    """TurboQuant-mse (R, Method).  Returns dict(idx, y, norms, codes)."""
    nu, y = rotate(x, rot)
    idx = assign(y, boundaries)
    return {"idx": idx, "y": y, "norms": nu, "codes": pack_codes(idx, bits),
            "centroids": np.asarray(centroids, dtype=np.float64)}


def dequantize_mse(idx, norms, rot, centroids) -> np.ndarray:
    """x_hat = ||x|| * Pi^T c[idx] (the transpose of the given Pi, not its inverse)."""
    c = np.asarray(centroids, dtype=np.float64)[np.asarray(idx)]
    return np.asarray(norms, dtype=np.float64)[:, None] * (c @ np.asarray(rot, dtype=np.float64))


def quantize_prod(x, rot, S, centroids, boundaries, bits: int):
    """TurboQuant-prod with ``bits`` total: (bits-1)-bit MSE stage + 1-bit QJL residual.

    Returns dict(idx, y, norms, chat, r, rnorms, proj, s, codes, signs).
    """
    S = np.asarray(S, dtype=np.float64)
    nu, y = rotate(x, rot)
    if bits > 1:
        idx = assign(y, boundaries)
        chat = np.asarray(centroids, dtype=np.float64)[idx]
    else:
        idx = np.zeros(y.shape, dtype=np.int64)
        chat = np.zeros_like(y)
    r = y - chat
    gamma = np.sqrt(np.sum(r * r, axis=1))
    proj = r @ S.T
    s = (proj >= 0).astype(np.int64)
    return {"idx": idx, "y": y, "norms": nu, "chat": chat, "r": r, "rnorms": gamma,
            "proj": proj, "s": s, "codes": pack_codes(idx, bits - 1) if bits > 1 else
            np.zeros((y.shape[0], 0), dtype=np.uint32), "signs": pack_signs(s)}


def dequantize_prod(chat, s, norms, rnorms, rot, S) -> np.ndarray:
    """Unbiased reconstruction ||x|| Pi^T (c_hat + sqrt(pi/2)/m * gamma * S^T (2s-1))."""
    S = np.asarray(S, dtype=np.float64)
    m = S.shape[0]
    sk = (2.0 * np.asarray(s, dtype=np.float64) - 1.0) @ S
    yhat = np.asarray(chat, dtype=np.float64) + math.sqrt(math.pi / 2.0) / m * \
        np.asarray(rnorms, dtype=np.float64)[:, None] * sk
    return np.asarray(norms, dtype=np.float64)[:, None] * (yhat @ np.asarray(rot, dtype=np.float64))


def estimate_mse(q, rot, idx, norms, centroids) -> np.ndarray:
    """<q, x_hat> for every (query, record): ||x|| <Pi q, c[idx]>.  Shape [nq, n]."""
    qr = np.asarray(q, dtype=np.float64) @ np.asarray(rot, dtype=np.float64).T
    c = np.asarray(centroids, dtype=np.float64)[np.asarray(idx)]
    return (qr @ c.T) * np.asarray(norms, dtype=np.float64)[None, :]


def estimate_prod(q, rot, S, chat, s, norms, rnorms) -> np.ndarray:
    """Unbiased QJL inner-product estimate (R, Method; Results: "exactly unbiased").

    est = ||x|| ( <Pi q, c_hat> + sqrt(pi/2)/m * ||r|| * <S Pi q, 2s - 1> ).  Shape [nq, n].
    """
    S = np.asarray(S, dtype=np.float64)
    m = S.shape[0]
    qr = np.asarray(q, dtype=np.float64) @ np.asarray(rot, dtype=np.float64).T
    uq = qr @ S.T
    mse = qr @ np.asarray(chat, dtype=np.float64).T
    qjl = uq @ (2.0 * np.asarray(s, dtype=np.float64) - 1.0).T
    corr = math.sqrt(math.pi / 2.0) / m * np.asarray(rnorms, dtype=np.float64)[None, :] * qjl
    return (mse + corr) * np.asarray(norms, dtype=np.float64)[None, :]
