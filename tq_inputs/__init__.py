"""Seeded synthetic inputs shared by the CPU oracle, the GPU tests and the bench.

This module only draws random numbers and shapes them into the workloads' inputs;
it holds none of the quantizer's arithmetic (no codebooks, no rotation of data, no
packing).  Both sides of every parity test receive the same arrays from here.

Workloads (the quantities the TurboQuant pages quantize):

* ``haar_rotation``  - the random orthogonal rotation Pi.  The review of
  "TurboQuant: Online Vector Quantization with Near-optimal Distortion Rate"
  (section *Method*) asks for "a random rotation"; the launch kit (LAUNCH.md,
  *Show HN post*) lists a dense-QR mode.  We draw Pi as the Q factor of a Gaussian
  matrix with the signs of R's diagonal folded in, which is Haar distributed.
* ``gaussian_matrix`` - the QJL projection S with i.i.d. N(0, 1) entries
  ("1-bit Quantized-JL", review *Method*).
* ``kv_spectrum`` / ``anisotropic`` - K/V rows with ~80 % of the variance in 4 of
  128 directions (SpectralQuant thread by @ashwingop, post 2).  The fractions are
  chosen so that greedy reverse water-filling gives the [5, 3, 2, 2] split of
  post 6 (the post's own lambda_0 = 0.50, lambda_3 = 0.04 cannot give it).
* ``unit_gaussian`` - unit-norm Gaussian vectors, the stand-in for the OpenAI3
  embeddings of the review's vector-search experiment (*Validation*).

Small draws use NumPy's PCG64 in float64 and are cast at the end (bf16 by
round-to-nearest-even through torch).  Draws too large for host memory use a
seeded ``torch.Generator`` on the target device; the oracle then receives exact
copies of the rows it needs.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "SEEDS", "haar_rotation", "hadamard_rotation", "gaussian_matrix", "kv_spectrum", "anisotropic",
    "iid_normal", "unit_gaussian", "to_bf16_f64", "anisotropic_torch", "normal_torch",
    "planted_outliers",
]

# Seed plan: role base + workload number (1..5).
SEEDS = {
    "rotation": 1000, "qjl": 2000, "basis": 3000, "keys": 4000, "values": 5000,
    "queries": 6000, "calib_keys": 7000, "calib_values": 7100, "db": 8000,
    "db_queries": 8001, "qjl_trials": 9000,
}


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def haar_rotation(d: int, seed: int, dtype=np.float32) -> np.ndarray:
    """Haar-random orthogonal d x d matrix (row-major; y = Pi @ x)."""
    g = _rng(seed).standard_normal((d, d))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return q.astype(dtype)


def hadamard_rotation(d: int, seed: int) -> np.ndarray:
    """Randomized Hadamard rotation H diag(s) / sqrt(d), d a power of two: H the Sylvester
    Hadamard matrix, s i.i.d. random signs (the launch kit's O(d log d) rotation mode).  Every
    entry is exactly +-float32(1/sqrt(d))."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    s = np.where(_rng(seed).random(d) < 0.5, -1.0, 1.0)
    c = np.float32(1.0 / np.sqrt(d))
    return (h * s[None, :]).astype(np.float32) * c


def gaussian_matrix(m: int, d: int, seed: int, dtype=np.float32) -> np.ndarray:
    """m x d matrix with i.i.d. N(0, 1) entries."""
    return _rng(seed).standard_normal((m, d)).astype(dtype)


def kv_spectrum(d: int = 128) -> np.ndarray:
    """Variance fractions per principal direction (sum 1), descending.

    Top four hold 80.2 % of the variance; the remaining 19.8 % is spread evenly.
    """
    top = np.array([0.72, 0.054, 0.016, 0.012])
    rest = np.full(d - 4, 0.198 / (d - 4))
    lam = np.concatenate([top, rest])
    return lam / lam.sum()


def iid_normal(shape, seed: int, std: float = 1.0) -> np.ndarray:
    """float64 N(0, std^2) draws."""
    return _rng(seed).standard_normal(shape) * std


def anisotropic(n: int, d: int, basis: np.ndarray, seed: int, lam=None) -> np.ndarray:
    """float64 rows k = U (sqrt(d * lam) * z), z ~ N(0, I): covariance U diag(d lam) U^T.

    tr(C) = d, so a query q ~ N(0, I) gives q.k / sqrt(d) unit variance.
    """
    lam = kv_spectrum(d) if lam is None else np.asarray(lam, dtype=np.float64)
    z = _rng(seed).standard_normal((n, d))
    return (z * np.sqrt(d * lam)[None, :]) @ basis.astype(np.float64).T


def planted_outliers(n: int, d: int, channels, scale: float, seed: int) -> np.ndarray:
    """float64 rows N(0, I) whose listed channels are multiplied by ``scale``: keys with a
    few high-magnitude channels, the structure the outlier-channel split targets."""
    x = _rng(seed).standard_normal((n, d))
    x[:, np.asarray(channels, dtype=np.int64)] *= scale
    return x


def unit_gaussian(n: int, d: int, seed: int) -> np.ndarray:
    """float64 rows drawn N(0, I) and scaled to unit norm."""
    g = _rng(seed).standard_normal((n, d))
    return g / np.linalg.norm(g, axis=1, keepdims=True)


def to_bf16_f64(a: np.ndarray):
    """Round to bfloat16 (RNE, via torch) and return (torch bf16 tensor, exact float64 copy)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t, t.to(torch.float64).numpy()


# ---- device-side draws for sizes that do not fit the host comfortably ----

def normal_torch(shape, seed: int, device, dtype=None):
    """N(0, 1) draws from a seeded torch generator on ``device`` (float32)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return t if dtype is None else t.to(dtype)


def anisotropic_torch(n: int, d: int, basis, seed: int, device, chunk: int = 1 << 21,
                      out_dtype=None, lam=None):
    """Same law as :func:`anisotropic`, drawn on ``device`` in chunks, returned as ``out_dtype``."""
    import torch
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    lam = kv_spectrum(d) if lam is None else np.asarray(lam, dtype=np.float64)
    scale = torch.tensor(np.sqrt(d * lam), dtype=torch.float32, device=device)
    ut = torch.as_tensor(np.ascontiguousarray(basis, dtype=np.float32), device=device).t().contiguous()
    out = torch.empty((n, d), dtype=out_dtype, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        z = torch.randn((e - s, d), generator=g, device=device, dtype=torch.float32)
        out[s:e] = ((z * scale) @ ut).to(out_dtype)
    return out
