"""ctypes binding of libtq (include/tq.h): argument marshalling only.

Every computation runs in the CUDA library; PyTorch supplies device memory and the
current stream.  If ``libtq.so`` is missing the first call raises -- there is no CPU
fallback.  Build it with ``python -m kv_cache_compression_rotation_b200.build``.
"""
from __future__ import annotations

import ctypes as C
import math
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK = 0
STATUS_NAMES = {0: "TQ_OK", 1: "TQ_ERR_INVALID_ARG", 2: "TQ_ERR_UNSUPPORTED", 3: "TQ_ERR_ALIGNMENT",
                4: "TQ_ERR_ALIAS", 5: "TQ_ERR_CUDA", 6: "TQ_ERR_TIMEOUT", 7: "TQ_ERR_NOT_CONVERGED",
                8: "TQ_ERR_WORKSPACE"}
DIST = {"beta": 0, "gaussian": 1}
KIND_MSE, KIND_PROD, KIND_SPECTRAL = 0, 1, 2
F32, BF16, F16 = 0, 1, 2
MAX_TOP = 8

EXPORTS = [
    "tq_version", "tq_last_error", "tq_codebook_build", "tq_waterfill", "tq_spectral_calibrate",
    "tq_spectral_unit_codebooks", "tq_record_layout", "tq_quantize_mse", "tq_quantize_prod",
    "tq_quantize_spectral", "tq_dequantize", "tq_score_workspace", "tq_score",
    "tq_decode_attn_workspace", "tq_decode_attn", "tq_get_status", "tq_set_wait_limit", "tq_lut_scale",
    "tq_decode_attn_fixed_ws", "tq_quantize_split", "tq_score_split_workspace", "tq_score_split",
    "tq_decode_attn_split_workspace", "tq_decode_attn_split", "tq_spectral_descriptor", "tq_spectral_prepare",
    "tq_decode_attn_paged", "tq_prefill_attn_workspace", "tq_prefill_attn", "tq_quantize_workspace",
    "tq_quantize_ws",
]


class TqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Quantizer_t(C.Structure):
    _fields_ = [
        ("kind", C.c_int32), ("d", C.c_int32), ("bits", C.c_int32), ("m", C.c_int32),
        ("rot", C.c_void_p), ("S", C.c_void_p), ("centroids", C.c_void_p), ("boundaries", C.c_void_p),
        ("k_top", C.c_int32), ("tail_bits", C.c_int32), ("qjl", C.c_int32),
        ("top_bits", C.c_int32 * MAX_TOP),
        ("dim_sigma", C.c_void_p), ("unit_centroids", C.c_void_p), ("unit_boundaries", C.c_void_p),
        ("lut_scale", C.c_float), ("rot_pm1", C.c_int32),
    ]


class Packed_t(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("signs", C.c_void_p), ("norms", C.c_void_p), ("rnorms", C.c_void_p)]


MAX_GROUPS = 4


class Split_t(C.Structure):
    _fields_ = [("n_groups", C.c_int32), ("d", C.c_int32),
                ("groups", C.POINTER(Quantizer_t) * MAX_GROUPS), ("cols", C.c_void_p * MAX_GROUPS)]


class Pages_t(C.Structure):
    _fields_ = [("block_table", C.c_void_p), ("page_size", C.c_int32), ("max_pages", C.c_int32),
                ("num_pages", C.c_int64)]


class Layout_t(C.Structure):
    _fields_ = [("code_words", C.c_int32), ("sign_words", C.c_int32), ("has_norms", C.c_int32),
                ("has_rnorms", C.c_int32)]


_lib_handle = None


def lib():
    """Load libtq.so (raises if it was not built)."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libtq.so not found at {LIB_PATH}; build it with "
                               "`python -m kv_cache_compression_rotation_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i32, i64, f64p = C.c_void_p, C.c_int32, C.c_int64, C.POINTER(C.c_double)
        qp = C.POINTER(Quantizer_t)
        sig = {
            "tq_version": ([], C.c_char_p),
            "tq_last_error": ([], C.c_char_p),
            "tq_codebook_build": ([i32, i32, i32, C.c_double, f64p, f64p, C.POINTER(i32)], C.c_int),
            "tq_waterfill": ([f64p, i32, i32, i32, C.POINTER(i32)], C.c_int),
            "tq_spectral_calibrate": ([vp, i64, i32, f64p, f64p], C.c_int),
            "tq_spectral_unit_codebooks": ([f64p, f64p], C.c_int),
            "tq_record_layout": ([qp, C.POINTER(Layout_t)], C.c_int),
            "tq_quantize_mse": ([qp, vp, i32, i64, Packed_t, vp], C.c_int),
            "tq_quantize_prod": ([qp, vp, i32, i64, Packed_t, vp], C.c_int),
            "tq_quantize_spectral": ([qp, vp, i32, i64, Packed_t, vp], C.c_int),
            "tq_quantize_workspace": ([qp, i32, i64, C.POINTER(C.c_size_t)], C.c_int),
            "tq_quantize_ws": ([qp, vp, i32, i64, Packed_t, vp, C.c_size_t, vp], C.c_int),
            "tq_dequantize": ([qp, Packed_t, i64, vp, vp], C.c_int),
            "tq_score_workspace": ([qp, i64, i64, i32, C.POINTER(C.c_size_t)], C.c_int),
            "tq_score": ([qp, vp, i32, i64, Packed_t, i64, i32, vp, vp, vp, C.c_size_t, vp], C.c_int),
            "tq_decode_attn_workspace": ([qp, i32, i32, i32, i64, C.POINTER(C.c_size_t)], C.c_int),
            "tq_decode_attn": ([qp, qp, vp, i32, i32, i32, i32, i64, vp, Packed_t, Packed_t, C.c_float,
                                vp, vp, C.c_size_t, vp], C.c_int),
            "tq_decode_attn_fixed_ws": ([qp, qp, vp, i32, i32, i32, i32, i64, vp, Packed_t, Packed_t,
                                         C.c_float, vp, vp], C.c_int),
            "tq_get_status": ([vp], C.c_int),
            "tq_set_wait_limit": ([i64], C.c_int),
            "tq_lut_scale": ([f64p, i32, C.POINTER(C.c_float)], C.c_int),
            "tq_spectral_descriptor": ([f64p, f64p, i32, i32, i32, i32, i32, vp, vp, vp, vp, C.POINTER(i32),
                                        C.POINTER(C.c_float)], C.c_int),
            "tq_spectral_prepare": ([vp, i64, i32, i32, i32, i32, i32, vp, vp, vp, vp, C.POINTER(i32),
                                     C.POINTER(C.c_float), f64p], C.c_int),
            "tq_decode_attn_paged": ([qp, qp, vp, vp, vp, i32, i32, i32, i32, vp, C.POINTER(Pages_t), Packed_t,
                                      Packed_t, C.c_float, vp, vp, C.c_size_t, vp], C.c_int),
            "tq_prefill_attn_workspace": ([qp, i32, i32, i32, i32, i64, C.POINTER(C.c_size_t)], C.c_int),
            "tq_prefill_attn": ([qp, qp, vp, i32, i32, i32, i32, i32, vp, vp, C.POINTER(Pages_t), i64, Packed_t,
                                 Packed_t, C.c_float, vp, vp, C.c_size_t, vp], C.c_int),
            "tq_quantize_split": ([C.POINTER(Split_t), vp, i32, i64, C.POINTER(Packed_t), vp], C.c_int),
            "tq_score_split_workspace": ([C.POINTER(Split_t), i64, i64, i32, C.POINTER(C.c_size_t)], C.c_int),
            "tq_score_split": ([C.POINTER(Split_t), vp, i32, i64, C.POINTER(Packed_t), i64, i32, vp, vp, vp,
                                C.c_size_t, vp], C.c_int),
            "tq_decode_attn_split_workspace": ([C.POINTER(Split_t), C.POINTER(Split_t), i32, i32, i32, i64,
                                                C.POINTER(C.c_size_t)], C.c_int),
            "tq_decode_attn_split": ([C.POINTER(Split_t), C.POINTER(Split_t), vp, i32, i32, i32, i32, i64, vp,
                                      C.POINTER(Packed_t), C.POINTER(Packed_t), C.c_float, vp, vp, C.c_size_t,
                                      vp], C.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib_handle = L
    return _lib_handle


def _check(status: int) -> None:
    if status != TQ_OK:
        raise TqError(status, lib().tq_last_error().decode())


def _dptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dtype_code(t) -> int:
    import torch
    return {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}[t.dtype]


def version() -> str:
    return lib().tq_version().decode()


# ------------------------------------------------------------------ host math
def codebook_build(bits: int, dist: str = "beta", d: int = 0, sigma: float = 0.0):
    """Lloyd-Max codebook: (centroids [2^b], boundaries [2^b-1], iterations) as float64."""
    k = 1 << bits
    c = np.zeros(k, dtype=np.float64)
    t = np.zeros(k - 1, dtype=np.float64)
    it = C.c_int32(0)
    _check(lib().tq_codebook_build(d, bits, DIST[dist], float(sigma),
                                   c.ctypes.data_as(C.POINTER(C.c_double)),
                                   t.ctypes.data_as(C.POINTER(C.c_double)), C.byref(it)))
    return c, t, it.value


def waterfill(lam, budget: int, max_bits: int = 8) -> np.ndarray:
    lam = np.ascontiguousarray(lam, dtype=np.float64)
    out = np.zeros(lam.shape[0], dtype=np.int32)
    _check(lib().tq_waterfill(lam.ctypes.data_as(C.POINTER(C.c_double)), lam.shape[0], budget, max_bits,
                              out.ctypes.data_as(C.POINTER(C.c_int32))))
    return out


def spectral_calibrate(X: np.ndarray):
    X = np.ascontiguousarray(X, dtype=np.float32)
    n, d = X.shape
    vecs = np.zeros((d, d), dtype=np.float64)
    vals = np.zeros(d, dtype=np.float64)
    _check(lib().tq_spectral_calibrate(X.ctypes.data, n, d, vecs.ctypes.data_as(C.POINTER(C.c_double)),
                                       vals.ctypes.data_as(C.POINTER(C.c_double))))
    return vecs, vals


def lut_scale(values) -> float:
    """Shared scale s for a half-precision table of `values` (entries v / s)."""
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = C.c_float(0.0)
    _check(lib().tq_lut_scale(v.ctypes.data_as(C.POINTER(C.c_double)), v.shape[0], C.byref(out)))
    return float(out.value)


def spectral_unit_codebooks():
    c = np.zeros(510, dtype=np.float64)
    t = np.zeros(502, dtype=np.float64)
    _check(lib().tq_spectral_unit_codebooks(c.ctypes.data_as(C.POINTER(C.c_double)),
                                            t.ctypes.data_as(C.POINTER(C.c_double))))
    return c, t


# ------------------------------------------------------------------ descriptors
@dataclass
class Packed:
    """Packed records (structure of arrays) on the device."""
    codes: object
    signs: object = None
    norms: object = None
    rnorms: object = None

    def as_c(self) -> Packed_t:
        return Packed_t(_dptr(self.codes) if self.codes is not None and self.codes.numel() else None,
                        _dptr(self.signs), _dptr(self.norms), _dptr(self.rnorms))


class Quantizer:
    """Device-resident quantizer descriptor (owns the tensors the C struct points at)."""

    def __init__(self, kind: int, d: int, rot, *, bits=0, m=0, S=None, centroids=None, boundaries=None,
                 k_top=0, tail_bits=0, qjl=0, top_bits=(), dim_sigma=None, unit_c=None, unit_t=None,
                 lut_scale=0.0, rot_pm1=None):
        self.kind, self.d, self.bits, self.m = kind, d, bits, m
        self._keep = [rot, S, centroids, boundaries, dim_sigma, unit_c, unit_t]
        self.rot, self.S, self.centroids, self.boundaries = rot, S, centroids, boundaries
        self.dim_sigma, self.unit_c, self.unit_t = dim_sigma, unit_c, unit_t
        self.k_top, self.tail_bits, self.qjl, self.top_bits = k_top, tail_bits, qjl, tuple(top_bits)
        tb = (C.c_int32 * MAX_TOP)(*(list(top_bits) + [0] * (MAX_TOP - len(top_bits))))
        self.c = Quantizer_t(kind, d, bits, m, _dptr(rot), _dptr(S), _dptr(centroids), _dptr(boundaries),
                             k_top, tail_bits, qjl, tb, _dptr(dim_sigma), _dptr(unit_c), _dptr(unit_t),
                             float(lut_scale), int(bool(rot_pm1)))

    @property
    def ref(self):
        return C.byref(self.c)

    @staticmethod
    def _dev(a, device):
        import torch
        return torch.as_tensor(np.ascontiguousarray(a, dtype=np.float32), device=device).contiguous()

    @staticmethod
    def _is_pm1(rot) -> bool:
        """True when every entry of rot is +-1/sqrt(d) in fp32 (Hadamard-type rotation)."""
        r = np.asarray(rot, dtype=np.float32)
        return bool(np.all(np.abs(r) == np.float32(1.0 / math.sqrt(r.shape[0]))))

    @classmethod
    def mse(cls, rot, bits: int, dist: str = "beta", sigma: float = 0.0, device="cuda"):
        d = rot.shape[0]
        c, t, _ = codebook_build(bits, dist, d=d, sigma=sigma)
        return cls(KIND_MSE, d, cls._dev(rot, device), bits=bits,
                   centroids=cls._dev(c, device), boundaries=cls._dev(t, device), lut_scale=lut_scale(c),
                   rot_pm1=cls._is_pm1(rot))

    @classmethod
    def prod(cls, rot, S, bits: int, dist: str = "beta", sigma: float = 0.0, device="cuda"):
        d = rot.shape[0]
        m = S.shape[0]
        cen = bnd = None
        sc = 0.0
        if bits > 1:
            c, t, _ = codebook_build(bits - 1, dist, d=d, sigma=sigma)
            cen, bnd = cls._dev(c, device), cls._dev(t, device)
            sc = lut_scale(c)
        return cls(KIND_PROD, d, cls._dev(rot, device), bits=bits, m=m, S=cls._dev(S, device),
                   centroids=cen, boundaries=bnd, lut_scale=sc)

    @classmethod
    def _spectral_from_host(cls, d, k_top, tail_bits, qjl, S_top, device, host):
        rot, sig, uc, ut, top, lut = host
        return cls(KIND_SPECTRAL, d, cls._dev(rot, device), S=None if S_top is None else cls._dev(S_top, device),
                   k_top=k_top, tail_bits=tail_bits, qjl=1 if qjl else 0, top_bits=list(top[:k_top]),
                   dim_sigma=cls._dev(sig, device), unit_c=cls._dev(uc, device), unit_t=cls._dev(ut, device),
                   lut_scale=lut)

    @staticmethod
    def _spectral_outputs(d):
        return (np.zeros((d, d), dtype=np.float32), np.zeros(d, dtype=np.float32), np.zeros(510, dtype=np.float32),
                np.zeros(502, dtype=np.float32), np.zeros(MAX_TOP, dtype=np.int32))

    @classmethod
    def spectral(cls, eigvecs, eigvals, k_top: int, budget_bits: int, tail_bits: int, qjl: bool, S_top=None,
                 max_bits: int = 8, device="cuda"):
        """SPECTRAL descriptor from a given eigen-decomposition (rows of eigvecs, descending
        eigvals): tq_spectral_descriptor water-fills the top bits and builds the scales and
        codebooks; this wrapper only copies its outputs to the device."""
        d = eigvecs.shape[0]
        vecs = np.ascontiguousarray(eigvecs, dtype=np.float64)
        vals = np.ascontiguousarray(eigvals, dtype=np.float64)
        rot, sig, uc, ut, top = cls._spectral_outputs(d)
        lut = C.c_float(0.0)
        _check(lib().tq_spectral_descriptor(vecs.ctypes.data_as(C.POINTER(C.c_double)),
                                            vals.ctypes.data_as(C.POINTER(C.c_double)), d, k_top, budget_bits,
                                            tail_bits, max_bits, rot.ctypes.data, sig.ctypes.data, uc.ctypes.data,
                                            ut.ctypes.data, top.ctypes.data_as(C.POINTER(C.c_int32)), C.byref(lut)))
        return cls._spectral_from_host(d, k_top, tail_bits, qjl, S_top, device,
                                       (rot, sig, uc, ut, top, float(lut.value)))

    @classmethod
    def spectral_calibrated(cls, X, k_top: int, budget_bits: int, tail_bits: int, qjl: bool, S_top=None,
                            max_bits: int = 8, device="cuda"):
        """SPECTRAL descriptor straight from calibration rows X [n, d] (tq_spectral_prepare:
        calibration, water-filling, scales and codebooks in the library).  Returns
        (quantizer, eigenvalues)."""
        X = np.ascontiguousarray(X, dtype=np.float32)
        n, d = X.shape
        rot, sig, uc, ut, top = cls._spectral_outputs(d)
        vals = np.zeros(d, dtype=np.float64)
        lut = C.c_float(0.0)
        _check(lib().tq_spectral_prepare(X.ctypes.data, n, d, k_top, budget_bits, tail_bits, max_bits,
                                         rot.ctypes.data, sig.ctypes.data, uc.ctypes.data, ut.ctypes.data,
                                         top.ctypes.data_as(C.POINTER(C.c_int32)), C.byref(lut),
                                         vals.ctypes.data_as(C.POINTER(C.c_double))))
        q = cls._spectral_from_host(d, k_top, tail_bits, qjl, S_top, device, (rot, sig, uc, ut, top, float(lut.value)))
        return q, vals

    def layout(self) -> Layout_t:
        L = Layout_t()
        _check(lib().tq_record_layout(self.ref, C.byref(L)))
        return L

    def alloc(self, n: int, device="cuda") -> Packed:
        """Zeroed packed arrays for n records."""
        import torch
        L = self.layout()
        codes = torch.zeros((n, L.code_words), dtype=torch.int32, device=device)
        signs = torch.zeros((n, L.sign_words), dtype=torch.int32, device=device) if L.sign_words else None
        norms = torch.zeros(n, dtype=torch.float32, device=device) if L.has_norms else None
        rnorms = torch.zeros(n, dtype=torch.float32, device=device) if L.has_rnorms else None
        return Packed(codes, signs, norms, rnorms)


# ------------------------------------------------------------------ device calls
def quantize(q: Quantizer, x, out: Optional[Packed] = None, stream=None) -> Packed:
    """tq_quantize_{mse,prod,spectral} of x [n, d] (fp32 / bf16 / fp16 CUDA tensor)."""
    assert x.is_cuda and x.is_contiguous() and x.shape[-1] == q.d
    n = x.numel() // q.d
    out = q.alloc(n, x.device) if out is None else out
    fn = {KIND_MSE: lib().tq_quantize_mse, KIND_PROD: lib().tq_quantize_prod,
          KIND_SPECTRAL: lib().tq_quantize_spectral}[q.kind]
    _check(fn(q.ref, x.data_ptr(), _dtype_code(x), n, out.as_c(), _stream(stream)))
    return out


def tq_quantize_workspace_bytes(q: Quantizer, x) -> int:
    ws = C.c_size_t(0)
    _check(lib().tq_quantize_workspace(q.ref, _dtype_code(x), x.numel() // q.d, C.byref(ws)))
    return ws.value


def quantize_ws(q: Quantizer, x, out: Optional[Packed] = None, workspace=None, stream=None) -> Packed:
    """tq_quantize_ws: the same records as quantize(), with device scratch (wide fp32 vectors
    take the tensor-core split-precision path)."""
    import torch
    assert x.is_cuda and x.is_contiguous() and x.shape[-1] == q.d
    n = x.numel() // q.d
    out = q.alloc(n, x.device) if out is None else out
    ws = C.c_size_t(0)
    _check(lib().tq_quantize_workspace(q.ref, _dtype_code(x), n, C.byref(ws)))
    if workspace is None or workspace.numel() < ws.value:
        workspace = torch.empty(max(ws.value, 16), dtype=torch.uint8, device=x.device)
    _check(lib().tq_quantize_ws(q.ref, x.data_ptr(), _dtype_code(x), n, out.as_c(), workspace.data_ptr(),
                                workspace.numel(), _stream(stream)))
    return out


def dequantize(q: Quantizer, packed: Packed, n: int, stream=None):
    import torch
    out = torch.empty((n, q.d), dtype=torch.float32, device=packed.codes.device)
    _check(lib().tq_dequantize(q.ref, packed.as_c(), n, out.data_ptr(), _stream(stream)))
    return out


def score(q: Quantizer, qv, packed: Packed, n: int, topk: int = 0, stream=None):
    """Dense estimates [nq, n], or (scores [nq, topk], ids [nq, topk]) when topk > 0."""
    import torch
    nq = qv.numel() // q.d
    ws = C.c_size_t(0)
    _check(lib().tq_score_workspace(q.ref, nq, n, topk, C.byref(ws)))
    work = torch.empty(max(ws.value, 16), dtype=torch.uint8, device=qv.device)
    if topk == 0:
        scores = torch.empty((nq, n), dtype=torch.float32, device=qv.device)
        ids = None
    else:
        scores = torch.empty((nq, topk), dtype=torch.float32, device=qv.device)
        ids = torch.empty((nq, topk), dtype=torch.int32, device=qv.device)
    _check(lib().tq_score(q.ref, qv.data_ptr(), _dtype_code(qv), nq, packed.as_c(), n, topk, scores.data_ptr(),
                          _dptr(ids), work.data_ptr(), ws.value, _stream(stream)))
    return scores if topk == 0 else (scores, ids)


class Split:
    """Outlier-channel split: group g is the quantizer ``groups[g]`` over the channels
    ``cols[g]`` (int32 CUDA tensor) of d-wide vectors."""

    def __init__(self, d: int, groups, cols):
        assert 1 <= len(groups) == len(cols) <= MAX_GROUPS
        self.d, self.groups, self.cols = d, list(groups), list(cols)
        gp = (C.POINTER(Quantizer_t) * MAX_GROUPS)(*[C.pointer(q.c) for q in self.groups])
        cp = (C.c_void_p * MAX_GROUPS)(*[_dptr(c) for c in self.cols])
        self.c = Split_t(len(self.groups), d, gp, cp)

    @property
    def ref(self):
        return C.byref(self.c)

    def alloc(self, n: int, device="cuda"):
        return [q.alloc(n, device) for q in self.groups]


def _packed_array(packs):
    return (Packed_t * len(packs))(*[p.as_c() for p in packs])


def quantize_split(sp: Split, x, out=None, stream=None):
    """tq_quantize_split of x [n, d]: one list entry of packed records per group."""
    assert x.is_cuda and x.is_contiguous() and x.shape[-1] == sp.d
    n = x.numel() // sp.d
    out = sp.alloc(n, x.device) if out is None else out
    _check(lib().tq_quantize_split(sp.ref, x.data_ptr(), _dtype_code(x), n, _packed_array(out), _stream(stream)))
    return out


def score_split(sp: Split, qv, packs, n: int, topk: int = 0, stream=None):
    """Summed split estimates [nq, n], or (scores, ids) of the top-k when topk > 0."""
    import torch
    nq = qv.numel() // sp.d
    ws = C.c_size_t(0)
    _check(lib().tq_score_split_workspace(sp.ref, nq, n, topk, C.byref(ws)))
    work = torch.empty(max(ws.value, 16), dtype=torch.uint8, device=qv.device)
    if topk == 0:
        scores = torch.empty((nq, n), dtype=torch.float32, device=qv.device)
        ids = None
    else:
        scores = torch.empty((nq, topk), dtype=torch.float32, device=qv.device)
        ids = torch.empty((nq, topk), dtype=torch.int32, device=qv.device)
    _check(lib().tq_score_split(sp.ref, qv.data_ptr(), _dtype_code(qv), nq, _packed_array(packs), n, topk,
                                scores.data_ptr(), _dptr(ids), work.data_ptr(), ws.value, _stream(stream)))
    return scores if topk == 0 else (scores, ids)


def decode_attn_split(ks: Split, vs: Split, q, seq_lens, kpacks, vpacks, Nmax: int, Hkv: int, scale=None,
                      out=None, stream=None):
    """tq_decode_attn_split for q [B, Hq, d] over split caches (one packed list per split)."""
    import torch
    B, Hq, d = q.shape
    assert d == ks.d == vs.d and q.is_contiguous()
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ws = C.c_size_t(0)
    _check(lib().tq_decode_attn_split_workspace(ks.ref, vs.ref, B, Hq, Hkv, Nmax, C.byref(ws)))
    work = torch.empty(max(ws.value, 16), dtype=torch.uint8, device=q.device)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device) if out is None else out
    _check(lib().tq_decode_attn_split(ks.ref, vs.ref, q.data_ptr(), _dtype_code(q), B, Hq, Hkv, Nmax,
                                      seq_lens.data_ptr(), _packed_array(kpacks), _packed_array(vpacks),
                                      float(scale), out.data_ptr(), work.data_ptr(), ws.value, _stream(stream)))
    return out


def decode_workspace_bytes(kq: Quantizer, B: int, Hq: int, Hkv: int, Nmax: int) -> int:
    ws = C.c_size_t(0)
    _check(lib().tq_decode_attn_workspace(kq.ref, B, Hq, Hkv, Nmax, C.byref(ws)))
    return ws.value


def decode_attn(kq: Quantizer, vq: Quantizer, q, seq_lens, kcache: Packed, vcache: Packed, Nmax: int,
                Hkv: int, scale: Optional[float] = None, out=None, workspace=None, stream=None):
    """One decode-attention step; q [B, Hq, d], seq_lens int32 [B] on the device."""
    import torch
    B, Hq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = decode_workspace_bytes(kq, B, Hq, Hkv, Nmax)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device) if out is None else out
    _check(lib().tq_decode_attn(kq.ref, vq.ref, q.data_ptr(), _dtype_code(q), B, Hq, Hkv, Nmax,
                                seq_lens.data_ptr(), kcache.as_c(), vcache.as_c(), float(scale), out.data_ptr(),
                                workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return out


class Pages:
    """Paged record pool: block_table int32 [B, max_pages] CUDA tensor of page ids, page_size
    tokens per page (a multiple of 16), num_pages pages; token t of (b, kv-head h) is record
    (block_table[b, t // page_size] * Hkv + h) * page_size + t % page_size of every array."""

    def __init__(self, block_table, page_size: int, num_pages: int):
        assert block_table.dtype.is_floating_point is False and block_table.is_contiguous()
        self.block_table, self.page_size, self.num_pages = block_table, page_size, num_pages
        self.max_pages = block_table.shape[1]
        self.c = Pages_t(block_table.data_ptr(), page_size, self.max_pages, num_pages)

    @property
    def ref(self):
        return C.byref(self.c)

    def records(self, Hkv: int) -> int:
        return self.num_pages * Hkv * self.page_size


def decode_attn_paged(kq: Quantizer, vq: Quantizer, q, seq_lens, pages: Pages, kpool: Packed, vpool: Packed,
                      Hkv: int, k_new=None, v_new=None, scale: Optional[float] = None, out=None, workspace=None,
                      stream=None):
    """tq_decode_attn_paged: append k_new / v_new [B*Hkv, d] (optional) as token seq_lens[b]-1,
    then one decode step over the pool; q [B, Hq, d]."""
    import torch
    B, Hq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = decode_workspace_bytes(kq, B, Hq, Hkv, pages.max_pages * pages.page_size)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device) if out is None else out
    _check(lib().tq_decode_attn_paged(kq.ref, vq.ref, q.data_ptr(), _dptr(k_new), _dptr(v_new), _dtype_code(q), B, Hq,
                                      Hkv, seq_lens.data_ptr(), pages.ref, kpool.as_c(), vpool.as_c(), float(scale),
                                      out.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return out


def prefill_attn(kq: Quantizer, vq: Quantizer, q, q_pos, kv_lens, kcache: Packed, vcache: Packed, Hkv: int,
                 Nmax: int = 0, pages: Optional[Pages] = None, scale: Optional[float] = None, out=None,
                 workspace=None, stream=None):
    """tq_prefill_attn: causal attention of q [B, Hq, T, d] at positions q_pos [B, T] over the
    packed cache ([B, Hkv, Nmax] records, or a paged pool)."""
    import torch
    B, Hq, T, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    n = pages.max_pages * pages.page_size if pages is not None else Nmax
    ws = C.c_size_t(0)
    _check(lib().tq_prefill_attn_workspace(kq.ref, B, Hq, Hkv, T, n, C.byref(ws)))
    if workspace is None or workspace.numel() < ws.value:
        workspace = torch.empty(max(ws.value, 16), dtype=torch.uint8, device=q.device)
    out = torch.empty((B, Hq, T, d), dtype=torch.float32, device=q.device) if out is None else out
    _check(lib().tq_prefill_attn(kq.ref, vq.ref, q.data_ptr(), _dtype_code(q), B, Hq, Hkv, T, q_pos.data_ptr(),
                                 kv_lens.data_ptr(), pages.ref if pages is not None else None, Nmax, kcache.as_c(),
                                 vcache.as_c(), float(scale), out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                 _stream(stream)))
    return out


def get_status(stream=None) -> int:
    """Synchronize and return the device status code (0 = OK, 6 = a bounded wait timed out)."""
    return lib().tq_get_status(_stream(stream))


def set_wait_limit(polls: int) -> None:
    _check(lib().tq_set_wait_limit(polls))
