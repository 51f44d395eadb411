"""libtq host functions and C-ABI checks that need no GPU.

The library must load and export every entry point include/tq.h declares; its host math
(codebooks, water-filling, calibration) must agree with the oracle; argument validation
must reject bad calls before any launch.
"""
import ctypes as C
import os
import re

import numpy as np
import pytest

import tq_inputs as ti
from oracle import spectral as OSP
from oracle.codebook import lloyd_max

K = pytest.importorskip("kv_cache_compression_rotation_b200")
T = K.tq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(T.LIB_PATH):
        from kv_cache_compression_rotation_b200 import build as B
        B.build()
    return T.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(T.EXPORTS)


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(T, "LIB_PATH", "/nonexistent/libtq.so")
    monkeypatch.setattr(T, "_lib_handle", None)
    with pytest.raises(RuntimeError):
        T.lib()


@pytest.mark.parametrize("dist,d,bits", [("beta", 128, b) for b in (1, 2, 3, 4, 5)] +
                         [("beta", 1536, b) for b in (1, 2, 3, 4)] +
                         [("beta", 8, b) for b in (1, 2, 3)] + [("beta", 2, 3), ("beta", 3, 2)] +
                         [("gaussian", None, b) for b in (1, 2, 3, 4, 5)])
def test_codebook_matches_oracle(lib, dist, d, bits):
    sigma = 0.37 if dist == "gaussian" else 0.0
    c, t, it = K.codebook_build(bits, dist, d=d or 0, sigma=sigma)
    co, to, _ = lloyd_max(bits, dist, d=d, sigma=sigma or None)
    # both stop at a largest move of 1e-13 * scale; the distance to the fixed point is
    # that move over (1 - contraction rate), far below 1e-9 relative for b <= 5
    assert np.max(np.abs(c - co) / np.abs(co)) < 1e-9
    assert np.max(np.abs(t - to)) < 1e-9 * np.max(np.abs(co))
    assert it >= 1


def test_codebook_rejects_bad_args(lib):
    with pytest.raises(T.TqError):
        K.codebook_build(0, "beta", d=128)
    with pytest.raises(T.TqError):
        K.codebook_build(3, "beta", d=1)
    with pytest.raises(T.TqError):
        K.codebook_build(3, "gaussian", sigma=-1.0)


def test_waterfill_matches_oracle(lib):
    rng = np.random.Generator(np.random.PCG64(7))
    for _ in range(50):
        k = int(rng.integers(1, 9))
        lam = rng.uniform(0.001, 1.0, size=k)
        budget = int(rng.integers(0, 30))
        assert list(K.waterfill(lam, budget, 8)) == list(OSP.waterfill(lam, budget, 8))
    assert list(K.waterfill(ti.kv_spectrum(128)[:4], 12)) == [5, 3, 2, 2]


def test_calibration_matches_oracle(lib):
    d, n = 128, 4096
    U = ti.haar_rotation(d, 3004).astype(np.float64)
    X = ti.anisotropic(n, d, U, 7000).astype(np.float32)
    v, w = K.spectral_calibrate(X)
    vo, wo = OSP.calibrate(X.astype(np.float64))
    assert np.max(np.abs(w - wo) / np.abs(wo).max()) < 1e-9
    # well-separated leading eigenvectors agree exactly, including the sign rule
    for j in range(4):
        assert np.max(np.abs(v[j] - vo[j])) < 1e-8
    # the tail is nearly degenerate: compare the projector onto it
    P = v[4:].T @ v[4:]
    Po = vo[4:].T @ vo[4:]
    assert np.max(np.abs(P - Po)) < 1e-8
    assert np.max(np.abs(v @ v.T - np.eye(d))) < 1e-10


def test_unit_codebooks(lib):
    c, t = K.spectral_unit_codebooks()
    for b in range(1, 9):
        co, to, _ = lloyd_max(b, "gaussian", sigma=1.0) if b <= 6 else (None, None, None)
        if co is None:
            continue
        off_c, off_t = (1 << b) - 2, (1 << b) - b - 1
        assert np.max(np.abs(c[off_c:off_c + (1 << b)] - co)) < 1e-9 * np.max(np.abs(co))
        assert np.max(np.abs(t[off_t:off_t + (1 << b) - 1] - to)) < 1e-9 * np.max(np.abs(co))


FAKE = 0x10000  # 16-byte aligned placeholder device address (never dereferenced here)


def _q(kind, d=128, bits=3, m=0, **kw):
    q = T.Quantizer_t()
    q.kind, q.d, q.bits, q.m = kind, d, bits, m
    q.rot = FAKE
    q.centroids = FAKE + 0x1000
    q.boundaries = FAKE + 0x2000
    q.S = kw.get("S", None)
    q.k_top = kw.get("k_top", 0)
    q.tail_bits = kw.get("tail_bits", 0)
    q.qjl = kw.get("qjl", 0)
    for i, b in enumerate(kw.get("top_bits", [])):
        q.top_bits[i] = b
    q.dim_sigma = kw.get("dim_sigma", None)
    q.unit_centroids = kw.get("unit_c", None)
    q.unit_boundaries = kw.get("unit_t", None)
    return q


def _layout(lib, q):
    L = T.Layout_t()
    st = lib.tq_record_layout(C.byref(q), C.byref(L))
    return st, L


def test_record_layouts(lib):
    st, L = _layout(lib, _q(T.KIND_MSE, bits=4))
    assert st == 0 and (L.code_words, L.sign_words, L.has_norms, L.has_rnorms) == (16, 0, 1, 0)
    st, L = _layout(lib, _q(T.KIND_MSE, bits=3))
    assert st == 0 and L.code_words == 12
    st, L = _layout(lib, _q(T.KIND_PROD, bits=3, m=128, S=FAKE))
    assert st == 0 and (L.code_words, L.sign_words, L.has_norms, L.has_rnorms) == (8, 4, 1, 1)
    st, L = _layout(lib, _q(T.KIND_PROD, d=1536, bits=2, m=1536, S=FAKE))
    assert st == 0 and (L.code_words, L.sign_words) == (48, 48)
    st, L = _layout(lib, _q(T.KIND_SPECTRAL, k_top=4, top_bits=[5, 3, 2, 2], tail_bits=1, qjl=1, S=FAKE,
                             dim_sigma=FAKE, unit_c=FAKE, unit_t=FAKE))
    assert st == 0 and (L.code_words, L.has_norms, L.has_rnorms) == (5, 0, 1)
    st, L = _layout(lib, _q(T.KIND_SPECTRAL, k_top=4, top_bits=[5, 3, 2, 2], tail_bits=1, qjl=0,
                             dim_sigma=FAKE, unit_c=FAKE, unit_t=FAKE))
    assert st == 0 and (L.code_words, L.has_rnorms) == (5, 0)


@pytest.mark.parametrize("mut,code", [
    (lambda q: setattr(q, "d", 1), 1), (lambda q: setattr(q, "bits", 9), 1),
    (lambda q: setattr(q, "rot", None), 1), (lambda q: setattr(q, "rot", FAKE + 4), 3),
    (lambda q: setattr(q, "kind", 7), 1), (lambda q: setattr(q, "centroids", None), 1),
])
def test_descriptor_validation(lib, mut, code):
    q = _q(T.KIND_MSE, bits=3)
    mut(q)
    st, _ = _layout(lib, q)
    assert st == code
    assert lib.tq_last_error()


def test_quantize_validation_before_launch(lib):
    q = _q(T.KIND_MSE, bits=3)
    pk = T.Packed_t(FAKE + 0x100000, None, FAKE + 0x200000, None)
    # kind mismatch, unknown dtype, misaligned input, aliasing output, n == 0 (no launch)
    assert lib.tq_quantize_prod(C.byref(q), FAKE + 0x300000, 0, 10, pk, None) == 1
    assert lib.tq_quantize_mse(C.byref(q), FAKE + 0x300000, 9, 10, pk, None) == 1
    assert lib.tq_quantize_mse(C.byref(q), FAKE + 0x300002, 0, 10, pk, None) == 3
    assert lib.tq_quantize_mse(C.byref(q), FAKE + 0x100000, 0, 10, pk, None) == 4
    assert lib.tq_quantize_mse(C.byref(q), FAKE + 0x300000, 0, 0, pk, None) == 0
    assert lib.tq_quantize_mse(C.byref(q), None, 0, 10, pk, None) == 1
    bad = T.Packed_t(None, None, FAKE + 0x200000, None)
    assert lib.tq_quantize_mse(C.byref(q), FAKE + 0x300000, 0, 10, bad, None) == 1


def test_decode_validation_before_launch(lib):
    kq = _q(T.KIND_MSE, bits=4)
    vq = _q(T.KIND_MSE, bits=4)
    pk = T.Packed_t(FAKE + 0x100000, None, FAKE + 0x200000, None)
    pv = T.Packed_t(FAKE + 0x400000, None, FAKE + 0x500000, None)
    ws = C.c_size_t(0)
    assert lib.tq_decode_attn_workspace(C.byref(kq), 2, 8, 2, 1000, C.byref(ws)) == 0 and ws.value > 0
    args = (FAKE + 0x600000, 1, 2, 8, 2, 1000, FAKE + 0x700000, pk, pv, C.c_float(0.1), FAKE + 0x800000)
    # workspace too small
    assert lib.tq_decode_attn(C.byref(kq), C.byref(vq), *args, FAKE + 0x900000, 16, None) == 8
    # Hq not a multiple of Hkv
    a2 = list(args); a2[3] = 3
    assert lib.tq_decode_attn(C.byref(kq), C.byref(vq), *a2, FAKE + 0x900000, ws.value, None) == 1
    # head dim outside what the decode supports
    k64 = _q(T.KIND_MSE, d=64, bits=4); v64 = _q(T.KIND_MSE, d=64, bits=4)
    assert lib.tq_decode_attn(C.byref(k64), C.byref(v64), *args, FAKE + 0x900000, 1 << 30, None) == 2
    # output aliasing the query
    a3 = list(args); a3[-1] = FAKE + 0x600000
    assert lib.tq_decode_attn(C.byref(kq), C.byref(vq), *a3, FAKE + 0x900000, ws.value, None) == 4


def test_score_validation(lib):
    q = _q(T.KIND_MSE, bits=3)
    pk = T.Packed_t(FAKE + 0x100000, None, FAKE + 0x200000, None)
    ws = C.c_size_t(0)
    assert lib.tq_score_workspace(C.byref(q), 4, 100, 10, C.byref(ws)) == 0
    assert lib.tq_score(C.byref(q), FAKE + 0x300000, 0, 4, pk, 100, 40, FAKE + 0x400000, FAKE + 0x500000,
                        FAKE + 0x600000, ws.value, None) == 2   # topk > 32
    assert lib.tq_score(C.byref(q), FAKE + 0x300000, 0, 4, pk, 100, 10, FAKE + 0x400000, FAKE + 0x500000,
                        FAKE + 0x600000, 8, None) == 8          # workspace


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lut_scale_tightens_half_precision_codebook(lib, bits):
    c, _, _ = K.codebook_build(bits, "beta", d=128)
    s = T.lut_scale(c)
    assert 1.0 <= s < 2.0
    plain = np.max(np.abs(c.astype(np.float16).astype(np.float64) - c) / np.abs(c))
    scaled = np.max(np.abs((c / s).astype(np.float16).astype(np.float64) * s - c) / np.abs(c))
    assert scaled <= min(plain, 1.5e-4)


def _split(groups, cols, d):
    sp = T.Split_t()
    sp.n_groups, sp.d = len(groups), d
    for i, (q, c) in enumerate(zip(groups, cols)):
        sp.groups[i] = C.pointer(q)
        sp.cols[i] = c
    return sp


def test_split_validation_before_launch(lib):
    qa, qb = _q(T.KIND_MSE, d=32, bits=3), _q(T.KIND_MSE, d=96, bits=2)
    pks = (T.Packed_t * 2)(T.Packed_t(FAKE + 0x100000, None, FAKE + 0x200000, None),
                           T.Packed_t(FAKE + 0x400000, None, FAKE + 0x500000, None))
    x = FAKE + 0x700000
    ok = _split([qa, qb], [FAKE + 0x800000, FAKE + 0x810000], 128)
    assert lib.tq_quantize_split(C.byref(ok), x, 1, 0, pks, None) == 0            # n == 0: no launch
    # widths that do not add up to d
    assert lib.tq_quantize_split(C.byref(_split([qa, qb], [FAKE, FAKE], 127)), x, 1, 10, pks, None) == 1
    # a NULL or misaligned channel list
    assert lib.tq_quantize_split(C.byref(_split([qa, qb], [FAKE, None], 128)), x, 1, 10, pks, None) == 1
    assert lib.tq_quantize_split(C.byref(_split([qa, qb], [FAKE, FAKE + 2], 128)), x, 1, 10, pks, None) == 3
    # no groups, too many groups, a spectral group
    assert lib.tq_quantize_split(C.byref(_split([], [], 128)), x, 1, 10, pks, None) == 1
    sp = _split([qa, qb], [FAKE, FAKE], 128)
    sp.n_groups = T.MAX_GROUPS + 1
    assert lib.tq_quantize_split(C.byref(sp), x, 1, 10, pks, None) == 1
    qs = _q(T.KIND_SPECTRAL, d=96, k_top=4, top_bits=[5, 3, 2, 2], tail_bits=1, dim_sigma=FAKE, unit_c=FAKE,
            unit_t=FAKE)
    assert lib.tq_quantize_split(C.byref(_split([qa, qs], [FAKE, FAKE], 128)), x, 1, 10, pks, None) == 2
    # two groups writing into overlapping records
    same = (T.Packed_t * 2)(pks[0], pks[0])
    assert lib.tq_quantize_split(C.byref(ok), x, 1, 10, same, None) == 4
    # score: workspace query, then a too-small workspace
    ws = C.c_size_t(0)
    assert lib.tq_score_split_workspace(C.byref(ok), 4, 1000, 10, C.byref(ws)) == 0 and ws.value > 4 * 128 * 4
    assert lib.tq_score_split(C.byref(ok), FAKE + 0x900000, 0, 4, pks, 1000, 10, FAKE + 0xA00000,
                              FAKE + 0xB00000, FAKE + 0xC00000, 16, None) == 8


def test_split_decode_validation_before_launch(lib):
    qa, qb = _q(T.KIND_MSE, d=32, bits=3), _q(T.KIND_MSE, d=96, bits=2)
    sp = _split([qa, qb], [FAKE + 0x800000, FAKE + 0x810000], 128)
    ws = C.c_size_t(0)
    assert lib.tq_decode_attn_split_workspace(C.byref(sp), C.byref(sp), 2, 8, 2, 1000, C.byref(ws)) == 0
    assert ws.value >= 2 * 8 * 128 * 4                               # at least the rotated queries
    # GQA group too large, Hq not a multiple of Hkv, a prod value group (prod key groups
    # are taken), mismatched widths
    assert lib.tq_decode_attn_split_workspace(C.byref(sp), C.byref(sp), 1, 16, 1, 1000, C.byref(ws)) == 2
    assert lib.tq_decode_attn_split_workspace(C.byref(sp), C.byref(sp), 1, 6, 4, 1000, C.byref(ws)) == 1
    qp = _q(T.KIND_PROD, d=96, bits=3, m=96, S=FAKE)
    spp = _split([qa, qp], [FAKE, FAKE], 128)
    assert lib.tq_decode_attn_split_workspace(C.byref(spp), C.byref(sp), 1, 8, 1, 1000, C.byref(ws)) == 0
    assert lib.tq_decode_attn_split_workspace(C.byref(sp), C.byref(spp), 1, 8, 1, 1000, C.byref(ws)) == 2
    q64 = _q(T.KIND_MSE, d=64, bits=2)
    sp96 = _split([qa, q64], [FAKE, FAKE], 96)
    assert lib.tq_decode_attn_split_workspace(C.byref(sp), C.byref(sp96), 1, 8, 1, 1000, C.byref(ws)) == 1
    # wider than the split decode supports
    big = _split([_q(T.KIND_MSE, d=200, bits=2), _q(T.KIND_MSE, d=100, bits=2)], [FAKE, FAKE], 300)
    assert lib.tq_decode_attn_split_workspace(C.byref(big), C.byref(big), 1, 8, 1, 1000, C.byref(ws)) == 2
    # a workspace that is too small fails before any launch
    pk = (T.Packed_t * 2)(T.Packed_t(FAKE + 0x100000, None, FAKE + 0x200000, None),
                          T.Packed_t(FAKE + 0x300000, None, FAKE + 0x400000, None))
    pv = (T.Packed_t * 2)(T.Packed_t(FAKE + 0x500000, None, FAKE + 0x600000, None),
                          T.Packed_t(FAKE + 0x700000, None, FAKE + 0x780000, None))
    assert lib.tq_decode_attn_split(C.byref(sp), C.byref(sp), FAKE + 0x900000, 1, 2, 8, 2, 1000, FAKE + 0xA00000,
                                    pk, pv, C.c_float(0.1), FAKE + 0xB00000, FAKE + 0xC00000, 16, None) == 8


def test_wait_limit_values(lib):
    """0 restores the default, -1 is the expire-at-once test hook, below -1 is refused."""
    assert lib.tq_set_wait_limit(-1) == 0
    assert lib.tq_set_wait_limit(-2) == 1            # TQ_ERR_INVALID_ARG
    assert lib.tq_set_wait_limit(0) == 0


def test_spectral_descriptor_matches_oracle(lib):
    """tq_spectral_descriptor: water-filled bits, per-dim scales and codebooks as the oracle's
    build_descriptor computes them from the same eigen-decomposition."""
    d, n = 128, 4096
    U = ti.haar_rotation(d, 3004).astype(np.float64)
    X = ti.anisotropic(n, d, U, 7000).astype(np.float32)
    vo, wo = OSP.calibrate(X.astype(np.float64))
    desc = OSP.build_descriptor(vo, wo, 4, 12, 1, True)
    rot = np.zeros((d, d), np.float32)
    sig = np.zeros(d, np.float32)
    uc = np.zeros(510, np.float32)
    ut = np.zeros(502, np.float32)
    top = np.zeros(8, np.int32)
    lut = C.c_float(0)
    dp = C.POINTER(C.c_double)
    st = lib.tq_spectral_descriptor(vo.ctypes.data_as(dp), wo.ctypes.data_as(dp), d, 4, 12, 1, 8, rot.ctypes.data,
                                    sig.ctypes.data, uc.ctypes.data, ut.ctypes.data,
                                    top.ctypes.data_as(C.POINTER(C.c_int32)), C.byref(lut))
    assert st == 0
    assert list(top[:4]) == list(desc["bits"][:4]) == [5, 3, 2, 2]
    assert np.allclose(sig, desc["sigma"], rtol=1e-7, atol=0)
    assert np.array_equal(rot, vo.astype(np.float32))
    for b in range(1, 7):
        co, to, _ = lloyd_max(b, "gaussian", sigma=1.0)
        off_c, off_t = (1 << b) - 2, (1 << b) - b - 1
        assert np.allclose(uc[off_c:off_c + (1 << b)], co, rtol=1e-6, atol=1e-7)
        assert np.allclose(ut[off_t:off_t + (1 << b) - 1], to, rtol=1e-6, atol=1e-7)
    assert 1.0 <= lut.value < 2.0
    # a negative sample eigenvalue is a zero variance: scale 0, no bits from water-filling
    w2 = wo.copy()
    w2[2] = -1e-3
    st = lib.tq_spectral_descriptor(vo.ctypes.data_as(dp), w2.ctypes.data_as(dp), d, 4, 12, 1, 8, rot.ctypes.data,
                                    sig.ctypes.data, uc.ctypes.data, ut.ctypes.data,
                                    top.ctypes.data_as(C.POINTER(C.c_int32)), C.byref(lut))
    assert st == 0 and sig[2] == 0.0 and top[2] == 0
    # top bits plus sign bits must fit one head word
    st = lib.tq_spectral_descriptor(vo.ctypes.data_as(dp), wo.ctypes.data_as(dp), d, 8, 40, 1, 8, rot.ctypes.data,
                                    sig.ctypes.data, uc.ctypes.data, ut.ctypes.data,
                                    top.ctypes.data_as(C.POINTER(C.c_int32)), C.byref(lut))
    assert st == 2


def test_spectral_prepare_is_calibrate_then_descriptor(lib):
    d, n = 128, 4096
    U = ti.haar_rotation(d, 3004).astype(np.float64)
    X = ti.anisotropic(n, d, U, 7000).astype(np.float32)
    vecs, vals = K.spectral_calibrate(X)
    rot = np.zeros((d, d), np.float32)
    sig = np.zeros(d, np.float32)
    uc = np.zeros(510, np.float32)
    ut = np.zeros(502, np.float32)
    top = np.zeros(8, np.int32)
    lut = C.c_float(0)
    ev = np.zeros(d)
    st = lib.tq_spectral_prepare(X.ctypes.data, n, d, 4, 12, 1, 8, rot.ctypes.data, sig.ctypes.data, uc.ctypes.data,
                                 ut.ctypes.data, top.ctypes.data_as(C.POINTER(C.c_int32)), C.byref(lut),
                                 ev.ctypes.data_as(C.POINTER(C.c_double)))
    assert st == 0
    assert np.array_equal(ev, vals) and np.array_equal(rot, vecs.astype(np.float32))
    assert np.array_equal(sig, np.sqrt(np.maximum(vals, 0)).astype(np.float32))
    assert list(top[:4]) == list(K.waterfill(vals[:4], 12))
