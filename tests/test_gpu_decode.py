"""GPU parity: decode attention straight from the packed cache vs the oracle."""
import math

import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as OQ
from oracle import spectral as OSP
from oracle.attention import decode_attention
from oracle.codebook import lloyd_max

from _parity import rel_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")

D = 128


def _cache_inputs(B, Hkv, Nmax, seed):
    U = ti.haar_rotation(D, 3000 + seed).astype(np.float64)
    kx = ti.anisotropic(B * Hkv * Nmax, D, U, 4000 + seed)
    vx = ti.anisotropic(B * Hkv * Nmax, D, U, 5000 + seed)
    kt, k64 = ti.to_bf16_f64(kx)
    vt, v64 = ti.to_bf16_f64(vx)
    return kt.cuda(), k64, vt.cuda(), v64


def _query(B, Hq, seed, dtype="bf16"):
    q = ti.iid_normal((B * Hq, D), 6000 + seed)
    if dtype == "bf16":
        qt, q64 = ti.to_bf16_f64(q)
    else:
        qt = torch.from_numpy(q.astype(np.float32))
        q64 = qt.double().numpy()
    return qt.reshape(B, Hq, D).cuda(), q64.reshape(B, Hq, D)


def _rows(B, Hkv, Nmax, b, h, n):
    base = (b * Hkv + h) * Nmax
    return slice(base, base + n)


DECODE_CASES = [
    # name, B, Hq, Hkv, Nmax, seq_lens, kind_k, bits_k, bits_v
    ("c3-small", 2, 8, 2, 3000, [3000, 1777], "mse", 4, 4),
    ("c2-small", 1, 32, 8, 1100, [1100], "prod", 3, 3),
    ("g1", 1, 2, 2, 700, [513], "mse", 4, 4),
    ("g16", 1, 32, 2, 900, [900], "mse", 3, 2),
    ("one-token", 3, 8, 2, 64, [1, 2, 64], "mse", 4, 4),
    ("bits1", 1, 8, 2, 1000, [999], "mse", 1, 1),
    ("bits2-4", 2, 8, 2, 800, [800, 17], "mse", 2, 4),
    ("prod2", 1, 8, 2, 1500, [1500], "prod", 2, 4),
    ("prod5", 1, 8, 2, 600, [600], "prod", 5, 3),
]


@pytest.mark.parametrize("name,B,Hq,Hkv,Nmax,seq_lens,kk,bk,bv", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_attention_parity(name, B, Hq, Hkv, Nmax, seq_lens, kk, bk, bv):
    seed = sum(ord(ch) for ch in name) % 97
    rot = ti.haar_rotation(D, 1002)
    S = ti.gaussian_matrix(D, D, 2002)
    kt, k64, vt, v64 = _cache_inputs(B, Hkv, Nmax, seed)
    qt, q64 = _query(B, Hq, seed)
    kq = K.Quantizer.prod(rot, S, bk) if kk == "prod" else K.Quantizer.mse(rot, bk)
    vq = K.Quantizer.mse(rot, bv)
    kc = K.quantize(kq, kt)
    vc = K.quantize(vq, vt)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    out = K.decode_attn(kq, vq, qt, sl, kc, vc, Nmax, Hkv).cpu().numpy()
    assert K.get_status() == 0

    cv, tv, _ = lloyd_max(bv, "beta", d=D)
    if kk == "prod":
        ck, tk, _ = lloyd_max(bk - 1, "beta", d=D)
    else:
        ck, tk, _ = lloyd_max(bk, "beta", d=D)
    cache = {}

    def kscores(b, h, qs):
        r = _rows(B, Hkv, Nmax, b, h, Nmax)
        if ("k", b, h) not in cache:
            cache[("k", b, h)] = OQ.quantize_prod(k64[r], rot, S, ck, tk, bk) if kk == "prod" else \
                OQ.quantize_mse(k64[r], rot, ck, tk, bk)
        o = cache[("k", b, h)]
        if kk == "prod":
            return OQ.estimate_prod(qs, rot, S, o["chat"], o["s"], o["norms"], o["rnorms"])
        return OQ.estimate_mse(qs, rot, o["idx"], o["norms"], ck)

    def vrows(b, h, n):
        r = _rows(B, Hkv, Nmax, b, h, Nmax)
        o = OQ.quantize_mse(v64[r], rot, cv, tv, bv)
        return OQ.dequantize_mse(o["idx"], o["norms"], rot, cv)[:n]

    ref = decode_attention(q64, seq_lens, Hkv, kscores, vrows, 1.0 / math.sqrt(D))
    err = rel_rows(out, ref)
    assert np.all(err <= 1e-3), f"max row error {err.max():.3e}"


def test_decode_spectral_parity():
    B, Hq, Hkv, Nmax, seq_lens = 2, 8, 2, 1500, [1500, 999]
    U = ti.haar_rotation(D, 3004).astype(np.float64)
    lam = D * ti.kv_spectrum(D)
    S4 = ti.gaussian_matrix(4, 4, 2004)
    rot = U.T.astype(np.float32)
    dk = OSP.build_descriptor(rot.astype(np.float64), lam, 4, 12, 1, True, S4)
    dv = OSP.build_descriptor(rot.astype(np.float64), lam, 4, 12, 1, False, None)
    kx = ti.anisotropic(B * Hkv * Nmax, D, U, 4004)
    vx = ti.anisotropic(B * Hkv * Nmax, D, U, 5004)
    kt, k64 = ti.to_bf16_f64(kx)
    vt, v64 = ti.to_bf16_f64(vx)
    qt, q64 = _query(B, Hq, 4)
    top = list(dk["bits"][:4])
    kq = K.Quantizer.spectral(rot, lam, 4, top, 1, True, S4)
    vq = K.Quantizer.spectral(rot, lam, 4, top, 1, False, None)
    kc = K.quantize(kq, kt.cuda())
    vc = K.quantize(vq, vt.cuda())
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    out = K.decode_attn(kq, vq, qt, sl, kc, vc, Nmax, Hkv).cpu().numpy()
    assert K.get_status() == 0

    def kscores(b, h, qs):
        o = OSP.quantize_spectral(k64[_rows(B, Hkv, Nmax, b, h, Nmax)], dk)
        return OSP.estimate_spectral(qs, dk, o["chat"], o["s"], o["rnorms"])

    def vrows(b, h, n):
        o = OSP.quantize_spectral(v64[_rows(B, Hkv, Nmax, b, h, Nmax)], dv)
        return OSP.dequantize_spectral(o["chat"], dv)[:n]

    ref = decode_attention(q64, seq_lens, Hkv, kscores, vrows, 1.0 / math.sqrt(D))
    err = rel_rows(out, ref)
    assert np.all(err <= 1e-3), f"max row error {err.max():.3e}"


def test_decode_matches_score_logits():
    """Two GPU routes, one estimator: softmax of tq_score's estimates reproduces decode."""
    B, Hq, Hkv, Nmax = 1, 4, 1, 513
    rot = ti.haar_rotation(D, 1002)
    kt, _, vt, _ = _cache_inputs(B, Hkv, Nmax, 11)
    qt, _ = _query(B, Hq, 11, "f32")
    kq = K.Quantizer.mse(rot, 4)
    vq = K.Quantizer.mse(rot, 4)
    kc, vc = K.quantize(kq, kt), K.quantize(vq, vt)
    out = K.decode_attn(kq, vq, qt, torch.tensor([Nmax], dtype=torch.int32, device="cuda"), kc, vc, Nmax, Hkv)
    s = K.score(kq, qt.reshape(Hq, D).contiguous(), kc, Nmax)
    p = torch.softmax(s.double() / math.sqrt(D), dim=1)
    vh = K.dequantize(vq, vc, Nmax).double()
    ref = (p @ vh).cpu().numpy()
    err = rel_rows(out.cpu().numpy().reshape(Hq, D), ref)
    assert np.all(err <= 1e-3)
