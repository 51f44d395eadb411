"""GPU parity: decode attention straight from the packed cache vs the oracle."""
import math

import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as OQ
from oracle import spectral as OSP
from oracle.attention import decode_attention
from oracle.codebook import lloyd_max

from _parity import adopt_mse, adopt_prod, adopt_spectral, as_u32, rel_rows

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


def _dev_records(codes, norms=None, signs=None, rnorms=None):
    """Oracle-packed records as device tensors (the decode kernel then sees exactly the
    codes the oracle chose, so the comparison is free of boundary-band flips)."""
    t = lambda a, dt: None if a is None else torch.from_numpy(np.ascontiguousarray(a).astype(dt)).cuda()
    return K.Packed(t(np.asarray(codes, dtype=np.uint32).view(np.int32), np.int32), t(
        None if signs is None else np.asarray(signs, dtype=np.uint32).view(np.int32), np.int32),
        t(norms, np.float32), t(rnorms, np.float32))


def _rows(B, Hkv, Nmax, b, h, n):
    base = (b * Hkv + h) * Nmax
    return slice(base, base + n)


def _check_norms(packed, ref):
    nrm = packed.norms.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(nrm - ref["norms"]) <= 1e-5 * np.maximum(ref["norms"], 1e-30))


def _rescored_reference(q64, seq_lens, B, Hkv, Nmax, rot, S, kk, bk, bv, kc, vc, okq, ovq, ck, tk, cv, tv):
    """Oracle attention over the GPU-quantized cache: the GPU's codes and sign bits are
    band-checked against the oracle's, then the oracle scores with them (a legitimate flip
    inside the 1e-5 band is adopted instead of being allowed to move the output)."""
    _check_norms(kc, okq)
    _check_norms(vc, ovq)
    if kk == "prod":
        a = adopt_prod(as_u32(kc.codes) if bk > 1 else None, as_u32(kc.signs), kc.rnorms.cpu().numpy(),
                       okq, bk, ck, tk, S)

        def kscores(b, h, qs):
            r = _rows(B, Hkv, Nmax, b, h, Nmax)
            return OQ.estimate_prod(qs, rot, S, a["chat"][r], a["s"][r], okq["norms"][r], a["rnorms"][r])
    else:
        kidx, _ = adopt_mse(as_u32(kc.codes), okq, bk, tk)

        def kscores(b, h, qs):
            r = _rows(B, Hkv, Nmax, b, h, Nmax)
            return OQ.estimate_mse(qs, rot, kidx[r], okq["norms"][r], ck)
    vidx, _ = adopt_mse(as_u32(vc.codes), ovq, bv, tv)
    vh = OQ.dequantize_mse(vidx, ovq["norms"], rot, cv)
    return decode_attention(q64, seq_lens, Hkv, kscores, lambda b, h, n: vh[_rows(B, Hkv, Nmax, b, h, n)],
                            1.0 / math.sqrt(D))


DECODE_CASES = [
    # name, B, Hq, Hkv, Nmax, seq_lens, kind_k, bits_k, bits_v
    ("c3-small", 2, 8, 2, 3000, [3000, 1777], "mse", 4, 4),
    ("c2-small", 1, 32, 8, 1100, [1100], "prod", 3, 3),
    ("g1", 1, 2, 2, 700, [513], "mse", 4, 4),
    ("g16", 1, 32, 2, 900, [900], "mse", 3, 2),
    ("one-token", 3, 8, 2, 64, [1, 2, 64], "mse", 4, 4),
    ("bits1", 1, 8, 2, 1000, [999], "mse", 1, 1),
    ("bits1-g8", 1, 16, 2, 700, [700], "mse", 1, 1),
    ("bits4-1", 2, 8, 2, 900, [900, 451], "mse", 4, 1),
    ("bits1-3", 1, 8, 2, 800, [800], "mse", 1, 3),
    ("bits2-4", 2, 8, 2, 800, [800, 17], "mse", 2, 4),
    ("bits2", 1, 8, 2, 900, [900], "mse", 2, 2),
    ("bits2-g8", 2, 16, 2, 500, [500, 263], "mse", 2, 2),
    ("bits3-2-g8", 1, 16, 2, 600, [600], "mse", 3, 2),
    ("prod2", 1, 8, 2, 1500, [1500], "prod", 2, 4),
    ("prod5", 1, 8, 2, 600, [600], "prod", 5, 3),
]


@pytest.mark.parametrize("name,B,Hq,Hkv,Nmax,seq_lens,kk,bk,bv", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_attention_parity(name, B, Hq, Hkv, Nmax, seq_lens, kk, bk, bv):
    """Strict parity of the decode step on the oracle's own records (<= 1e-3 per row),
    then the full GPU path (GPU quantize -> GPU decode) on the same inputs."""
    seed = sum(ord(ch) for ch in name) % 97
    rot = ti.haar_rotation(D, 1002)
    S = ti.gaussian_matrix(D, D, 2002)
    kt, k64, vt, v64 = _cache_inputs(B, Hkv, Nmax, seed)
    qt, q64 = _query(B, Hq, seed)
    kq = K.Quantizer.prod(rot, S, bk) if kk == "prod" else K.Quantizer.mse(rot, bk)
    vq = K.Quantizer.mse(rot, bv)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")

    cv, tv, _ = lloyd_max(bv, "beta", d=D)
    ck, tk, _ = lloyd_max(bk - 1 if kk == "prod" else bk, "beta", d=D)
    okq = OQ.quantize_prod(k64, rot, S, ck, tk, bk) if kk == "prod" else OQ.quantize_mse(k64, rot, ck, tk, bk)
    ovq = OQ.quantize_mse(v64, rot, cv, tv, bv)
    vh = OQ.dequantize_mse(ovq["idx"], ovq["norms"], rot, cv)

    def kscores(b, h, qs):
        r = _rows(B, Hkv, Nmax, b, h, Nmax)
        if kk == "prod":
            return OQ.estimate_prod(qs, rot, S, okq["chat"][r], okq["s"][r], okq["norms"][r], okq["rnorms"][r])
        return OQ.estimate_mse(qs, rot, okq["idx"][r], okq["norms"][r], ck)

    ref = decode_attention(q64, seq_lens, Hkv, kscores,
                           lambda b, h, n: vh[_rows(B, Hkv, Nmax, b, h, n)], 1.0 / math.sqrt(D))

    kc_o = _dev_records(okq["codes"], okq["norms"], okq.get("signs"), okq.get("rnorms"))
    vc_o = _dev_records(ovq["codes"], ovq["norms"])
    out = K.decode_attn(kq, vq, qt, sl, kc_o, vc_o, Nmax, Hkv).cpu().numpy()
    assert K.get_status() == 0
    err = rel_rows(out, ref)
    assert np.all(err <= 1e-3), f"max row error {err.max():.3e}"

    # full GPU path (GPU quantize -> GPU decode): the oracle rescores with the GPU's
    # band-checked codes, and every row must again agree to 1e-3
    kc, vc = K.quantize(kq, kt), K.quantize(vq, vt)
    out2 = K.decode_attn(kq, vq, qt, sl, kc, vc, Nmax, Hkv).cpu().numpy()
    assert K.get_status() == 0
    ref2 = _rescored_reference(q64, seq_lens, B, Hkv, Nmax, rot, S, kk, bk, bv, kc, vc, okq, ovq, ck, tk, cv, tv)
    err2 = rel_rows(out2, ref2)
    assert np.all(err2 <= 1e-3), f"max row error {err2.max():.3e}"


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
    kq = K.Quantizer.spectral(rot, lam, 4, 12, 1, True, S4)
    vq = K.Quantizer.spectral(rot, lam, 4, 12, 1, False, None)
    assert list(kq.top_bits) == list(dk["bits"][:4]) == list(vq.top_bits)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    ok = OSP.quantize_spectral(k64, dk)
    ov = OSP.quantize_spectral(v64, dv)
    vh = OSP.dequantize_spectral(ov["chat"], dv)

    def kscores(b, h, qs):
        r = _rows(B, Hkv, Nmax, b, h, Nmax)
        return OSP.estimate_spectral(qs, dk, ok["chat"][r], ok["s"][r], ok["rnorms"][r])

    ref = decode_attention(q64, seq_lens, Hkv, kscores, lambda b, h, n: vh[_rows(B, Hkv, Nmax, b, h, n)],
                           1.0 / math.sqrt(D))
    out = K.decode_attn(kq, vq, qt, sl, _dev_records(ok["codes"], rnorms=ok["rnorms"]),
                        _dev_records(ov["codes"]), Nmax, Hkv).cpu().numpy()
    assert K.get_status() == 0
    err = rel_rows(out, ref)
    assert np.all(err <= 1e-3), f"max row error {err.max():.3e}"
    kc, vc = K.quantize(kq, kt.cuda()), K.quantize(vq, vt.cuda())
    out2 = K.decode_attn(kq, vq, qt, sl, kc, vc, Nmax, Hkv).cpu().numpy()
    assert K.get_status() == 0
    ak = adopt_spectral(as_u32(kc.codes), kc.rnorms.cpu().numpy(), ok, dk, k64)
    av = adopt_spectral(as_u32(vc.codes), None, ov, dv, v64)
    vh2 = OSP.dequantize_spectral(av["chat"], dv)

    def kscores2(b, h, qs):
        r = _rows(B, Hkv, Nmax, b, h, Nmax)
        return OSP.estimate_spectral(qs, dk, ak["chat"][r], ak["s"][r], ak["rnorms"][r])

    ref2 = decode_attention(q64, seq_lens, Hkv, kscores2, lambda b, h, n: vh2[_rows(B, Hkv, Nmax, b, h, n)],
                            1.0 / math.sqrt(D))
    err2 = rel_rows(out2, ref2)
    assert np.all(err2 <= 1e-3), f"max row error {err2.max():.3e}"


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


def test_decode_hadamard_rotation():
    """Keys and values quantized with a randomized Hadamard rotation (tensor-core +-1 path);
    decode reads them with the same dense rotation folded into the query and the output."""
    B, Hq, Hkv, Nmax, seq_lens = 2, 8, 2, 2000, [2000, 1234]
    rot = ti.hadamard_rotation(D, 1602)
    kt, k64, vt, v64 = _cache_inputs(B, Hkv, Nmax, 31)
    qt, q64 = _query(B, Hq, 31)
    kq, vq = K.Quantizer.mse(rot, 4), K.Quantizer.mse(rot, 4)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    c, t, _ = lloyd_max(4, "beta", d=D)
    okq = OQ.quantize_mse(k64, rot, c, t, 4)
    ovq = OQ.quantize_mse(v64, rot, c, t, 4)
    vh = OQ.dequantize_mse(ovq["idx"], ovq["norms"], rot, c)
    ref = decode_attention(q64, seq_lens, Hkv,
                           lambda b, h, qs: OQ.estimate_mse(qs, rot, okq["idx"][_rows(B, Hkv, Nmax, b, h, Nmax)],
                                                            okq["norms"][_rows(B, Hkv, Nmax, b, h, Nmax)], c),
                           lambda b, h, n: vh[_rows(B, Hkv, Nmax, b, h, n)], 1.0 / math.sqrt(D))
    out = K.decode_attn(kq, vq, qt, sl, _dev_records(okq["codes"], okq["norms"]),
                        _dev_records(ovq["codes"], ovq["norms"]), Nmax, Hkv).cpu().numpy()
    assert K.get_status() == 0
    err = rel_rows(out, ref)
    assert np.all(err <= 1e-3), f"max row error {err.max():.3e}"
    kc, vc = K.quantize(kq, kt), K.quantize(vq, vt)
    out2 = K.decode_attn(kq, vq, qt, sl, kc, vc, Nmax, Hkv).cpu().numpy()
    assert K.get_status() == 0
    ref2 = _rescored_reference(q64, seq_lens, B, Hkv, Nmax, rot, None, "mse", 4, 4, kc, vc, okq, ovq, c, t, c, t)
    err2 = rel_rows(out2, ref2)
    assert np.all(err2 <= 1e-3), f"max row error {err2.max():.3e}"


PROD_VALUE_CASES = [
    # name, B, Hq, Hkv, Nmax, seq_lens, key kind, key bits, value bits (values as prod)
    ("pv-mse4-prod3", 2, 8, 2, 1500, [1500, 733], "mse", 4, 3),
    ("pv-prod3-prod3", 1, 32, 8, 1100, [1100], "prod", 3, 3),
    ("pv-g8", 1, 8, 1, 900, [900], "mse", 3, 4),
    ("pv-g1-bits2", 2, 4, 4, 700, [1, 699], "mse", 2, 2),
    ("pv-prod5", 1, 8, 2, 600, [600], "prod", 4, 5),
]


@pytest.mark.parametrize("name,B,Hq,Hkv,Nmax,seq_lens,kk,bk,bv", PROD_VALUE_CASES, ids=[c[0] for c in PROD_VALUE_CASES])
def test_decode_prod_values(name, B, Hq, Hkv, Nmax, seq_lens, kk, bk, bv):
    """Values quantized as TurboQuant-prod: the step uses their unbiased reconstruction
    ||v|| Pi^T (c[code] + sqrt(pi/2)/m ||r|| S^T (2s - 1)).  GPU quantize -> GPU decode, the
    oracle rescoring with the GPU's band-checked key and value records, 1e-3 per row."""
    seed = sum(ord(ch) for ch in name) % 89
    rot = ti.haar_rotation(D, 1003)
    S = ti.gaussian_matrix(D, D, 2003)
    Sv = ti.gaussian_matrix(D, D, 2103)
    kt, k64, vt, v64 = _cache_inputs(B, Hkv, Nmax, seed)
    qt, q64 = _query(B, Hq, seed)
    kq = K.Quantizer.prod(rot, S, bk) if kk == "prod" else K.Quantizer.mse(rot, bk)
    vq = K.Quantizer.prod(rot, Sv, bv)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    kc, vc = K.quantize(kq, kt), K.quantize(vq, vt)
    out = K.decode_attn(kq, vq, qt, sl, kc, vc, Nmax, Hkv).cpu().numpy()
    assert K.get_status() == 0
    ck, tk, _ = lloyd_max(bk - 1 if kk == "prod" else bk, "beta", d=D)
    cv, tv, _ = lloyd_max(bv - 1, "beta", d=D)
    okq = OQ.quantize_prod(k64, rot, S, ck, tk, bk) if kk == "prod" else OQ.quantize_mse(k64, rot, ck, tk, bk)
    ovq = OQ.quantize_prod(v64, rot, Sv, cv, tv, bv)
    _check_norms(kc, okq)
    _check_norms(vc, ovq)
    if kk == "prod":
        a = adopt_prod(as_u32(kc.codes), as_u32(kc.signs), kc.rnorms.cpu().numpy(), okq, bk, ck, tk, S)
        ks = lambda r, qs: OQ.estimate_prod(qs, rot, S, a["chat"][r], a["s"][r], okq["norms"][r], a["rnorms"][r])
    else:
        kidx, _ = adopt_mse(as_u32(kc.codes), okq, bk, tk)
        ks = lambda r, qs: OQ.estimate_mse(qs, rot, kidx[r], okq["norms"][r], ck)
    av = adopt_prod(as_u32(vc.codes), as_u32(vc.signs), vc.rnorms.cpu().numpy(), ovq, bv, cv, tv, Sv)
    vh = OQ.dequantize_prod(av["chat"], av["s"], ovq["norms"], av["rnorms"], rot, Sv)
    ref = decode_attention(q64, seq_lens, Hkv, lambda b, h, qs: ks(_rows(B, Hkv, Nmax, b, h, Nmax), qs),
                           lambda b, h, n: vh[_rows(B, Hkv, Nmax, b, h, n)], 1.0 / math.sqrt(D))
    err = rel_rows(out, ref)
    assert np.all(err <= 1e-3), f"max row error {err.max():.3e}"
