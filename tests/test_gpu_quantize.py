"""GPU parity: quantize / dequantize through the C ABI against the oracle."""
import functools
import math

import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as OQ
from oracle import spectral as OSP
from oracle.codebook import lloyd_max as _lloyd_max

from _parity import adopt_spectral, as_u32, code_mismatches, sign_mismatches

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")


@functools.lru_cache(maxsize=None)
def lloyd_max(bits, dist, d=None):
    return _lloyd_max(bits, dist, d=d)


def _inputs(n, d, dtype, seed, zero_rows=()):
    x = ti.anisotropic(n, d, ti.haar_rotation(d, seed + 1).astype(np.float64), seed, lam=None) \
        if d == 128 else ti.iid_normal((n, d), seed) * 2.0
    for r in zero_rows:
        x[r] = 0.0
    if dtype == "bf16":
        xt, x64 = ti.to_bf16_f64(x)
    elif dtype == "f16":
        xt = torch.from_numpy(x.astype(np.float16))
        x64 = xt.to(torch.float64).numpy()
    else:
        xt = torch.from_numpy(x.astype(np.float32))
        x64 = xt.to(torch.float64).numpy()
    return xt.cuda().contiguous(), x64


MSE_CASES = [
    # d, bits, dtype, n   (d=128 16-bit input, bits <= 4 runs the tensor-core kernel)
    (128, 3, "f32", 4096),
    (128, 4, "bf16", 1000),
    (128, 4, "bf16", 128 * 148 * 2 + 37),
    (128, 1, "bf16", 5000),
    (128, 2, "bf16", 5000),
    (128, 3, "bf16", 5000),
    (128, 4, "f16", 3000),
    (128, 4, "bf16", 1),
    (8, 2, "f32", 777),
    (32, 5, "f32", 300),
    (96, 6, "bf16", 100),
    (1536, 4, "bf16", 64),
    (64, 7, "f32", 200),          # the top of the ABI's MSE range (CUDA-core kernel)
    (64, 8, "bf16", 150),
]


@pytest.mark.parametrize("d,bits,dtype,n", MSE_CASES)
def test_quantize_mse_parity(d, bits, dtype, n):
    rot = ti.haar_rotation(d, 1000 + d)
    x, x64 = _inputs(n, d, dtype, 4000 + d + bits, zero_rows=[0] if n > 10 else [])
    q = K.Quantizer.mse(rot, bits)
    out = K.quantize(q, x)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    c, t, _ = lloyd_max(bits, "beta", d=d)
    ref = OQ.quantize_mse(x64, rot, c, t, bits)
    zero = [0] if n > 10 else []
    bad, exempt, _ = code_mismatches(as_u32(out.codes), ref["codes"], d, bits, ref["y"], t, skip_rows=zero)
    assert bad == 0, f"{bad} code mismatches outside the band ({exempt} exempt)"
    assert exempt <= max(2, 1e-4 * n * d)
    # a zero vector has u = 0: every coordinate sits on the middle boundary t = 0 and
    # takes the lower cell, code 2^(b-1) - 1
    from oracle.quantizer import unpack_codes
    for r in zero:
        assert np.all(unpack_codes(as_u32(out.codes)[r:r + 1], d, bits) == (1 << (bits - 1)) - 1)
    nrm = out.norms.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(nrm - ref["norms"]) <= 1e-5 * np.maximum(ref["norms"], 1e-30))
    # reconstruction from the GPU's own records matches the oracle's (records without exemptions)
    xh = K.dequantize(q, out, n).cpu().numpy().astype(np.float64)
    xr = OQ.dequantize_mse(ref["idx"], ref["norms"], rot, c)
    same = np.all(as_u32(out.codes) == ref["codes"], axis=1)
    err = np.max(np.abs(xh[same] - xr[same]), axis=1) / np.maximum(ref["norms"][same], 1e-30)
    assert np.all(err < 1e-5)


@pytest.mark.parametrize("bits,dtype,n", [(4, "bf16", 128 * 148 + 77), (3, "bf16", 3000), (2, "f16", 2000),
                                           (1, "bf16", 1000), (4, "f32", 700)])
def test_quantize_mse_hadamard_parity(bits, dtype, n):
    """Randomized Hadamard rotation (entries +-1/sqrt(d)): the tensor-core kernel multiplies by
    the exact +-1 matrix; the oracle uses the dense rotation as given."""
    d = 128
    rot = ti.hadamard_rotation(d, 1500 + bits)
    x, x64 = _inputs(n, d, dtype, 4500 + bits, zero_rows=[0])
    q = K.Quantizer.mse(rot, bits)
    assert q.c.rot_pm1 == 1
    out = K.quantize(q, x)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    c, t, _ = lloyd_max(bits, "beta", d=d)
    ref = OQ.quantize_mse(x64, rot, c, t, bits)
    bad, exempt, _ = code_mismatches(as_u32(out.codes), ref["codes"], d, bits, ref["y"], t, skip_rows=[0])
    assert bad == 0, f"{bad} code mismatches outside the band ({exempt} exempt)"
    from oracle.quantizer import unpack_codes
    assert np.all(unpack_codes(as_u32(out.codes)[0:1], d, bits) == (1 << (bits - 1)) - 1)
    nrm = out.norms.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(nrm - ref["norms"]) <= 1e-5 * np.maximum(ref["norms"], 1e-30))


def test_quantize_pm1_flag_rejects_other_rotations():
    """rot_pm1 with a rotation whose entries are not +-1/sqrt(d) is reported, not trusted."""
    d = 128
    rot = ti.haar_rotation(d, 1502)
    x, _ = _inputs(256, d, "bf16", 4600)
    q = K.Quantizer.mse(rot, 4)
    q.c.rot_pm1 = 1
    K.quantize(q, x)
    torch.cuda.synchronize()
    assert K.get_status() == 1          # TQ_ERR_INVALID_ARG
    assert K.get_status() == 0          # reading the status clears it


@pytest.mark.parametrize("d,bits,m,dtype,n", [(128, 3, 128, "bf16", 2000), (64, 2, 64, "f32", 500),
                                              (128, 1, 128, "f32", 300), (128, 5, 256, "bf16", 400),
                                              (64, 6, 64, "f32", 200), (64, 7, 64, "bf16", 200),
                                              (64, 8, 96, "f32", 150), (64, 9, 64, "bf16", 150),
                                              # d = m = 128 with 16-bit input: the tensor-core kernel
                                              # (rotation and QJL projection on tcgen05), ragged tiles
                                              (128, 2, 128, "bf16", 128 * 148 + 5), (128, 4, 128, "f16", 3001),
                                              (128, 5, 128, "bf16", 1000), (128, 3, 128, "f16", 1)])
def test_quantize_prod_parity(d, bits, m, dtype, n):
    rot = ti.haar_rotation(d, 1100 + d)
    S = ti.gaussian_matrix(m, d, 2000 + d)
    x, x64 = _inputs(n, d, dtype, 4100 + d + bits)
    q = K.Quantizer.prod(rot, S, bits)
    out = K.quantize(q, x)
    if bits > 1:
        c, t, _ = lloyd_max(bits - 1, "beta", d=d)
    else:
        c = t = None
    ref = OQ.quantize_prod(x64, rot, S, c, t, bits)
    skip = set()
    if bits > 1:
        bad, exempt, skip = code_mismatches(as_u32(out.codes), ref["codes"], d, bits - 1, ref["y"], t)
        assert bad == 0
    sbad, sex = sign_mismatches(as_u32(out.signs), ref["signs"], m, ref["proj"], S, skip)
    assert sbad == 0, f"{sbad} sign mismatches outside the band"
    assert sex <= max(3, 2e-3 * n)
    rn = out.rnorms.cpu().numpy().astype(np.float64)
    ok = np.array([i not in skip for i in range(n)])
    assert np.all(np.abs(rn[ok] - ref["rnorms"][ok]) <= 1e-5 * np.maximum(ref["rnorms"][ok], 1e-6) + 1e-6)
    nrm = out.norms.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(nrm - ref["norms"]) <= 1e-5 * ref["norms"])
    xh = K.dequantize(q, out, n).cpu().numpy().astype(np.float64)
    xr = OQ.dequantize_prod(ref["chat"], ref["s"], ref["norms"], ref["rnorms"], rot, S)
    same = np.all(as_u32(out.signs) == ref["signs"], axis=1) & ok
    err = np.max(np.abs(xh[same] - xr[same]), axis=1) / ref["norms"][same]
    assert np.all(err < 1e-4)


def _spectral_desc(qjl, d=128):
    """Quantizer inputs: the generator's own basis and spectrum stand in for a calibration."""
    U = ti.haar_rotation(d, 3004).astype(np.float64)
    lam = d * ti.kv_spectrum(d)
    S4 = ti.gaussian_matrix(4, 4, 2004)
    rot = U.T.astype(np.float32)                     # row j = eigenvector j
    desc = OSP.build_descriptor(rot.astype(np.float64), lam, 4, 12, 1, qjl, S4)
    return U, rot, lam, S4, desc


@pytest.mark.parametrize("qjl", [True, False])
def test_quantize_spectral_parity(qjl):
    d, n = 128, 3000
    U, rot, lam, S4, desc = _spectral_desc(qjl)
    xt, x64 = ti.to_bf16_f64(ti.anisotropic(n, d, U, 4004))
    q = K.Quantizer.spectral(rot, lam, 4, 12, 1, qjl, S4 if qjl else None)
    assert list(q.top_bits) == list(desc["bits"][:4])      # the library's water-filling
    out = K.quantize(q, xt.cuda())
    ref = OSP.quantize_spectral(x64, desc)
    # coordinate by coordinate: a differing code must be a neighbour with the oracle's z_j
    # within 1e-5 ||x|| of the boundary between them; a differing QJL sign must have its
    # projection (recomputed from the adopted top codes) within the band; gamma to 1e-5 ||x||
    a = adopt_spectral(as_u32(out.codes), out.rnorms.cpu().numpy() if qjl else None, ref, desc, x64)
    assert a["exempt"] <= max(3, 1e-4 * n * d)
    # reconstruction from the GPU's records equals the oracle's on the adopted codes
    xh = K.dequantize(q, out, n).cpu().numpy()
    xr = OSP.dequantize_spectral(a["chat"], desc)
    assert np.max(np.abs(xh - xr)) < 1e-4 * np.max(np.abs(xr))


@pytest.mark.parametrize("d,kind,bits,n", [(1536, "prod", 2, 3000), (1536, "prod", 4, 1000), (256, "prod", 3, 777),
                                           (1536, "mse", 3, 500), (512, "mse", 1, 129), (256, "prod", 5, 1),
                                           (128, "mse", 3, 4096), (384, "prod", 3, 300), (128, "prod", 2, 257)])
def test_quantize_wide_tensor_core_parity(d, kind, bits, n):
    """tq_quantize_ws on fp32 vectors with d a multiple of 128: the rotation and the QJL
    projection as split-precision tensor-core products; records band-checked against the
    oracle (codes and signs), norms and residual norms to 1e-5."""
    from _parity import adopt_mse, adopt_prod
    rot = ti.haar_rotation(d, 1200 + d)
    S = ti.gaussian_matrix(d, d, 2200 + d)
    x = ti.unit_gaussian(n, d, 4200 + d + bits) * 3.0
    if n > 5:
        x[3] = 0.0                                  # a zero vector
    xt = torch.from_numpy(x.astype(np.float32)).cuda()
    x64 = xt.double().cpu().numpy()
    q = K.Quantizer.prod(rot, S, bits) if kind == "prod" else K.Quantizer.mse(rot, bits)
    out = K.quantize_ws(q, xt)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    nrm = out.norms.cpu().numpy().astype(np.float64)
    ref_n = np.linalg.norm(x64, axis=1)
    assert np.all(np.abs(nrm - ref_n) <= 1e-5 * np.maximum(ref_n, 1e-30))
    skip = [3] if n > 5 else []
    if kind == "mse":
        c, t, _ = lloyd_max(bits, "beta", d=d)
        ref = OQ.quantize_mse(x64, rot, c, t, bits)
        if skip:
            ref["codes"][3] = as_u32(out.codes)[3]   # the zero row: checked below
        adopt_mse(as_u32(out.codes), ref, bits, t)
    else:
        c, t, _ = lloyd_max(bits - 1, "beta", d=d)
        ref = OQ.quantize_prod(x64, rot, S, c, t, bits)
        keep = np.ones(n, dtype=bool)
        keep[skip] = False
        sub = {k: (v[keep] if isinstance(v, np.ndarray) and v.shape[:1] == (n,) else v) for k, v in ref.items()}
        a = adopt_prod(as_u32(out.codes)[keep], as_u32(out.signs)[keep], out.rnorms.cpu().numpy()[keep], sub, bits,
                       c, t, S)
        assert a["idx"].shape == (keep.sum(), d)
    from oracle.quantizer import unpack_codes
    bm = bits - 1 if kind == "prod" else bits
    for r in skip:                                   # u = 0: every code is the middle one
        assert np.all(unpack_codes(as_u32(out.codes)[r:r + 1], d, bm) == (1 << (bm - 1)) - 1)


def test_quantize_ws_matches_plain_call_elsewhere():
    """Shapes outside the wide path: tq_quantize_ws writes the records tq_quantize_* writes."""
    d, n = 128, 1000
    rot = ti.haar_rotation(d, 1301)
    xt = torch.from_numpy(ti.iid_normal((n, d), 4301).astype(np.float32)).to(torch.bfloat16).cuda()
    q = K.Quantizer.mse(rot, 4)
    a, b = K.quantize(q, xt), K.quantize_ws(q, xt)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes) and torch.equal(a.norms, b.norms)
