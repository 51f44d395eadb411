"""GPU parity at the full 8k-context SpectralQuant workload (B=32, Hkv=8, Hq=32, d=128,
context 8192), in the launch configuration bench.py times (``--workload c4``), built from
library calls only: tq_spectral_prepare on 4096 calibration keys (and, separately, values)
gives the eigenvector rotation, the water-filled [5, 3, 2, 2] top bits with a 1-bit tail
and the per-dim scales; QJL on the top 4 dims of the keys.

The oracle runs its own chain on the same calibration rows (calibrate -> build_descriptor
-> quantize_spectral -> attention).  The two calibrations are compared first; then for
sampled (batch, kv-head) groups the GPU's records are band-checked coordinate by
coordinate against the oracle's, the oracle rescores with them, and the decode output of
those groups must agree to 1e-3 per row.
"""
import math

import numpy as np
import pytest

import tq_inputs as ti
from oracle import spectral as OSP
from oracle.attention import decode_attention

from _parity import adopt_spectral, as_u32, rel_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")

B, HKV, HQ, N, D = 32, 8, 32, 8192, 128
G = HQ // HKV
CFG = 4


@pytest.fixture(scope="module")
def workload():
    dev = torch.device("cuda")
    U = ti.haar_rotation(D, ti.SEEDS["basis"] + CFG)
    ck = ti.anisotropic(4096, D, U.astype(np.float64), ti.SEEDS["calib_keys"] + CFG).astype(np.float32)
    cv = ti.anisotropic(4096, D, U.astype(np.float64), ti.SEEDS["calib_values"] + CFG).astype(np.float32)
    S4 = ti.gaussian_matrix(4, 4, ti.SEEDS["qjl"] + CFG)
    kq, kval = K.Quantizer.spectral_calibrated(ck, 4, 12, 1, True, S4, device=dev)
    vq, vval = K.Quantizer.spectral_calibrated(cv, 4, 12, 1, False, None, device=dev)
    vk, wk = OSP.calibrate(ck.astype(np.float64))
    vv, wv = OSP.calibrate(cv.astype(np.float64))
    dk = OSP.build_descriptor(vk, wk, 4, 12, 1, True, S4)
    dv = OSP.build_descriptor(vv, wv, 4, 12, 1, False, None)
    n = B * HKV * N
    kx = ti.anisotropic_torch(n, D, U, ti.SEEDS["keys"] + CFG, dev)
    vx = ti.anisotropic_torch(n, D, U, ti.SEEDS["values"] + CFG, dev)
    q = ti.normal_torch((B, HQ, D), ti.SEEDS["queries"] + CFG, dev, dtype=torch.bfloat16)
    kc, vc = K.quantize(kq, kx), K.quantize(vq, vx)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    yield dict(kq=kq, vq=vq, kval=kval, vval=vval, dk=dk, dv=dv, wk=wk, wv=wv, vk=vk, vv=vv,
               kx=kx, vx=vx, q=q, kc=kc, vc=vc)


def test_spectral8k_calibration_and_descriptor(workload):
    """The library's calibration equals the oracle's (eigenvalues to 1e-9 of the largest,
    every eigenvector to 1e-8 after the sign rule) and gives the same bit split."""
    w = workload
    for q, val, vo, wo, desc in ((w["kq"], w["kval"], w["vk"], w["wk"], w["dk"]),
                                 (w["vq"], w["vval"], w["vv"], w["wv"], w["dv"])):
        assert np.max(np.abs(val - wo)) < 1e-9 * wo[0]
        rot = q.rot.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(rot - vo)) < 1e-6          # fp32 copy of the eigenvectors
        assert list(q.top_bits) == list(desc["bits"][:4]) == [5, 3, 2, 2]


def test_spectral8k_decode_sampled_groups(workload):
    w = workload
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    out = K.decode_attn(w["kq"], w["vq"], w["q"], sl, w["kc"], w["vc"], N, HKV)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    o = out.cpu().numpy()
    assert np.all(np.isfinite(o))
    for b, h in [(0, 0), (13, 5), (31, 7)]:
        sel = slice((b * HKV + h) * N, (b * HKV + h + 1) * N)
        k64 = w["kx"][sel].double().cpu().numpy()
        v64 = w["vx"][sel].double().cpu().numpy()
        ok = OSP.quantize_spectral(k64, w["dk"])
        ov = OSP.quantize_spectral(v64, w["dv"])
        ak = adopt_spectral(as_u32(w["kc"].codes[sel]), w["kc"].rnorms[sel].cpu().numpy(), ok, w["dk"], k64)
        av = adopt_spectral(as_u32(w["vc"].codes[sel]), None, ov, w["dv"], v64)
        assert ak["exempt"] + av["exempt"] <= max(4, 1e-5 * N * D)
        vh = OSP.dequantize_spectral(av["chat"], w["dv"])
        q64 = w["q"][b:b + 1, h * G:(h + 1) * G].double().cpu().numpy()
        ref = decode_attention(
            q64, [N], 1, lambda bb, hh, qs: OSP.estimate_spectral(qs, w["dk"], ak["chat"], ak["s"], ak["rnorms"]),
            lambda bb, hh, nn: vh[:nn], 1.0 / math.sqrt(D))[0]
        err = rel_rows(o[b, h * G:(h + 1) * G], ref)
        assert np.all(err <= 1e-3), f"group {(b, h)}: max row error {err.max():.3e}"
