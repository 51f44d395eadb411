"""GPU parity at the full 32k-context prod workload (B=1, Hkv=8, Hq=32, d=128, context
32768; TurboQuant-prod b=3 keys with m=128 QJL rows, TurboQuant-mse b=3 values), in the
launch configuration bench.py times (``--workload c2``).

Sampled: for two (batch, kv-head) groups the GPU's own records (quantized at full size)
are band-checked against the oracle's quantization of the same rows, the oracle rescores
with them, and the decode output of those groups' query heads must agree to 1e-3 per
row.  A spread of rows over the whole cache is checked the same way; every other output
row must be finite.
"""
import math

import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as OQ
from oracle.attention import decode_attention
from oracle.codebook import lloyd_max

from _parity import adopt_mse, adopt_prod, as_u32, rel_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")

B, HKV, HQ, N, D = 1, 8, 32, 32768, 128
G = HQ // HKV
CFG = 2


@pytest.fixture(scope="module")
def workload():
    dev = torch.device("cuda")
    rot = ti.haar_rotation(D, ti.SEEDS["rotation"] + CFG)
    S = ti.gaussian_matrix(D, D, ti.SEEDS["qjl"] + CFG)
    U = ti.haar_rotation(D, ti.SEEDS["basis"] + CFG)
    kq = K.Quantizer.prod(rot, S, 3, device=dev)
    vq = K.Quantizer.mse(rot, 3, device=dev)
    n = B * HKV * N
    kx = ti.anisotropic_torch(n, D, U, ti.SEEDS["keys"] + CFG, dev)
    vx = ti.anisotropic_torch(n, D, U, ti.SEEDS["values"] + CFG, dev)
    q = ti.normal_torch((B, HQ, D), ti.SEEDS["queries"] + CFG, dev, dtype=torch.bfloat16)
    kc, vc = K.quantize(kq, kx), K.quantize(vq, vx)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    ck, tk, _ = lloyd_max(2, "beta", d=D)
    cv, tv, _ = lloyd_max(3, "beta", d=D)
    yield dict(rot=rot, S=S, kq=kq, vq=vq, kx=kx, vx=vx, q=q, kc=kc, vc=vc, ck=ck, tk=tk, cv=cv, tv=tv)


def _take(t, sel):
    return t[sel].cpu().numpy()


def test_prod32k_quantize_sampled_rows(workload):
    w = workload
    n = B * HKV * N
    rng = np.random.Generator(np.random.PCG64(21))
    rows = np.unique(np.concatenate([rng.integers(0, n, 4000), [0, 1, 31, 32, n - 33, n - 1]]))
    idx = torch.from_numpy(rows).cuda()
    ref = OQ.quantize_prod(w["kx"].index_select(0, idx).double().cpu().numpy(), w["rot"], w["S"], w["ck"], w["tk"], 3)
    kc = w["kc"]
    a = adopt_prod(as_u32(kc.codes.index_select(0, idx)), as_u32(kc.signs.index_select(0, idx)),
                   kc.rnorms.index_select(0, idx).cpu().numpy(), ref, 3, w["ck"], w["tk"], w["S"])
    assert a["idx"].shape == (rows.size, D)
    nrm = kc.norms.index_select(0, idx).cpu().numpy()
    assert np.max(np.abs(nrm - ref["norms"]) / ref["norms"]) < 1e-5


def test_prod32k_decode_sampled_groups(workload):
    w = workload
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    out = K.decode_attn(w["kq"], w["vq"], w["q"], sl, w["kc"], w["vc"], N, HKV)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    o = out.cpu().numpy()
    assert np.all(np.isfinite(o))
    for b, h in [(0, 1), (0, 6)]:
        sel = slice((b * HKV + h) * N, (b * HKV + h + 1) * N)
        ok = OQ.quantize_prod(w["kx"][sel].double().cpu().numpy(), w["rot"], w["S"], w["ck"], w["tk"], 3)
        ov = OQ.quantize_mse(w["vx"][sel].double().cpu().numpy(), w["rot"], w["cv"], w["tv"], 3)
        kc, vc = w["kc"], w["vc"]
        a = adopt_prod(as_u32(kc.codes[sel]), as_u32(kc.signs[sel]), _take(kc.rnorms, sel), ok, 3,
                       w["ck"], w["tk"], w["S"])
        vidx, _ = adopt_mse(as_u32(vc.codes[sel]), ov, 3, w["tv"])
        vh = OQ.dequantize_mse(vidx, ov["norms"], w["rot"], w["cv"])
        q64 = w["q"][b:b + 1, h * G:(h + 1) * G].double().cpu().numpy()
        ref = decode_attention(
            q64, [N], 1,
            lambda bb, hh, qs: OQ.estimate_prod(qs, w["rot"], w["S"], a["chat"], a["s"], ok["norms"], a["rnorms"]),
            lambda bb, hh, nn: vh[:nn], 1.0 / math.sqrt(D))[0]
        err = rel_rows(o[b, h * G:(h + 1) * G], ref)
        assert np.all(err <= 1e-3), f"group {(b, h)}: max row error {err.max():.3e}"
