"""GPU parity at the full 128k-context decode workload (B=8, Hkv=8, Hq=32, d=128,
context 131072, mse b=4 keys and values), in the launch configuration bench.py times.

The oracle cannot process 8.4 M vectors, so the comparison is on samples:
  * quantize: 4096 rows spread over the whole K array (tile boundaries, the last row)
    against the oracle's quantization of those rows (codes bit-exact outside the 1e-5
    band, norms to 1e-5 relative);
  * decode: for sampled (batch, kv-head) groups the GPU cache slice is overwritten with
    the oracle's own records, the full-size decode runs, and those groups' query heads
    are compared with the oracle's attention over the same records (1e-3 per row).
    Every other output row must be finite.
Inputs come from the seeded generators of tq_inputs (drawn on the device in chunks).
"""
import math

import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as OQ
from oracle.attention import decode_attention
from oracle.codebook import lloyd_max

from _parity import as_u32, code_mismatches, rel_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")

B, HKV, HQ, N, D, BITS = 8, 8, 32, 131072, 128, 4
G = HQ // HKV


@pytest.fixture(scope="module")
def workload():
    dev = torch.device("cuda")
    rot = ti.haar_rotation(D, ti.SEEDS["rotation"] + 3)
    U = ti.haar_rotation(D, ti.SEEDS["basis"] + 3)
    kq = K.Quantizer.mse(rot, BITS, device=dev)
    vq = K.Quantizer.mse(rot, BITS, device=dev)
    n = B * HKV * N
    kx = ti.anisotropic_torch(n, D, U, ti.SEEDS["keys"] + 3, dev)
    vx = ti.anisotropic_torch(n, D, U, ti.SEEDS["values"] + 3, dev)
    q = ti.normal_torch((B, HQ, D), ti.SEEDS["queries"] + 3, dev, dtype=torch.bfloat16)
    kc, vc = K.quantize(kq, kx), K.quantize(vq, vx)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    c, t, _ = lloyd_max(BITS, "beta", d=D)
    yield dict(rot=rot, kq=kq, vq=vq, kx=kx, vx=vx, q=q, kc=kc, vc=vc, c=c, t=t)


def test_fullsize_quantize_sampled_rows(workload):
    w = workload
    n = B * HKV * N
    rng = np.random.Generator(np.random.PCG64(11))
    rows = np.unique(np.concatenate([
        rng.integers(0, n, 3900),
        np.arange(0, 128 * 148 * 2, 128 * 37),          # starts of tiles across the persistent grid
        [0, 127, 128, n - 129, n - 128, n - 1]]))
    idx = torch.from_numpy(rows).cuda()
    x64 = w["kx"].index_select(0, idx).double().cpu().numpy()
    ref = OQ.quantize_mse(x64, w["rot"], w["c"], w["t"], BITS)
    gcodes = as_u32(w["kc"].codes.index_select(0, idx))
    gnorms = w["kc"].norms.index_select(0, idx).cpu().numpy()
    bad, exempt, _ = code_mismatches(gcodes, ref["codes"], D, BITS, ref["y"], w["t"])
    assert bad == 0, f"{bad} code mismatches outside the band ({exempt} exempt)"
    assert np.max(np.abs(gnorms - ref["norms"]) / ref["norms"]) < 1e-5


@pytest.mark.parametrize("ragged", [False, True])
def test_fullsize_decode_sampled_groups(workload, ragged):
    w = workload
    lens = [N] * B
    if ragged:
        lens[2] = N - 77
        lens[7] = 1 + 176 * 5
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    kc = K.Packed(w["kc"].codes.clone(), None, w["kc"].norms.clone(), None)
    vc = K.Packed(w["vc"].codes.clone(), None, w["vc"].norms.clone(), None)
    groups = [(2, 5), (7, 7)] if ragged else [(0, 0), (5, 3)]
    refs = {}
    for b, h in groups:
        r0 = (b * HKV + h) * N
        n = lens[b]
        sel = slice(r0, r0 + n)
        k64 = w["kx"][sel].double().cpu().numpy()
        v64 = w["vx"][sel].double().cpu().numpy()
        ok = OQ.quantize_mse(k64, w["rot"], w["c"], w["t"], BITS)
        ov = OQ.quantize_mse(v64, w["rot"], w["c"], w["t"], BITS)
        kc.codes[sel] = torch.from_numpy(np.asarray(ok["codes"], dtype=np.uint32).view(np.int32)).cuda()
        kc.norms[sel] = torch.from_numpy(ok["norms"].astype(np.float32)).cuda()
        vc.codes[sel] = torch.from_numpy(np.asarray(ov["codes"], dtype=np.uint32).view(np.int32)).cuda()
        vc.norms[sel] = torch.from_numpy(ov["norms"].astype(np.float32)).cuda()
        vh = OQ.dequantize_mse(ov["idx"], ov["norms"], w["rot"], w["c"])
        q64 = w["q"][b:b + 1, h * G:(h + 1) * G].double().cpu().numpy()
        refs[(b, h)] = decode_attention(
            q64, [n], 1, lambda bb, hh, qs, ok=ok: OQ.estimate_mse(qs, w["rot"], ok["idx"], ok["norms"], w["c"]),
            lambda bb, hh, nn, vh=vh: vh[:nn], 1.0 / math.sqrt(D))[0]
    out = K.decode_attn(w["kq"], w["vq"], w["q"], sl, kc, vc, N, HKV)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    o = out.cpu().numpy()
    assert np.all(np.isfinite(o))
    for (b, h), ref in refs.items():
        err = rel_rows(o[b, h * G:(h + 1) * G], ref)
        assert np.all(err <= 1e-3), f"group {(b, h)}: max row error {err.max():.3e}"
