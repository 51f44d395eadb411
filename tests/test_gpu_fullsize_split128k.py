"""GPU parity of the outlier-split path at the 128k-context decode shapes (B=8, Hkv=8, Hq=32,
d=128, context 131072; keys and values split 32 channels at 3 bits + 96 at 2 bits, the
2.5-bit setting of the TurboQuant review's KV experiments), in the launch configuration
`bench.py --workload split` times: the tensor-core split quantize and split decode.

The oracle cannot process 8.4 M vectors, so the comparison is on samples:
  * quantize: 4096 rows spread over the array against the oracle's split quantization of
    those rows (codes bit-exact outside the 1e-5 band, norms to 1e-5 relative);
  * decode: for sampled (batch, kv-head) groups, the oracle's split attention over the
    GPU's own records of those groups (1e-3 per row); every other output row is finite.
"""
import numpy as np
import pytest

import tq_inputs as ti
from oracle import attention as OA
from oracle import quantizer as OQ
from oracle import split as OS
from oracle.codebook import lloyd_max

from _parity import as_u32, code_mismatches, rel_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")

B, HKV, HQ, N, D = 8, 8, 32, 131072, 128
PLANTED = np.sort(np.random.Generator(np.random.PCG64(78)).choice(D, 32, replace=False))
GROUPS = [PLANTED, np.setdiff1d(np.arange(D), PLANTED)]
BITS = [3, 2]


def _planted(n, seed, dev):
    x = ti.normal_torch((n, D), seed, dev)
    x[:, torch.from_numpy(PLANTED).to(dev)] *= 6.0
    return x.to(torch.bfloat16).contiguous()


@pytest.fixture(scope="module")
def workload():
    dev = torch.device("cuda")
    ins, qs = [], []
    for ch, b in zip(GROUPS, BITS):
        dg = len(ch)
        rot = ti.haar_rotation(dg, 1300 + dg)
        c, t, _ = lloyd_max(b, "beta", d=dg)
        ins.append({"kind": "mse", "rot": rot.astype(np.float64), "centroids": c, "boundaries": t, "bits": b})
        qs.append(K.Quantizer.mse(rot, b, device=dev))
    cols = [torch.from_numpy(np.asarray(ch, dtype=np.int32)).to(dev) for ch in GROUPS]
    sp = K.Split(D, qs, cols)
    n = B * HKV * N
    kx = _planted(n, ti.SEEDS["keys"] + 12, dev)
    kp = K.quantize_split(sp, kx)
    vx = _planted(n, ti.SEEDS["values"] + 12, dev)
    vp = K.quantize_split(sp, vx)
    del vx
    torch.cuda.synchronize()
    assert K.get_status() == 0
    q = ti.normal_torch((B, HQ, D), ti.SEEDS["queries"] + 12, dev)
    yield dict(sp=sp, ins=ins, kx=kx, kp=kp, vp=vp, q=q)


def test_fullsize_split_quantize_sampled_rows(workload):
    w = workload
    n = B * HKV * N
    rng = np.random.Generator(np.random.PCG64(12))
    rows = np.unique(np.concatenate([rng.integers(0, n, 4000), [0, 127, 128, n - 129, n - 128, n - 1]]))
    idx = torch.from_numpy(rows).cuda()
    x64 = w["kx"].index_select(0, idx).double().cpu().numpy()
    ref = OS.quantize_split(x64, GROUPS, w["ins"])
    for g, (ch, r) in enumerate(zip(GROUPS, ref)):
        gc = as_u32(w["kp"][g].codes.index_select(0, idx))
        gn = w["kp"][g].norms.index_select(0, idx).cpu().numpy().astype(np.float64)
        bad, exempt, _ = code_mismatches(gc, r["codes"], len(ch), BITS[g], r["y"], w["ins"][g]["boundaries"])
        assert bad == 0, f"group {g}: {bad} code mismatches outside the band ({exempt} exempt)"
        assert np.all(np.abs(gn - r["norms"]) <= 1e-5 * r["norms"])


@pytest.mark.parametrize("ragged", [False, True])
def test_fullsize_split_decode_sampled_groups(workload, ragged):
    w = workload
    lens = [N] * B
    if ragged:
        lens[3] = N - 77
        lens[6] = 1 + 352 * 3
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o = K.decode_attn_split(w["sp"], w["sp"], w["q"], seq, w["kp"], w["vp"], N, HKV)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    o = o.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    G = HQ // HKV
    q64 = w["q"].cpu().numpy().astype(np.float64)
    for b, h in [(0, 0), (3, 5), (6, 2), (7, 7)]:
        n_ = lens[b]
        base = (b * HKV + h) * N

        def recs(packs):
            out = []
            for pk, ch, g in zip(packs, GROUPS, w["ins"]):
                idx = OQ.unpack_codes(as_u32(pk.codes[base:base + n_]), len(ch), g["bits"])
                out.append({"idx": idx, "norms": pk.norms[base:base + n_].cpu().numpy().astype(np.float64)})
            return out

        kr, vr = recs(w["kp"]), recs(w["vp"])
        qs = q64[b, h * G:(h + 1) * G]
        logits = OS.estimate_split(qs, kr, GROUPS, w["ins"]) / np.sqrt(D)
        ref = OA.softmax_attend(logits, OS.dequantize_split(vr, GROUPS, w["ins"], D))
        err = rel_rows(o[b, h * G:(h + 1) * G], ref)
        assert np.all(err <= 1e-3), f"(b={b}, h={h}) max row error {err.max():.2e}"
