"""GPU parity: outlier-channel split (quantize and summed estimates) against the oracle.

Setting of the TurboQuant review, Method: 32 outlier channels at 3 bits plus 96 channels
at 2 bits, each group an independent TurboQuant instance; keys with planted high-magnitude
channels, found by the oracle's online detection rule.
"""
import numpy as np
import pytest

import tq_inputs as ti
from oracle import attention as OA
from oracle import quantizer as OQ
from oracle import split as OS
from oracle.codebook import lloyd_max
from oracle.search import topk as otopk

from _parity import as_u32, code_mismatches, rel_rows, sign_mismatches

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")

D = 128
PLANTED = np.sort(np.random.Generator(np.random.PCG64(77)).choice(D, 32, replace=False))


def _setup(kind, n, seed, dtype="bf16", bits=(3, 2), zero_rows=False):
    x = ti.planted_outliers(n, D, PLANTED, 6.0, seed)
    if zero_rows:
        x[3] = 0.0                                      # a zero row
        x[5, PLANTED] = 0.0                             # a row whose outlier group is zero
    if dtype == "bf16":
        xt, x64 = ti.to_bf16_f64(x)
    else:
        x32 = x.astype(np.float32)
        xt, x64 = torch.from_numpy(x32), x32.astype(np.float64)
    groups = OS.split_groups(D, OS.outlier_channels(x64, 32))
    assert np.array_equal(groups[0], PLANTED)
    ins, qs = [], []
    for g, (ch, b) in enumerate(zip(groups, bits)):
        dg = len(ch)
        rot = ti.haar_rotation(dg, 1200 + dg)
        if kind == "mse":
            c, t, _ = lloyd_max(b, "beta", d=dg)
            ins.append({"kind": "mse", "rot": rot.astype(np.float64), "centroids": c, "boundaries": t, "bits": b})
            qs.append(K.Quantizer.mse(rot, b))
        else:
            S = ti.gaussian_matrix(dg, dg, 2200 + dg)
            c, t, _ = lloyd_max(b - 1, "beta", d=dg)
            ins.append({"kind": "prod", "rot": rot.astype(np.float64), "S": S.astype(np.float64),
                        "centroids": c, "boundaries": t, "bits": b})
            qs.append(K.Quantizer.prod(rot, S, b))
    cols = [torch.from_numpy(np.asarray(ch, dtype=np.int32)).cuda() for ch in groups]
    sp = K.Split(D, qs, cols)
    return xt.cuda().contiguous(), x64, groups, ins, sp


# 16-bit MSE splits of 32 @ 3 + 96 @ 2 or 32 @ 4 + 96 @ 3 bits take the tensor-core pass over
# whole rows; fp32 rows and prod groups the CUDA-core kernel with the gather on the load
@pytest.mark.parametrize("kind,n,dtype,bits", [("mse", 3000, "bf16", (3, 2)), ("mse", 777, "f32", (3, 2)),
                                               ("prod", 1500, "bf16", (3, 2)), ("mse", 1500, "bf16", (4, 3)),
                                               ("mse", 129, "bf16", (3, 2))])
def test_quantize_split_parity(kind, n, dtype, bits):
    x, x64, groups, ins, sp = _setup(kind, n, 4300 + n, dtype, bits, zero_rows=True)
    out = K.quantize_split(sp, x)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    ref = OS.quantize_split(x64, groups, ins)
    for g, (ch, r, o) in enumerate(zip(groups, ref, out)):
        dg, b = len(ch), ins[g]["bits"]
        bm = b if kind == "mse" else b - 1
        bad, exempt, skip = code_mismatches(as_u32(o.codes), r["codes"], dg, bm, r["y"], ins[g]["boundaries"])
        assert bad == 0, f"group {g}: {bad} code mismatches outside the band"
        assert exempt <= max(2, 1e-4 * n * dg)
        nrm = o.norms.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(nrm - r["norms"]) <= 1e-5 * r["norms"])
        if kind == "prod":
            sbad, sex = sign_mismatches(as_u32(o.signs), r["signs"], dg, r["proj"], ins[g]["S"], skip)
            assert sbad == 0 and sex <= max(3, 2e-3 * n)
            rn = o.rnorms.cpu().numpy().astype(np.float64)
            ok = np.array([i not in skip for i in range(n)])
            assert np.all(np.abs(rn[ok] - r["rnorms"][ok]) <= 1e-5 * np.maximum(r["rnorms"][ok], 1e-6) + 1e-6)


def test_quantize_split_equals_gathered_single_instances():
    # on the CUDA-core path (fp32 rows) the split call writes exactly what the single-instance
    # call writes for the gathered rows (same kernel, gather on the load)
    n = 1000
    x, x64, groups, ins, sp = _setup("mse", n, 4400, "f32")
    out = K.quantize_split(sp, x)
    for g, ch in enumerate(groups):
        xg = x[:, torch.from_numpy(np.asarray(ch)).cuda()].contiguous().float()
        single = K.quantize(sp.groups[g], xg)
        assert torch.equal(single.codes, out[g].codes)
        assert torch.equal(single.norms, out[g].norms)


# below 4096 records the CUDA-core estimator accumulates the groups; from 4096 on one
# split-precision tensor-core product covers every group's columns
@pytest.mark.parametrize("kind,n", [("mse", 2000), ("prod", 2000), ("mse", 6000), ("prod", 4500)])
def test_score_split_parity(kind, n):
    nq = 12
    x, x64, groups, ins, sp = _setup(kind, n, 4500)
    qv = ti.iid_normal((nq, D), 6500).astype(np.float32)
    out = K.quantize_split(sp, x)
    s = K.score_split(sp, torch.from_numpy(qv).cuda(), out, n).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    ref = OS.quantize_split(x64, groups, ins)
    same = np.ones(n, dtype=bool)
    for o, r in zip(out, ref):
        same &= np.all(as_u32(o.codes) == r["codes"], axis=1)
        if kind == "prod":
            same &= np.all(as_u32(o.signs) == r["signs"], axis=1)
    est = OS.estimate_split(qv.astype(np.float64), ref, groups, ins)
    scale = np.linalg.norm(qv, axis=1)[:, None] * np.linalg.norm(x64, axis=1)[None, :]
    assert same.mean() > 0.99
    assert np.all(np.abs(s - est)[:, same] <= 1e-3 * scale[:, same])
    # top-k of the summed estimate: sorted, scores are the estimates of the returned ids,
    # and every id clearly inside the oracle's top-k is present
    k = 10
    vals, ids = K.score_split(sp, torch.from_numpy(qv).cuda(), out, n, topk=k)
    vals, ids = vals.cpu().numpy().astype(np.float64), ids.cpu().numpy()
    rid, rval = otopk(est, k)
    for i in range(nq):
        tol = 1e-3 * np.max(scale[i])
        assert np.all(np.diff(vals[i]) <= 0)
        assert np.all(np.abs(vals[i] - est[i, ids[i]]) <= tol)
        must = rid[i][rval[i] > rval[i, -1] + 2 * tol]
        assert set(must.tolist()) <= set(ids[i].tolist())


def test_bad_channel_index_reports_status():
    x, x64, groups, ins, sp = _setup("mse", 300, 4600)
    bad = sp.cols[1].clone()
    bad[5] = D                                            # one past the last channel
    sp2 = K.Split(D, sp.groups, [sp.cols[0], bad])
    K.quantize_split(sp2, x)
    torch.cuda.synchronize()
    assert K.get_status() == 1                            # TQ_ERR_INVALID_ARG
    assert K.get_status() == 0


def _records_from_gpu(packs, groups, ins):
    """The GPU's own records as oracle record dicts (codes unpacked, fp32 norms; a PROD
    group adds c[idx], its sign bits and its residual norms)."""
    recs = []
    for pk, ch, g in zip(packs, groups, ins):
        nrm = pk.norms.cpu().numpy().astype(np.float64)
        if g["kind"] == "mse":
            idx = OQ.unpack_codes(as_u32(pk.codes), len(ch), g["bits"])
            recs.append({"idx": idx, "norms": nrm})
        else:
            idx = OQ.unpack_codes(as_u32(pk.codes), len(ch), g["bits"] - 1)
            m = g["S"].shape[0]
            recs.append({"idx": idx, "norms": nrm, "chat": np.asarray(g["centroids"], dtype=np.float64)[idx],
                         "s": OQ.unpack_signs(as_u32(pk.signs), m),
                         "rnorms": pk.rnorms.cpu().numpy().astype(np.float64)})
    return recs


# MSE splits with GQA groups of at most 4 heads and rows of a multiple of 4 records take the
# tensor-core kernel; 8 heads per group or an odd row length the CUDA-core one
@pytest.mark.parametrize("kkind,B,Hkv,Hq,Nmax,lens", [("mse", 2, 2, 8, 700, [700, 333]),
                                                       ("mse", 1, 4, 8, 3000, [2999]),
                                                       ("mse", 3, 1, 1, 300, [1, 300, 17]),
                                                       ("mse", 2, 4, 16, 4100, [4100, 2055]),
                                                       ("mse", 1, 2, 6, 1028, [1027]),
                                                       ("mse", 1, 1, 8, 501, [501]),
                                                       ("prod", 2, 2, 8, 700, [700, 333]),
                                                       ("prod", 1, 2, 4, 2100, [2100]),
                                                       ("prod", 3, 1, 1, 300, [1, 300, 17])])
def test_decode_attn_split_parity(kkind, B, Hkv, Hq, Nmax, lens):
    # the attention step read straight from split caches against the oracle's split
    # attention on the same records (keys with planted outlier channels, 32 @ 3 b + 96 @ 2 b
    # MSE or TurboQuant-prod instances; values split the same way, MSE)
    n = B * Hkv * Nmax
    kx, k64, groups, kins, ks = _setup(kkind, n, 4700 + Nmax)
    vx64 = ti.iid_normal((n, D), 4800 + Nmax)
    vxt, vx64 = ti.to_bf16_f64(vx64)
    vx = vxt.cuda().contiguous()
    if kkind == "mse":
        vins, vs = kins, ks                                # the same split for the values
    else:
        _, _, vgroups, vins, vs = _setup("mse", 2000, 4750)
        assert all(np.array_equal(a, b) for a, b in zip(groups, vgroups))
    kp = K.quantize_split(ks, kx)
    vp = K.quantize_split(vs, vx)
    q64 = ti.iid_normal((B, Hq, D), 4900 + Nmax)
    q = torch.from_numpy(q64.astype(np.float32)).cuda()
    seq = torch.tensor(lens, dtype=torch.int32).cuda()
    o = K.decode_attn_split(ks, vs, q, seq, kp, vp, Nmax, Hkv).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    kr, vr = _records_from_gpu(kp, groups, kins), _records_from_gpu(vp, groups, vins)

    def rows(recs, b, h, n_):
        base = (b * Hkv + h) * Nmax
        return [{k: v[base:base + n_] for k, v in r.items()} for r in recs]

    scale = 1.0 / np.sqrt(D)
    ref = OA.decode_attention(q.cpu().numpy().astype(np.float64), lens, Hkv,
                              lambda b, h, qs: OS.estimate_split(qs, rows(kr, b, h, lens[b]), groups, kins),
                              lambda b, h, n_: OS.dequantize_split(rows(vr, b, h, n_), groups, vins, D), scale)
    err = rel_rows(o, ref)
    assert np.all(err <= 1e-3), f"max row error {err.max():.2e}"
