"""GPU parity: inner-product estimates and exhaustive top-k vs the oracle."""
import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as OQ
from oracle.codebook import lloyd_max
from oracle.search import topk as otopk

from _parity import adopt_mse, adopt_prod, as_u32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")


def test_scores_c1_mse_fp32():
    """Single head d=128, 4096 fp32 keys ~ N(0, 1/d), 64 queries, mse b=3."""
    d, n, nq, b = 128, 4096, 64, 3
    rot = ti.haar_rotation(d, 1001)
    x = ti.iid_normal((n, d), 4001, std=1 / np.sqrt(d)).astype(np.float32)
    qv = ti.iid_normal((nq, d), 6001, std=1 / np.sqrt(d)).astype(np.float32)
    q = K.Quantizer.mse(rot, b)
    pk = K.quantize(q, torch.from_numpy(x).cuda())
    s = K.score(q, torch.from_numpy(qv).cuda(), pk, n).cpu().numpy().astype(np.float64)
    c, t, _ = lloyd_max(b, "beta", d=d)
    ref = OQ.quantize_mse(x.astype(np.float64), rot, c, t, b)
    # band-check the GPU's codes, then rescore every record with them
    idx, exempt = adopt_mse(as_u32(pk.codes), ref, b, t)
    assert exempt <= max(2, 1e-4 * n * d)
    est = OQ.estimate_mse(qv.astype(np.float64), rot, idx, ref["norms"], c)
    scale = np.linalg.norm(qv, axis=1)[:, None] * np.linalg.norm(x, axis=1)[None, :]
    assert np.all(np.abs(s - est) <= 1e-3 * scale)
    # quality context: estimates vs exact inner products (MSE stage is biased by 1 - D_3)
    exact = qv.astype(np.float64) @ x.astype(np.float64).T
    slope = np.sum(est * exact) / np.sum(exact * exact)
    assert 0.9 < slope < 1.0


@pytest.mark.parametrize("d,bits,n,nq", [(128, 3, 3000, 16), (1536, 2, 2000, 8), (1536, 4, 1000, 8)])
def test_scores_prod(d, bits, n, nq):
    rot = ti.haar_rotation(d, 1005)
    S = ti.gaussian_matrix(d, d, 2005)
    x = ti.unit_gaussian(n, d, 8000).astype(np.float32)
    qv = ti.unit_gaussian(nq, d, 8001).astype(np.float32)
    q = K.Quantizer.prod(rot, S, bits)
    pk = K.quantize(q, torch.from_numpy(x).cuda())
    s = K.score(q, torch.from_numpy(qv).cuda(), pk, n).cpu().numpy().astype(np.float64)
    c, t, _ = lloyd_max(bits - 1, "beta", d=d)
    ref = OQ.quantize_prod(x.astype(np.float64), rot, S, c, t, bits)
    a = adopt_prod(as_u32(pk.codes), as_u32(pk.signs), pk.rnorms.cpu().numpy(), ref, bits, c, t, S)
    est = OQ.estimate_prod(qv.astype(np.float64), rot, S, a["chat"], a["s"], ref["norms"], a["rnorms"])
    assert np.all(np.abs(s - est) <= 1e-3)       # unit-norm q and x: 1e-3 ||q|| ||x||


@pytest.mark.parametrize("bits", [2, 4])
def test_topk_search(bits):
    """Exhaustive top-10 by estimated inner product (unit-norm Gaussian DB, d=1536)."""
    d, n, nq, k = 1536, 20000, 12, 10
    rot = ti.haar_rotation(d, 1005)
    S = ti.gaussian_matrix(d, d, 2005)
    x = ti.unit_gaussian(n, d, 8000).astype(np.float32)
    qv = ti.unit_gaussian(nq, d, 8001).astype(np.float32)
    q = K.Quantizer.prod(rot, S, bits)
    pk = K.quantize(q, torch.from_numpy(x).cuda())
    vals, ids = K.score(q, torch.from_numpy(qv).cuda(), pk, n, topk=k)
    vals, ids = vals.cpu().numpy().astype(np.float64), ids.cpu().numpy()
    c, t, _ = lloyd_max(bits - 1, "beta", d=d)
    ref = OQ.quantize_prod(x.astype(np.float64), rot, S, c, t, bits)
    a = adopt_prod(as_u32(pk.codes), as_u32(pk.signs), pk.rnorms.cpu().numpy(), ref, bits, c, t, S)
    est = OQ.estimate_prod(qv.astype(np.float64), rot, S, a["chat"], a["s"], ref["norms"], a["rnorms"])
    rid, rval = otopk(est, k)
    tol = 1e-3
    for i in range(nq):
        # the GPU's list is sorted, its scores match the oracle's estimates of the same ids,
        # and every id the oracle ranks clearly inside the top-k is present
        assert np.all(np.diff(vals[i]) <= 0)
        assert np.all(np.abs(vals[i] - est[i, ids[i]]) <= tol)
        kth = rval[i, -1]
        must = rid[i][rval[i] > kth + 2 * tol]
        assert set(must.tolist()) <= set(ids[i].tolist())
        assert np.all(est[i, ids[i]] >= kth - 2 * tol)


@pytest.mark.parametrize("d,kind,bits,n,nq", [(1536, "prod", 2, 5000, 7), (256, "mse", 3, 4500, 130),
                                              (512, "prod", 5, 4099, 3), (512, "mse", 2, 4100, 9),
                                              (384, "mse", 1, 4500, 6)])
def test_scores_wide_tensor_core(d, kind, bits, n, nq):
    """Dense estimates on the tensor cores (d a multiple of 128, at least 4096 records): every
    (query, record) estimate equals the oracle's on the GPU's band-checked records to 1e-3
    (unit-norm queries and records); the ragged last column tile and query tile included."""
    rot = ti.haar_rotation(d, 1405 + d)
    S = ti.gaussian_matrix(d, d, 2405 + d)
    x = ti.unit_gaussian(n, d, 8100 + d).astype(np.float32)
    qv = ti.unit_gaussian(nq, d, 8101 + d).astype(np.float32)
    q = K.Quantizer.prod(rot, S, bits) if kind == "prod" else K.Quantizer.mse(rot, bits)
    pk = K.quantize(q, torch.from_numpy(x).cuda())
    s = K.score(q, torch.from_numpy(qv).cuda(), pk, n).cpu().numpy().astype(np.float64)
    assert K.get_status() == 0
    if kind == "prod":
        c, t, _ = lloyd_max(bits - 1, "beta", d=d)
        ref = OQ.quantize_prod(x.astype(np.float64), rot, S, c, t, bits)
        a = adopt_prod(as_u32(pk.codes), as_u32(pk.signs), pk.rnorms.cpu().numpy(), ref, bits, c, t, S)
        est = OQ.estimate_prod(qv.astype(np.float64), rot, S, a["chat"], a["s"], ref["norms"], a["rnorms"])
    else:
        c, t, _ = lloyd_max(bits, "beta", d=d)
        ref = OQ.quantize_mse(x.astype(np.float64), rot, c, t, bits)
        idx, _ = adopt_mse(as_u32(pk.codes), ref, bits, t)
        est = OQ.estimate_mse(qv.astype(np.float64), rot, idx, ref["norms"], c)
    assert np.max(np.abs(s - est)) <= 1e-3


def test_topk_segments_ties():
    """The tensor-core path takes the top-k over segments of ~16k estimates and then over their
    candidates; the result must be that of one pass over the row: descending estimate, ties to
    the lower id.  n = 40,000 makes three segments (boundaries at 13,334 and 26,668); one record
    is copied to ids in all three and is query 0, so its copies tie at the top.  The reference is
    a host top-k of the same call's dense estimates."""
    d, n, nq, k = 256, 40000, 6, 12
    rot = ti.haar_rotation(d, 1406)
    x = ti.unit_gaussian(n, d, 8102).astype(np.float32)
    dup = [5, 123, 13333, 13334, 20000, 26668, 39999]
    x[dup] = x[123]
    qv = ti.unit_gaussian(nq, d, 8103).astype(np.float32)
    qv[0] = x[123]
    q = K.Quantizer.mse(rot, 3)
    pk = K.quantize(q, torch.from_numpy(x).cuda())
    qt = torch.from_numpy(qv).cuda()
    dense = K.score(q, qt, pk, n).cpu().numpy()
    vals, ids = K.score(q, qt, pk, n, topk=k)
    vals, ids = vals.cpu().numpy(), ids.cpu().numpy()
    assert K.get_status() == 0
    for i in range(nq):
        order = np.lexsort((np.arange(n), -dense[i].astype(np.float64)))[:k]
        assert ids[i].tolist() == order.tolist(), f"query {i}"
        assert np.array_equal(vals[i], dense[i, order])
    # the copies carry equal records, hence equal estimates, and lead query 0 in id order
    assert ids[0][:len(dup)].tolist() == sorted(dup)
