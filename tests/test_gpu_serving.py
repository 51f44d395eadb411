"""GPU parity of the serving forms against the oracle's serving module: a decode step that
appends its token into a paged pool and attends over it (tq_decode_attn_paged), and causal
prefill over the packed cache, contiguous and paged (tq_prefill_attn).

Each check reads the GPU's own records back, band-checks them against the oracle's
quantization of the same rows, and compares the attention output with the oracle's on
those records: per (batch, head, position) row, max |o - o_ref| <= 1e-3 max |o_ref|.
"""
import math

import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as OQ
from oracle.attention import decode_attention
from oracle.codebook import lloyd_max
from oracle.serving import page_slots, prefill_attention

from _parity import adopt_mse, adopt_prod, as_u32, rel_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")

D = 128


def _slots(table, P, Hkv, b, h, n):
    """Pool record of tokens 0..n-1 of (b, h): the oracle's page slot of the page, per head."""
    base = page_slots(table, P, b, n)            # page * P + t % P
    page, off = base // P, base % P
    return (page * Hkv + h) * P + off


def _sub(pk, rows):
    idx = torch.from_numpy(np.asarray(rows, dtype=np.int64)).cuda()
    g = lambda t: None if t is None else t.index_select(0, idx)
    return K.Packed(g(pk.codes), g(pk.signs), g(pk.norms), g(pk.rnorms))


def _scatter(pool, recs, rows):
    idx = torch.from_numpy(np.asarray(rows, dtype=np.int64)).cuda()
    for a, b in ((pool.codes, recs.codes), (pool.signs, recs.signs), (pool.norms, recs.norms),
                 (pool.rnorms, recs.rnorms)):
        if a is not None:
            a.index_copy_(0, idx, b)


def _setup(kind, seed, B, Hkv, N):
    """kind: mse (K, V mse 4), prod (K prod 3, V mse 3), prodv (K prod 3, V prod 3; one S)."""
    rot = ti.haar_rotation(D, 1010 + seed)
    S = ti.gaussian_matrix(D, D, 2010 + seed)
    U = ti.haar_rotation(D, 3010 + seed).astype(np.float64)
    kt, k64 = ti.to_bf16_f64(ti.anisotropic(B * Hkv * N, D, U, 4010 + seed))
    vt, v64 = ti.to_bf16_f64(ti.anisotropic(B * Hkv * N, D, U, 5010 + seed))
    kq = K.Quantizer.prod(rot, S, 3) if kind in ("prod", "prodv") else K.Quantizer.mse(rot, 4)
    vq = K.Quantizer.prod(rot, S, 3) if kind == "prodv" else K.Quantizer.mse(rot, 3 if kind == "prod" else 4)
    return rot, S, kq, vq, kt.cuda(), k64.reshape(B, Hkv, N, D), vt.cuda(), v64.reshape(B, Hkv, N, D)


def _oracle_records(kind, rot, S, k64, v64):
    kp = kind in ("prod", "prodv")
    ck, tk, _ = lloyd_max(2 if kp else 4, "beta", d=D)
    cv, tv, _ = lloyd_max({"mse": 4, "prod": 3, "prodv": 2}[kind], "beta", d=D)
    ok = OQ.quantize_prod(k64, rot, S, ck, tk, 3) if kp else OQ.quantize_mse(k64, rot, ck, tk, 4)
    ov = OQ.quantize_prod(v64, rot, S, cv, tv, 3) if kind == "prodv" else \
        OQ.quantize_mse(v64, rot, cv, tv, 3 if kind == "prod" else 4)
    return ok, ov, (ck, tk, cv, tv)


def _adopted_callbacks(kind, rot, S, gk, gv, ok, ov, books):
    """Oracle score and value callbacks over the GPU's band-checked records of one row set."""
    ck, tk, cv, tv = books
    if kind in ("prod", "prodv"):
        a = adopt_prod(as_u32(gk.codes), as_u32(gk.signs), gk.rnorms.cpu().numpy(), ok, 3, ck, tk, S)
        ks = lambda qs: OQ.estimate_prod(qs, rot, S, a["chat"], a["s"], ok["norms"], a["rnorms"])
    else:
        kidx, _ = adopt_mse(as_u32(gk.codes), ok, 4, tk)
        ks = lambda qs: OQ.estimate_mse(qs, rot, kidx, ok["norms"], ck)
    if kind == "prodv":
        av = adopt_prod(as_u32(gv.codes), as_u32(gv.signs), gv.rnorms.cpu().numpy(), ov, 3, cv, tv, S)
        vh = OQ.dequantize_prod(av["chat"], av["s"], ov["norms"], av["rnorms"], rot, S)
    else:
        vidx, _ = adopt_mse(as_u32(gv.codes), ov, 3 if kind == "prod" else 4, tv)
        vh = OQ.dequantize_mse(vidx, ov["norms"], rot, cv)
    for g, o in ((gk, ok), (gv, ov)):
        nrm = g.norms.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(nrm - o["norms"]) / o["norms"]) < 1e-5
    return ks, vh


@pytest.mark.parametrize("kind", ["mse", "prod", "prodv"])
def test_paged_decode_appends_then_attends(kind):
    B, Hq, Hkv, P, max_pages = 2, 8, 2, 64, 40
    lens = [1500, 777]                       # tokens including the one this step appends
    N = max(lens)
    rot, S, kq, vq, kt, k64, vt, v64 = _setup(kind, {"mse": 1, "prod": 2, "prodv": 6}[kind], B, Hkv, N)
    num_pages = B * max_pages + 5
    table = np.random.Generator(np.random.PCG64(17)).permutation(num_pages)[:B * max_pages].reshape(B, max_pages)
    pages = K.Pages(torch.from_numpy(table.astype(np.int32)).cuda(), P, num_pages)
    kpool, vpool = kq.alloc(pages.records(Hkv)), vq.alloc(pages.records(Hkv))
    # the earlier tokens go into the pool through the block table (quantized as a batch)
    kc_all, vc_all = K.quantize(kq, kt), K.quantize(vq, vt)
    for b in range(B):
        for h in range(Hkv):
            n0 = lens[b] - 1
            src = np.arange((b * Hkv + h) * N, (b * Hkv + h) * N + n0)
            dst = _slots(table, P, Hkv, b, h, n0)
            _scatter(kpool, _sub(kc_all, src), dst)
            _scatter(vpool, _sub(vc_all, src), dst)
    # this step's key and value: token lens[b] - 1 of every (b, h)
    new_rows = np.array([(b * Hkv + h) * N + lens[b] - 1 for b in range(B) for h in range(Hkv)])
    idx = torch.from_numpy(new_rows).cuda()
    k_new, v_new = kt.index_select(0, idx).contiguous(), vt.index_select(0, idx).contiguous()
    qt, q64 = ti.to_bf16_f64(ti.iid_normal((B * Hq, D), 6010))
    q = qt.reshape(B, Hq, D).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = K.decode_attn_paged(kq, vq, q, seq, pages, kpool, vpool, Hkv, k_new=k_new, v_new=v_new)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    o = out.cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hkv):
            n = lens[b]
            dst = _slots(table, P, Hkv, b, h, n)
            gk, gv = _sub(kpool, dst), _sub(vpool, dst)
            # the appended record equals what the batch quantize wrote for that row
            last = (b * Hkv + h) * N + n - 1
            assert np.array_equal(as_u32(gk.codes)[-1], as_u32(kc_all.codes[last:last + 1])[0])
            assert np.array_equal(as_u32(gv.codes)[-1], as_u32(vc_all.codes[last:last + 1])[0])
            ok, ov, books = _oracle_records(kind, rot, S, k64[b, h, :n], v64[b, h, :n])
            ks, vh = _adopted_callbacks(kind, rot, S, gk, gv, ok, ov, books)
            ref = decode_attention(q64.reshape(B, Hq, D)[b:b + 1, h * G:(h + 1) * G], [n], 1,
                                   lambda bb, hh, qs: ks(qs), lambda bb, hh, m: vh[:m], 1.0 / math.sqrt(D))[0]
            err = rel_rows(o[b, h * G:(h + 1) * G], ref)
            assert np.all(err <= 1e-3), f"{(b, h)}: {err.max():.3e}"


def test_paged_decode_bad_page_id_is_reported():
    B, Hq, Hkv, P, max_pages = 1, 4, 1, 32, 4
    rot = ti.haar_rotation(D, 1013)
    kq, vq = K.Quantizer.mse(rot, 4), K.Quantizer.mse(rot, 4)
    num_pages = 4
    table = torch.tensor([[0, 1, 7, 3]], dtype=torch.int32, device="cuda")     # page 7 does not exist
    pages = K.Pages(table, P, num_pages)
    kpool, vpool = kq.alloc(pages.records(Hkv)), vq.alloc(pages.records(Hkv))
    q = torch.ones((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([100], dtype=torch.int32, device="cuda")
    K.decode_attn_paged(kq, vq, q, seq, pages, kpool, vpool, Hkv)
    assert K.get_status() == 1          # TQ_ERR_INVALID_ARG, recorded on the device
    assert K.get_status() == 0


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("kind", ["mse", "prod"])
def test_prefill_is_causal_attention_over_the_cache(kind, paged):
    B, Hq, Hkv, T = 2, 8, 2, 37
    lens = [900, 1203]
    N = 1216 if not paged else max(lens)
    rot, S, kq, vq, kt, k64, vt, v64 = _setup(kind, 3 if kind == "mse" else 4, B, Hkv, N)
    kc, vc = K.quantize(kq, kt), K.quantize(vq, vt)
    # positions: a chunk ending at the last cached token, and scattered sorted positions
    pos = np.stack([np.arange(lens[0] - T, lens[0]),
                    np.sort(np.random.Generator(np.random.PCG64(5)).choice(lens[1], T, replace=False))]).astype(np.int32)
    qt, q64 = ti.to_bf16_f64(ti.iid_normal((B * Hq * T, D), 6011))
    q = qt.reshape(B, Hq, T, D).cuda()
    qpos = torch.from_numpy(pos).cuda()
    kvl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    if paged:
        P, max_pages = 32, (N + 31) // 32
        num_pages = B * max_pages
        table = np.random.Generator(np.random.PCG64(23)).permutation(num_pages).reshape(B, max_pages)
        pages = K.Pages(torch.from_numpy(table.astype(np.int32)).cuda(), P, num_pages)
        kpool, vpool = kq.alloc(pages.records(Hkv)), vq.alloc(pages.records(Hkv))
        for b in range(B):
            for h in range(Hkv):
                src = np.arange((b * Hkv + h) * N, (b * Hkv + h) * N + lens[b])
                dst = _slots(table, P, Hkv, b, h, lens[b])
                _scatter(kpool, _sub(kc, src), dst)
                _scatter(vpool, _sub(vc, src), dst)
        out = K.prefill_attn(kq, vq, q, qpos, kvl, kpool, vpool, Hkv, pages=pages)
    else:
        out = K.prefill_attn(kq, vq, q, qpos, kvl, kc, vc, Hkv, Nmax=N)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    o = out.cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hkv):
            n = lens[b]
            rows = np.arange((b * Hkv + h) * N, (b * Hkv + h) * N + n)
            ok, ov, books = _oracle_records(kind, rot, S, k64[b, h, :n], v64[b, h, :n])
            ks, vh = _adopted_callbacks(kind, rot, S, _sub(kc, rows), _sub(vc, rows), ok, ov, books)
            qq = q64.reshape(B, Hq, T, D)[b:b + 1, h * G:(h + 1) * G]
            ref = prefill_attention(qq, pos[b:b + 1], 1, lambda bb, hh, qs: ks(qs), lambda bb, hh, m: vh[:m],
                                    1.0 / math.sqrt(D))[0]
            err = rel_rows(o[b, h * G:(h + 1) * G].reshape(G * T, D), ref.reshape(G * T, D))
            assert np.all(err <= 1e-3), f"{(b, h)}: {err.max():.3e}"


def test_prefill_of_the_last_position_is_the_decode_step():
    """Two GPU routes, one step: a one-query prefill at position len - 1 equals decode."""
    B, Hq, Hkv, N = 2, 8, 2, 1000
    lens = [1000, 613]
    rot, S, kq, vq, kt, _, vt, _ = _setup("mse", 5, B, Hkv, N)
    kc, vc = K.quantize(kq, kt), K.quantize(vq, vt)
    q = torch.from_numpy(ti.iid_normal((B, Hq, D), 6012).astype(np.float32)).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    dec = K.decode_attn(kq, vq, q, seq, kc, vc, N, Hkv)
    pos = torch.tensor([[lens[0] - 1], [lens[1] - 1]], dtype=torch.int32, device="cuda")
    pre = K.prefill_attn(kq, vq, q.reshape(B, Hq, 1, D).contiguous(), pos, seq, kc, vc, Hkv, Nmax=N)
    torch.cuda.synchronize()
    assert K.get_status() == 0
    err = rel_rows(pre.reshape(B, Hq, D).cpu().numpy(), dec.cpu().numpy())
    assert np.all(err <= 1e-5), err.max()
