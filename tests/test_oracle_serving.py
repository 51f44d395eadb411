"""Pins for oracle.serving: paged cache, append-then-attend, causal prefill over the cache."""
import numpy as np
import pytest

import tq_inputs as ti
from oracle import attention as A
from oracle import quantizer as Q
from oracle import serving as SV
from oracle.codebook import lloyd_max

torch = pytest.importorskip("torch")

D = 64


@pytest.fixture(scope="module")
def book():
    c, t, _ = lloyd_max(3, "beta", d=D)
    return ti.haar_rotation(D, 21).astype(np.float64), c, t


def _mse_callbacks(rec_k, rec_v, rot, c, slots):
    """Attention callbacks over per-(b, h) record sets; slots(b, h, n) lists the records."""
    def ks(b, h, qs):
        s = slots(b, h, None)
        return Q.estimate_mse(qs, rot, rec_k["idx"][s], rec_k["norms"][s], c)

    def vr(b, h, n):
        s = slots(b, h, n)
        return Q.dequantize_mse(rec_v["idx"][s], rec_v["norms"][s], rot, c)
    return ks, vr


def test_prefill_with_exact_cache_is_masked_softmax_attention():
    # exact keys/values: the causal prefill equals torch's scaled-dot-product attention
    # with the same boolean mask (float64 on the CPU)
    B, Hkv, Hq, T, n = 2, 2, 4, 5, 12
    K = ti.iid_normal((B, Hkv, n, D), 1)
    V = ti.iid_normal((B, Hkv, n, D), 2)
    q = ti.iid_normal((B, Hq, T, D), 3)
    pos = np.array([[7, 8, 9, 10, 11], [0, 3, 3, 6, 11]])
    scale = 1.0 / np.sqrt(D)
    got = SV.prefill_attention(q, pos, Hkv, lambda b, h, qs: qs @ K[b, h].T, lambda b, h, m: V[b, h, :m], scale)
    G = Hq // Hkv
    for b in range(B):
        m = int(pos[b].max()) + 1
        mask = torch.from_numpy(np.arange(m)[None, :] <= pos[b][:, None])
        for hq in range(Hq):
            h = hq // G
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[b, hq])[None], torch.from_numpy(K[b, h, :m])[None],
                torch.from_numpy(V[b, h, :m])[None], attn_mask=mask[None], scale=scale)[0].numpy()
            np.testing.assert_allclose(got[b, hq], ref, rtol=1e-12, atol=1e-12)


def test_prefill_of_one_query_at_the_end_is_the_decode_step(book):
    rot, c, t = book
    B, Hkv, Hq, n = 2, 2, 8, 40
    K = ti.iid_normal((B * Hkv * n, D), 4)
    V = ti.iid_normal((B * Hkv * n, D), 5)
    rk, rv = Q.quantize_mse(K, rot, c, t, 3), Q.quantize_mse(V, rot, c, t, 3)
    lens = [n, 23]
    q = ti.iid_normal((B, Hq, D), 6)

    def slots(b, h, m):
        base = (b * Hkv + h) * n
        return np.arange(base, base + (lens[b] if m is None else m))
    ks, vr = _mse_callbacks(rk, rv, rot, c, slots)
    scale = 1.0 / np.sqrt(D)
    dec = A.decode_attention(q, lens, Hkv, ks, vr, scale)
    pos = np.array([[lens[0] - 1], [lens[1] - 1]])
    pre = SV.prefill_attention(q[:, :, None, :], pos, Hkv, ks, vr, scale)[:, :, 0, :]
    np.testing.assert_allclose(pre, dec, rtol=1e-13, atol=1e-13)


def test_paged_cache_reads_the_same_records_as_the_contiguous_one(book):
    # records written into a pool through a shuffled block table give the attention
    # of the contiguous layout exactly
    rot, c, t = book
    B, Hkv, Hq, P, pages = 2, 1, 2, 8, 5
    n = P * pages
    K = ti.iid_normal((B * n, D), 7)
    V = ti.iid_normal((B * n, D), 8)
    rk, rv = Q.quantize_mse(K, rot, c, t, 3), Q.quantize_mse(V, rot, c, t, 3)
    lens = [n, 29]
    q = ti.iid_normal((B, Hq, D), 9)
    perm = np.random.Generator(np.random.PCG64(3)).permutation(B * pages)
    table = perm.reshape(B, pages)
    pool_k = {k: np.zeros_like(v) for k, v in rk.items() if k in ("idx", "norms")}
    pool_v = {k: np.zeros_like(v) for k, v in rv.items() if k in ("idx", "norms")}
    for b in range(B):
        dst = SV.page_slots(table, P, b, n)
        for pool, rec in ((pool_k, rk), (pool_v, rv)):
            pool["idx"][dst] = rec["idx"][b * n:(b + 1) * n]
            pool["norms"][dst] = rec["norms"][b * n:(b + 1) * n]
    scale = 1.0 / np.sqrt(D)
    contiguous = A.decode_attention(q, lens, Hkv, *_mse_callbacks(
        rk, rv, rot, c, lambda b, h, m: np.arange(b * n, b * n + (lens[b] if m is None else m))), scale)
    paged = A.decode_attention(q, lens, Hkv, *_mse_callbacks(
        pool_k, pool_v, rot, c, lambda b, h, m: SV.page_slots(table, P, b, lens[b] if m is None else m)), scale)
    np.testing.assert_array_equal(paged, contiguous)


def test_append_then_attend_matches_quantizing_the_whole_stream(book):
    # quantization is per vector and online: appending the step's token to a cache built
    # from the earlier tokens gives the records (and the attention) of the whole stream
    rot, c, t = book
    n = 30
    K = ti.iid_normal((n + 1, D), 10)
    V = ti.iid_normal((n + 1, D), 11)
    whole_k, whole_v = Q.quantize_mse(K, rot, c, t, 3), Q.quantize_mse(V, rot, c, t, 3)
    old_k, old_v = Q.quantize_mse(K[:n], rot, c, t, 3), Q.quantize_mse(V[:n], rot, c, t, 3)
    new_k, new_v = Q.quantize_mse(K[n:], rot, c, t, 3), Q.quantize_mse(V[n:], rot, c, t, 3)
    for whole, old, new in ((whole_k, old_k, new_k), (whole_v, old_v, new_v)):
        assert np.array_equal(np.concatenate([old["codes"], new["codes"]]), whole["codes"])
        np.testing.assert_allclose(np.concatenate([old["norms"], new["norms"]]), whole["norms"], rtol=1e-15)
    # the first step of a sequence attends to its own token only: the output is v_hat
    q = ti.iid_normal((1, 2, D), 12)
    one = A.decode_attention(q, [1], 1, *_mse_callbacks(new_k, new_v, rot, c,
                                                        lambda b, h, m: np.arange(1)), 1.0 / np.sqrt(D))
    vhat = Q.dequantize_mse(new_v["idx"], new_v["norms"], rot, c)[0]
    np.testing.assert_allclose(one[0], np.stack([vhat, vhat]), rtol=1e-14, atol=1e-14)


def test_page_slots_hand_example():
    # P = 4 tokens per page; sequence 0 owns pages 2 then 0, sequence 1 pages 1 then 3:
    # token t sits at slot page * 4 + t % 4 of page table[b][t // 4]
    table = [[2, 0], [1, 3]]
    assert SV.page_slots(table, 4, 0, 7).tolist() == [8, 9, 10, 11, 0, 1, 2]
    assert SV.page_slots(table, 4, 1, 6).tolist() == [4, 5, 6, 7, 12, 13]
