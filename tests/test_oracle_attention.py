"""Pins for oracle.attention and oracle.search: textbook reductions and library routines."""
import math

import numpy as np
from scipy.special import softmax

import tq_inputs as ti
from oracle.attention import decode_attention, exact_attention, softmax_attend
from oracle.codebook import lloyd_max
from oracle import quantizer as Q
from oracle.search import topk


def test_softmax_attend_matches_scipy():
    rng = np.random.Generator(np.random.PCG64(1))
    logits = rng.standard_normal((4, 37)) * 5
    v = rng.standard_normal((37, 16))
    assert np.allclose(softmax_attend(logits, v), softmax(logits, axis=1) @ v, rtol=1e-13, atol=1e-14)


def test_single_token_returns_its_value():
    rng = np.random.Generator(np.random.PCG64(2))
    v = rng.standard_normal((1, 8))
    assert np.allclose(softmax_attend(rng.standard_normal((3, 1)), v), np.repeat(v, 3, axis=0), rtol=0, atol=1e-15)


def test_identical_keys_average_values():
    rng = np.random.Generator(np.random.PCG64(3))
    v = rng.standard_normal((9, 8))
    logits = np.full((2, 9), 1.7)
    assert np.allclose(softmax_attend(logits, v), np.repeat(v.mean(axis=0, keepdims=True), 2, axis=0), atol=1e-14)


def test_gqa_head_mapping():
    """Query head h reads KV head h // (Hq / Hkv): make each KV head's values a constant."""
    B, Hq, Hkv, N, d = 2, 8, 2, 5, 4
    K = np.zeros((B, Hkv, N, d))
    V = np.zeros((B, Hkv, N, d))
    for h in range(Hkv):
        V[:, h] = 10.0 * h + 1.0
    q = np.ones((B, Hq, d))
    out = exact_attention(q, K, V, [N, 3], 0.5)
    for hq in range(Hq):
        assert np.allclose(out[:, hq], 10.0 * (hq // (Hq // Hkv)) + 1.0)


def test_seq_lens_respected():
    B, Hq, Hkv, N, d = 1, 1, 1, 6, 3
    K = np.zeros((B, Hkv, N, d))
    V = np.arange(N, dtype=np.float64)[None, None, :, None] * np.ones((B, Hkv, N, d))
    out = exact_attention(np.zeros((B, Hq, d)), K, V, [4], 1.0)
    assert np.allclose(out, 1.5)                      # mean of 0,1,2,3


def test_fine_quantization_approaches_exact_attention():
    """With many bits the quantized attention converges to exact attention."""
    d, N, G = 64, 256, 4
    rot = ti.haar_rotation(d, 101)
    K = ti.iid_normal((N, d), 102)
    V = ti.iid_normal((N, d), 103)
    q = ti.iid_normal((1, G, d), 104)
    errs = []
    for b in (2, 4, 6):
        c, t, _ = lloyd_max(b, "beta", d=d)
        kq = Q.quantize_mse(K, rot, c, t, b)
        vq = Q.quantize_mse(V, rot, c, t, b)
        vh = Q.dequantize_mse(vq["idx"], vq["norms"], rot, c)
        o = decode_attention(q, [N], 1,
                             lambda bb, h, qs: Q.estimate_mse(qs, rot, kq["idx"], kq["norms"], c),
                             lambda bb, h, n: vh[:n], 1 / math.sqrt(d))
        ref = exact_attention(q, K[None, None], V[None, None], [N], 1 / math.sqrt(d))
        errs.append(np.max(np.abs(o - ref)) / np.max(np.abs(ref)))
    # RMS quantization error falls ~2x per bit (D_b ~ 4^-b): expect ~16x over 4 bits
    assert errs[0] > errs[1] > errs[2]
    assert errs[0] / errs[2] > 8
    assert errs[2] < 0.05


def test_topk_matches_full_sort_with_ties():
    rng = np.random.Generator(np.random.PCG64(5))
    s = np.round(rng.standard_normal((6, 500)), 1)    # many exact ties
    ids, vals = topk(s, 10)
    for i in range(6):
        order = sorted(range(500), key=lambda j: (-s[i, j], j))[:10]
        assert list(ids[i]) == order
        assert np.array_equal(vals[i], s[i, order])
