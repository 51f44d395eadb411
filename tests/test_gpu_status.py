"""Device-side bounded waits: a host-set limit makes every bounded wait of the tensor-core
quantize and of the decode kernel expire, the status word reports TQ_ERR_TIMEOUT on every
such launch, and the next call on the same context is correct.

The timeout comes from the host-set limit only (TQ_WAIT_EXPIRE_AT_ONCE: each wait gives up
before its first poll); the kernels drain the copies they issued, free their tensor memory
and exit.  Nothing faults or hangs.
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

EXPIRE_AT_ONCE = -1
TIMEOUT = 6


def _expired(fn):
    """Run fn with every bounded wait expiring at once; return the status it left."""
    assert K.get_status() == 0
    K.set_wait_limit(EXPIRE_AT_ONCE)
    try:
        fn()
        st = K.get_status()
    finally:
        K.set_wait_limit(0)
    return st


def test_quantize_wait_timeout_is_reported_and_recovers():
    d, n, b = 128, 128 * 600, 4
    rot = ti.haar_rotation(d, 1003)
    xt, x64 = ti.to_bf16_f64(ti.iid_normal((n, d), 4003))
    xt = xt.cuda()
    q = K.Quantizer.mse(rot, b)
    for _ in range(2):                       # deterministic: every launch times out
        assert _expired(lambda: K.quantize(q, xt)) == TIMEOUT
    assert K.get_status() == 0               # reading the status cleared it
    out = K.quantize(q, xt)
    assert K.get_status() == 0
    c, t, _ = lloyd_max(b, "beta", d=d)
    ref = OQ.quantize_mse(x64, rot, c, t, b)
    bad, _, _ = code_mismatches(as_u32(out.codes), ref["codes"], d, b, ref["y"], t)
    assert bad == 0


def test_decode_wait_timeout_is_reported_and_recovers():
    D, B, Hq, Hkv, N, b = 128, 2, 8, 2, 2000, 4
    rot = ti.haar_rotation(D, 1007)
    U = ti.haar_rotation(D, 3007).astype(np.float64)
    kt, k64 = ti.to_bf16_f64(ti.anisotropic(B * Hkv * N, D, U, 4007))
    vt, v64 = ti.to_bf16_f64(ti.anisotropic(B * Hkv * N, D, U, 5007))
    qt, q64 = ti.to_bf16_f64(ti.iid_normal((B * Hq, D), 6007))
    kq, vq = K.Quantizer.mse(rot, b), K.Quantizer.mse(rot, b)
    c, t, _ = lloyd_max(b, "beta", d=D)
    ok = OQ.quantize_mse(k64, rot, c, t, b)
    ov = OQ.quantize_mse(v64, rot, c, t, b)
    dev = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).astype(dt)).cuda()
    kc = K.Packed(dev(ok["codes"].view(np.int32), np.int32), None, dev(ok["norms"], np.float32))
    vc = K.Packed(dev(ov["codes"].view(np.int32), np.int32), None, dev(ov["norms"], np.float32))
    seq = torch.tensor([N, 1234], dtype=torch.int32, device="cuda")
    q = qt.reshape(B, Hq, D).cuda()
    for _ in range(2):
        assert _expired(lambda: K.decode_attn(kq, vq, q, seq, kc, vc, N, Hkv)) == TIMEOUT
    out = K.decode_attn(kq, vq, q, seq, kc, vc, N, Hkv).cpu().numpy()
    assert K.get_status() == 0
    vh = OQ.dequantize_mse(ov["idx"], ov["norms"], rot, c)
    rows = lambda bb, h, n: slice((bb * Hkv + h) * N, (bb * Hkv + h) * N + n)
    ref = decode_attention(q64.reshape(B, Hq, D), [N, 1234], Hkv,
                           lambda bb, h, qs: OQ.estimate_mse(qs, rot, ok["idx"][rows(bb, h, N)],
                                                             ok["norms"][rows(bb, h, N)], c),
                           lambda bb, h, n: vh[rows(bb, h, n)], 1.0 / math.sqrt(D))
    assert np.all(rel_rows(out, ref) <= 1e-3)

