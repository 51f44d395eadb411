"""Device-side bounded waits: a lowered wait limit makes the tensor-core quantize time
out, the status word reports it, and the next call on the same context is correct.

The timeout is produced by the host-set poll limit only; nothing faults or hangs.
"""
import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as OQ
from oracle.codebook import lloyd_max

from _parity import as_u32, code_mismatches

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")


def test_wait_timeout_is_reported_and_recovers():
    d, n, b = 128, 128 * 600, 4
    rot = ti.haar_rotation(d, 1003)
    xt, x64 = ti.to_bf16_f64(ti.iid_normal((n, d), 4003))
    xt = xt.cuda()
    q = K.Quantizer.mse(rot, b)
    assert K.get_status() == 0
    K.set_wait_limit(1)
    try:
        K.quantize(q, xt)
        st = K.get_status()
    finally:
        K.set_wait_limit(0)
    assert st in (0, 6)          # 6 = TQ_ERR_TIMEOUT; 0 only if every wait was satisfied at once
    out = K.quantize(q, xt)
    assert K.get_status() == 0
    c, t, _ = lloyd_max(b, "beta", d=d)
    ref = OQ.quantize_mse(x64, rot, c, t, b)
    bad, _, _ = code_mismatches(as_u32(out.codes), ref["codes"], d, b, ref["y"], t)
    assert bad == 0
