"""GPU: tq_decode_attn_fixed_ws (scratch in the library's fixed device array, no
workspace argument) agrees with tq_decode_attn (caller workspace) on two calls in a row.

Collected last so that it also runs after every other GPU test of the session has used
the device.  Both routes run the same kernels, so the comparison uses the decode parity
tolerance of the other decode tests: per (batch, head) row, max |o - o_ref| <= 1e-3 max |o_ref|.
"""
import ctypes as C
import math

import numpy as np
import pytest

import tq_inputs as ti

from _parity import rel_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")
T = K.tq

D = 128
FIXED_BYTES = 8 << 20


def _fixed(kq, vq, q, sl, kc, vc, Nmax, Hkv, out):
    B, Hq, _ = q.shape
    st = T.lib().tq_decode_attn_fixed_ws(kq.ref, vq.ref, q.data_ptr(), T._dtype_code(q), B, Hq, Hkv, Nmax,
                                         sl.data_ptr(), kc.as_c(), vc.as_c(), C.c_float(1.0 / math.sqrt(D)),
                                         out.data_ptr(), None)
    assert st == 0, T.lib().tq_last_error().decode()
    return out


CASES = [
    # name, B, Hq, Hkv, Nmax, seq_lens, key kind, key bits, value bits
    ("small-mse", 2, 8, 2, 3000, [3000, 1777], "mse", 4, 4),
    ("small-prod", 1, 32, 8, 1100, [1100], "prod", 3, 3),
    ("ctx128k", 8, 32, 8, 131072, [131072, 131072, 100000, 77777, 131072, 65536, 1, 131072], "mse", 4, 4),
]


@pytest.mark.parametrize("name,B,Hq,Hkv,Nmax,seq_lens,kk,bk,bv", CASES, ids=[c[0] for c in CASES])
def test_fixed_scratch_matches_workspace_call(name, B, Hq, Hkv, Nmax, seq_lens, kk, bk, bv):
    seed = sum(ord(ch) for ch in name) % 97
    rot = ti.haar_rotation(D, 1002)
    S = ti.gaussian_matrix(D, D, 2002)
    U = ti.haar_rotation(D, 3000 + seed).astype(np.float64)
    n = B * Hkv * Nmax
    kx = ti.anisotropic_torch(n, D, U, 4000 + seed, "cuda")
    vx = ti.anisotropic_torch(n, D, U, 5000 + seed, "cuda")
    q = ti.normal_torch((B, Hq, D), 6000 + seed, "cuda", torch.bfloat16)
    kq = K.Quantizer.prod(rot, S, bk) if kk == "prod" else K.Quantizer.mse(rot, bk)
    vq = K.Quantizer.mse(rot, bv)
    assert K.decode_workspace_bytes(kq, B, Hq, Hkv, Nmax) <= FIXED_BYTES
    kc, vc = K.quantize(kq, kx), K.quantize(vq, vx)
    del kx, vx
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    ref = K.decode_attn(kq, vq, q, sl, kc, vc, Nmax, Hkv).cpu().numpy()
    B_, Hq_, _ = q.shape
    outs = [torch.full((B_, Hq_, D), float("nan"), dtype=torch.float32, device=q.device) for _ in range(2)]
    torch.cuda.synchronize()
    for i in range(2):
        if i == 1:
            # the first call did the address lookup; from here on neither the driver's view
            # of free device memory nor torch's allocator may move
            free0, _ = torch.cuda.mem_get_info()
            torch0 = torch.cuda.memory_allocated()
        _fixed(kq, vq, q, sl, kc, vc, Nmax, Hkv, outs[i])
        torch.cuda.synchronize()
        if i == 1:
            assert torch.cuda.mem_get_info()[0] == free0
            assert torch.cuda.memory_allocated() == torch0
        assert K.get_status() == 0
        o = outs[i].cpu().numpy()
        assert np.all(np.isfinite(o))
        err = rel_rows(o, ref)
        assert np.all(err <= 1e-3), f"max row error {err.max():.3e}"


def test_fixed_scratch_rejects_oversize_shape():
    rot = ti.haar_rotation(D, 1002)
    kq = K.Quantizer.mse(rot, 4)
    vq = K.Quantizer.mse(rot, 4)
    B, Hq, Hkv, Nmax = 64, 64, 8, 1 << 20
    assert K.decode_workspace_bytes(kq, B, Hq, Hkv, Nmax) > FIXED_BYTES
    FAKE = 0x10000   # rejected on size before any pointer is touched
    pk = T.Packed_t(FAKE, None, FAKE, None)
    st = T.lib().tq_decode_attn_fixed_ws(kq.ref, vq.ref, FAKE, T.BF16, B, Hq, Hkv, Nmax, FAKE, pk, pk,
                                         C.c_float(0.1), FAKE, None)
    assert st == 8
    assert b"fixed array" in T.lib().tq_last_error()


def test_fixed_scratch_checks_shape_before_size():
    """A bad shape gets tq_decode_attn's status even when its scratch would not fit."""
    rot = ti.haar_rotation(D, 1002)
    kq = K.Quantizer.mse(rot, 4)
    vq = K.Quantizer.mse(rot, 4)
    FAKE = 0x10000   # refused before any pointer is touched
    pk = T.Packed_t(FAKE, None, FAKE, None)
    st = T.lib().tq_decode_attn_fixed_ws(kq.ref, vq.ref, FAKE, T.BF16, 64, 60, 8, 1 << 20, FAKE, pk, pk,
                                         C.c_float(0.1), FAKE, None)
    assert st == 1                       # Hq not a multiple of Hkv: TQ_ERR_INVALID_ARG
