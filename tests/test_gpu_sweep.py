"""GPU: the inner-product distortion sweep (TurboQuant review, Figure 3(a)) through the
library: quantize with tq_quantize_mse / tq_quantize_prod and estimate with tq_score, for
b = 1..5 bits, on unit keys x and queries y = rho x + sqrt(1 - rho^2) z correlated with them.

Per pair, the GPU estimate <y, x_hat> equals the oracle's estimate on the GPU's
band-checked records to 1e-3 (unit vectors); the per-width mean squared error and squared
bias then agree with the oracle's own sweep, and both put the crossover where the caption
does: prod better through 3 bits, mse above.
"""
import json
import os

import numpy as np
import pytest

import tq_inputs as ti
from oracle import quantizer as OQ
from oracle.codebook import lloyd_max
from oracle.sweep import correlated_pairs, sweep

from _parity import adopt_mse, adopt_prod, as_u32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

K = pytest.importorskip("kv_cache_compression_rotation_b200")

D, NP, RHO = 128, 4096, 0.9


def test_ip_distortion_sweep_matches_oracle(golden_dir):
    x = ti.unit_gaussian(NP, D, 4009).astype(np.float32).astype(np.float64)
    z = ti.unit_gaussian(NP, D, 6009)
    y = correlated_pairs(x, z, RHO).astype(np.float32).astype(np.float64)
    rot = ti.haar_rotation(D, 1009)
    S = ti.gaussian_matrix(D, D, 2009)
    books = {b: lloyd_max(b, "beta", d=D)[:2] for b in range(1, 6)}
    xt = torch.from_numpy(x.astype(np.float32)).cuda()
    yt = torch.from_numpy(y.astype(np.float32)).cuda()
    exact = np.sum(x * y, axis=1)
    gpu = {"mse": {}, "prod": {}}
    for b in range(1, 6):
        for kind in ("mse", "prod"):
            q = K.Quantizer.mse(rot, b) if kind == "mse" else K.Quantizer.prod(rot, S, b)
            pk = K.quantize(q, xt)
            est = K.score(q, yt, pk, NP).diagonal().double().cpu().numpy()
            assert K.get_status() == 0
            if kind == "mse":
                c, t = books[b]
                ref = OQ.quantize_mse(x, rot, c, t, b)
                idx, _ = adopt_mse(as_u32(pk.codes), ref, b, t)
                xh = OQ.dequantize_mse(idx, ref["norms"], rot, c)
            else:
                c, t = books[b - 1] if b > 1 else (None, None)
                ref = OQ.quantize_prod(x, rot, S, c, t, b)
                a = adopt_prod(as_u32(pk.codes) if b > 1 else None, as_u32(pk.signs), pk.rnorms.cpu().numpy(),
                               ref, b, c, t, S)
                xh = OQ.dequantize_prod(a["chat"], a["s"], ref["norms"], a["rnorms"], rot, S)
            assert np.max(np.abs(est - np.sum(xh * y, axis=1))) <= 1e-3
            e = est - exact
            gpu[kind][b] = (float(np.mean(e * e)), float(np.mean(e) ** 2))
    ref = sweep(x, y, range(1, 6), rot, S, books)
    for kind in ("mse", "prod"):
        for b in range(1, 6):
            assert abs(gpu[kind][b][0] - ref[kind][b][0]) <= 0.02 * ref[kind][b][0] + 1e-7
    g = json.load(open(os.path.join(golden_dir, "pages_printed.json")))["ip_distortion_crossover"]
    for res in (gpu, ref):
        wins = [b for b in range(1, 6) if res["prod"][b][0] < res["mse"][b][0]]
        assert wins == list(range(1, g["crossover_bits"] + 1))
