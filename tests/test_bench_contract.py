"""bench.py's reference arm on the host cores: the JSON line it prints (no GPU needed)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                        "--cpu-seconds", "2"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["value"] > 0 and line["higher_is_better"] is True and line["steps"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert "workload" in line["config"]


def test_secondary_workloads_have_no_reference_arm():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "split"], cwd=ROOT,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and "unavailable" in line


class _OracleLib:
    """Stands in for the library on the CPU (the oracle's quantize and estimator), so the
    sweep's glue in bench.py runs without a GPU."""

    class Quantizer:
        def __init__(self, kind, rot, bits, S=None):
            import numpy as np
            from oracle.codebook import lloyd_max
            self.kind, self.rot, self.bits, self.S = kind, np.asarray(rot, dtype=np.float64), bits, S
            d = self.rot.shape[0]
            b = bits if kind == "mse" else bits - 1
            self.c, self.t = lloyd_max(b, "beta", d=d)[:2] if b > 0 else (None, None)

        @classmethod
        def mse(cls, rot, b, device=None):
            return cls("mse", rot, b)

        @classmethod
        def prod(cls, rot, S, b, device=None):
            import numpy as np
            return cls("prod", rot, b, np.asarray(S, dtype=np.float64))

    @staticmethod
    def quantize(q, x):
        from oracle import quantizer as OQ
        x = x.double().numpy()
        if q.kind == "mse":
            return OQ.quantize_mse(x, q.rot, q.c, q.t, q.bits)
        return OQ.quantize_prod(x, q.rot, q.S, q.c, q.t, q.bits)

    @staticmethod
    def score(q, y, rec, n):
        import torch
        from oracle import quantizer as OQ
        y = y.double().numpy()
        if q.kind == "mse":
            e = OQ.estimate_mse(y, q.rot, rec["idx"], rec["norms"], q.c)
        else:
            e = OQ.estimate_prod(y, q.rot, q.S, rec["chat"], rec["s"], rec["norms"], rec["rnorms"])
        return torch.from_numpy(e)


def test_sweep_glue_reproduces_the_crossover_with_the_oracle_as_library():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    rows = bench.ip_sweep(_OracleLib, torch.device("cpu"), n=1500, rho=0.9)
    assert sorted(rows) == [1, 2, 3, 4, 5]
    assert all(rows[b]["prod"]["mean_sq"] < rows[b]["mse"]["mean_sq"] for b in (1, 2, 3))
    assert all(rows[b]["mse"]["mean_sq"] < rows[b]["prod"]["mean_sq"] for b in (4, 5))
    assert rows[1]["mse"]["bias_sq"] > 0.5 * rows[1]["mse"]["mean_sq"]
