"""Host logic of the multi-GPU bench path, as two gloo ranks on CPU.

With N GPUs every rank runs the same per-GPU workload on its own batch (weak scaling, no
collective on the data path).  The only cross-rank steps are a barrier and the max of the
per-rank device times, from which rank 0 reports whole-job throughput.
"""
import datetime
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        m = bench.max_over_ranks(times[rank], torch.device("cpu"))
        v = bench.weak_scaling_value(world, 1.0e9, m)
        out.put((rank, m, v, bench.rank_seed_offset(rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_aggregate():
    world, port = 2, _free_port()
    times = [3.0, 5.0]                       # per-rank ms per step
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    # every rank sees the slowest rank's time; the job moved 2 x 1 GB in 5 ms
    assert [r[1] for r in res] == [5.0, 5.0]
    assert all(abs(r[2] - 2 * 1.0e9 / 5e-3 / 1e9) < 1e-9 for r in res)
    # each rank draws its own batch
    assert res[0][3] != res[1][3]


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.25, torch.device("cpu")) == 4.25
    assert abs(bench.weak_scaling_value(1, 5.0e9, 2.0) - 2500.0) < 1e-9
