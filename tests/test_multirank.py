"""The multi-GPU path's host logic on CPU: two gloo ranks.

bench.py runs one process per GPU, each on its own independent memories (no collective
on the data path); the job's time is the slowest rank's and its throughput counts every
rank's tokens.  Here two ranks on 127.0.0.1 exercise exactly those helpers.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from sparse_weight_memory_chunk_b200.inputs import WORKLOADS, gen_qvg
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [2.5, 3.25][rank]
        ms = bench.max_over_ranks(local_ms, world, "cpu")
        w = bench.rank_workload(WORKLOADS[1], rank)
        q, _, _ = gen_qvg(w, M=1, T=4)
        out.put((rank, ms, bench.job_throughput(1000, world, ms), w.seed, q.tobytes()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_time_and_inputs():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, ms, thr, seed, qb = out.get(timeout=120)
        res[r] = (ms, thr, seed, qb)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks report the slowest rank's time, and the job counts both ranks' tokens
    assert res[0][0] == res[1][0] == 3.25
    assert np.isclose(res[0][1], 2 * 1000 / 3.25e-3)
    # rank 0 is the workload itself; rank 1 draws other sequences
    from sparse_weight_memory_chunk_b200.inputs import WORKLOADS
    assert res[0][2] == WORKLOADS[1].seed and res[1][2] != res[0][2]
    assert res[0][3] != res[1][3]


def test_single_rank_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.5, 1, "cpu") == 1.5
    assert bench.job_throughput(4096 * 4, 1, 2.0) == 4096 * 4 / 2e-3
