"""The N > 1 bench path on CPU: two gloo ranks, each with its own replica, the
slowest rank's time decides, and throughput counts the units of all ranks.
The DSA path has no data-path collective (sequences are independent), so
only the timing reduction is exercised here."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from synth import get_workload, make_inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # each rank draws its own replica (seed + rank) of a small workload
        inp = make_inputs(get_workload("decode_b32_ctx128k", B=2, L=300), seed=rank, device="cpu")
        local_ms = 10.0 * (rank + 1)                  # rank 1 is the slow one
        total = bench.reduce_over_ranks(local_ms, world, dist, "cpu")
        v = bench.job_throughput(inp.Q, world, 5, total)
        digest = int(inp.indexer[0]["k_idx"][:64].to(torch.int64).sum())
        q.put((rank, total, v, digest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank_and_all_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res[0][1] == res[1][1] == 20.0             # max over ranks
    assert res[0][2] == pytest.approx(2 * 2 * 5 / 0.020)   # Q=2 per rank, 2 ranks, 5 steps
    assert res[0][3] != res[1][3]                     # replicas are drawn independently


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.reduce_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(32, 1, 10, 2.0) == pytest.approx(160000.0)
