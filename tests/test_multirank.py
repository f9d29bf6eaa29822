"""The multi-process path of bench.py on CPU: two gloo ranks.

bench.py runs one independent replica per GPU (the layer shards by tokens
with no exchange); the only cross-rank steps are the barrier and the max over
ranks of the device timings.  These run here with the gloo backend.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    times = [1.0 + rank, 5.0 - rank, 2.0 * (rank + 1)]
    got = bench.reduce_max_over_ranks(times)
    dist.barrier()
    out[rank] = got
    dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert out[0] == out[1] == [2.0, 5.0, 4.0]


def test_whole_job_rate_counts_every_rank():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    # 105 tokens per step on each of 4 ranks, slowest rank 2 ms -> 210000 tokens/s
    assert bench.whole_job_rate(105, 4, 2.0) == pytest.approx(210000.0)
    assert bench.reduce_max_over_ranks([3.0, 1.5]) == [3.0, 1.5]
