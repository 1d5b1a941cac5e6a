"""The multi-GPU path of bench.py, exercised with world-size-2 gloo ranks on CPU.

The layer forward has no exchange step on one GPU, so N GPUs run N
independent replicas ("replicas only"): the only cross-rank work is the
barrier around the timed region and the max-over-ranks of the step time.
These tests run exactly that host logic in two processes over gloo.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, per_rank_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.rank_env()
        assert (w, r, lr) == (world, rank, rank)
        dist.barrier()
        slowest = bench.reduce_max_over_ranks(per_rank_ms[rank], world, "cpu")
        out.put((rank, slowest, bench.job_throughput(4096, world, slowest)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("per_rank_ms", [[1.0, 3.0], [2.5, 0.5]])
def test_two_gloo_ranks_report_the_slowest_rank(per_rank_ms):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, per_rank_ms, out))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    results = sorted(out.get(timeout=10) for _ in range(2))
    want = max(per_rank_ms)
    for rank, slowest, tput in results:
        assert slowest == want
        assert tput == pytest.approx(2 * 4096 / (want / 1e3))


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.reduce_max_over_ranks(1.25, 1, "cpu") == 1.25
    assert bench.job_throughput(4096, 1, 1.0) == pytest.approx(4.096e6)
