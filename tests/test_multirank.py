"""The multi-rank plumbing of bench.py on CPU: two gloo ranks.

The decode shards by batch (sequences are independent), so ranks exchange
nothing but the timing: the whole-job rate is all ranks' bytes over the
slowest rank's time."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        dist.barrier()
        slowest = bench.max_over_ranks(times[rank], torch.device("cpu"))
        gbs, tfs = bench.whole_job_rates(1_000_000_000, 2_000_000_000_000, world, slowest)
        out.put((rank, slowest, gbs, tfs))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    times = [2.0, 5.0]                                  # ms per step on rank 0, rank 1
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, slowest, gbs, tfs in res:
        assert slowest == 5.0                           # max over ranks, on every rank
        assert gbs == pytest.approx(2 * 1e9 / 5e-3 / 1e9)   # both ranks' bytes / slowest time
        assert tfs == pytest.approx(2 * 2e12 / 5e-3 / 1e12)


def test_single_rank_rates():
    sys.path.insert(0, ROOT)
    import bench
    gbs, tfs = bench.whole_job_rates(604_000_000, 18_000_000_000, 1, 0.125)
    assert gbs == pytest.approx(4832.0)
    assert tfs == pytest.approx(144.0)
