"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing its own
independent problem; the step time is the max over ranks and the throughput
sums every rank's tokens.  No GPU needed."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, ms_by_rank, tokens, out):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms, value = bench.reduce_over_ranks(ms_by_rank[rank], tokens, world)
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_summed_tokens():
    world, tokens = 2, 1_965_600.0          # 2 x 32760 x 30 block-tokens per rank
    ms_by_rank = [500.0, 620.0]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, world, port, ms_by_rank, tokens, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs)
        for r in range(world):
            ms, value = out[r]
            assert ms == 620.0                                   # slowest rank decides
            assert value == pytest.approx(world * tokens / 0.620)


def test_single_rank_is_local():
    import bench
    ms, value = bench.reduce_over_ranks(400.0, 1000.0, 1)
    assert ms == 400.0 and value == pytest.approx(2500.0)
