"""The multi-rank logic of bench.py on CPU: two gloo ranks, no GPU.

The path shards without a data-path collective (every rank runs its own
request); the only cross-rank steps are a barrier and the max-reduction of
the step time, which sets the whole-job throughput.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, ms_by_rank, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    dist.barrier()
    ms, value = bench.job_time_and_value(ms_by_rank[rank], 131072, world, lambda x: bench.dist_max(x, "cpu"))
    dist.barrier()
    out[rank] = (ms, value)
    dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank():
    world = 2
    ms_by_rank = [0.40, 0.55]
    with mp.get_context("spawn").Manager() as m:     # no fork after torch's threads start
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), ms_by_rank, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, value = res[r]
        assert ms == pytest.approx(0.55)
        assert value == pytest.approx(world * 131072 / 0.55e-3)


def test_single_rank_needs_no_group():
    import bench
    ms, value = bench.job_time_and_value(0.5, 1000, 1, None)
    assert ms == 0.5 and value == pytest.approx(2e6)


def _rank_leaves(rank, world, port, out):
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=10))
    if rank == 1:
        os._exit(0)                      # leaves between steps, nothing in flight
    import bench
    try:
        bench.dist_max(0.5, "cpu")
        out[rank] = "completed"
    except Exception as e:  # noqa: BLE001 - any error is the expected outcome
        out[rank] = "error: " + type(e).__name__
    os._exit(0)


def test_a_rank_that_leaves_ends_the_others_with_an_error():
    # The surviving rank's step-time reduction must end with an error (peer
    # gone or timeout), not wait for good.
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_leaves, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        alive = [p for p in procs if p.is_alive()]
        for p in alive:
            p.kill()
        assert not alive, "a rank did not finish"
        assert str(out.get(0, "")).startswith("error"), dict(out)
