"""The multi-rank host path of bench.py (replicas, max over ranks) on CPU with
the gloo backend, world size 2 -- no GPU involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, ret):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from sparse_bit_attention_smoothing_b200.replicas import job_throughput, max_over_ranks, rank_env
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = rank_env()
        assert (r, w, lr) == (rank, world, rank)
        dist.barrier()
        # per-rank device times differ; every rank must see the same maxima
        ms, e2e = 10.0 + 5.0 * rank, 30.0 - 7.0 * rank
        mx = max_over_ranks([ms, e2e])
        ret[rank] = (mx, job_throughput(1.0e12, w, mx[0]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    ret = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, ret)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    expect_ms = max(10.0 + 5.0 * r for r in range(world))
    expect_e2e = max(30.0 - 7.0 * r for r in range(world))
    for r in range(world):
        mx, val = ret[r]
        assert mx == [expect_ms, expect_e2e]
        assert val == pytest.approx(world * 1.0e12 / (expect_ms * 1e-3))


def test_single_process_is_identity():
    from sparse_bit_attention_smoothing_b200.replicas import job_throughput, max_over_ranks
    assert max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert job_throughput(2.0, 1, 1000.0) == pytest.approx(2.0)
    with pytest.raises(ValueError):
        job_throughput(1.0, 1, 0.0)


def _failing_worker(rank, world, port, ret):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        # this rank fails between steps, before the timing collective
        ret[rank] = "left"
        os._exit(3)
    try:
        from sparse_bit_attention_smoothing_b200.replicas import max_over_ranks
        max_over_ranks([1.0])
        ret[rank] = "no error"
    except Exception as e:  # the survivor learns of it through the collective's error
        ret[rank] = "error: " + type(e).__name__
    os._exit(0)


def test_rank_leaving_between_steps_is_reported_to_the_other():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    ret = ctx.Manager().dict()
    procs = [ctx.Process(target=_failing_worker, args=(r, world, port, ret)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert procs[1].exitcode == 3
    assert procs[0].exitcode == 0
    assert ret[0].startswith("error")
