"""Multi-rank host logic of bench.py on CPU: two gloo ranks, replicas, max-over-ranks timing."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms_by_rank, out):
    import torch.distributed as dist

    from joint_attention_block_b200 import replicas

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        replicas.barrier()
        value, ms = replicas.job_throughput(4608.0 * 10, ms_by_rank[rank])
        out.put((rank, value, ms))
        replicas.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    world, port = 2, _free_port()
    ms_by_rank = [20.0, 25.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, ms_by_rank, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, value, ms in res:
        assert ms == 25.0  # max over ranks
        assert value == pytest.approx(4608.0 * 10 * 2 / 0.025)  # units of both ranks / slowest time


def test_single_process_is_identity():
    from joint_attention_block_b200 import replicas

    value, ms = replicas.job_throughput(100.0, 50.0)
    assert ms == 50.0 and value == pytest.approx(2000.0)
