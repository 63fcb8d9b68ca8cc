"""The multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU)."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        # rank r measured (1 + r, 5 - r, 2): the job takes the slowest rank's time of each
        out = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 2.0], world, torch.device("cpu"))
        torch.distributed.barrier()
        q.put((rank, out))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {0: [2.0, 5.0, 2.0], 1: [2.0, 5.0, 2.0]}


def test_single_rank_and_reference_arm_rank_logic():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([3.0, 1.0], 1, torch.device("cpu")) == [3.0, 1.0]

    class Args:  # only rank 0 runs the oracle arm; the other ranks return without work
        workload = "gqa_decode_llama8b"
        steps = warmup = 3

    assert bench.run_reference(Args(), 1, 2, torch.device("cpu")) is None
