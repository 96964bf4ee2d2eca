"""The multi-GPU path is N independent replicas (tokens are independent
given replicated weights; no collective on the layer's data path). What the
ranks share is host logic: the slowest rank's time (a MAX all-reduce) and
the whole-job throughput. These tests run that logic on two gloo ranks on
the CPU, as the bench does over NCCL."""
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports a step time of 1 + r ms and an end-to-end time of 5 - r ms
        out = bench.max_over_ranks([1.0 + rank, 5.0 - rank], "cpu")
        q.put((rank, out))
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = dict(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert got[0] == got[1] == [2.0, 5.0]


def test_single_process_times_pass_through():
    assert bench.max_over_ranks([3.0, 4.5], "cpu") == [3.0, 4.5]


@pytest.mark.parametrize("world", [1, 2, 8])
def test_replica_throughput_counts_every_rank(world):
    # 2,048 tokens per rank in 0.5 ms (the slowest rank): world x 4.096 M tokens/s
    assert bench.replicas_tokens_per_s(world, 2048, 0.5) == pytest.approx(world * 4.096e6)
