"""Multi-rank host logic of the benchmark on CPU with the gloo backend (world size 2).

Replicas run independent prefills (one prompt per rank): no collective touches the
data path; the ranks only agree on the slowest rank's time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from learned_token_pruning_tg_b200 import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 5.5][rank]                       # rank 1 is the slower replica
        ms_max = bench.reduce_max(ms, torch.device("cpu"))
        seed = bench.replica_seed(synth.L128K, rank)
        q.put((rank, ms_max, seed, bench.job_throughput(1000, world, ms_max)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [5.5, 5.5]                  # max over ranks on both
    assert res[0][2] != res[1][2]                             # each replica has its own prompt
    assert res[0][3] == pytest.approx(1000 * 2 / 5.5e-3)      # whole-job tokens/s


def test_single_process_reduce_is_identity():
    assert bench.reduce_max(4.25, torch.device("cpu")) == 4.25
