"""The multi-GPU replica plumbing (rank parsing, barrier, max over ranks) with
world_size 2 on the CPU (gloo)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from padding_free_moe_b200 import replicas


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    info = replicas.rank_info()
    replicas.init(info, "gloo", timeout_s=60)
    replicas.barrier(info)
    # each replica "timed" a different duration; everyone must agree on the slowest
    got = replicas.max_over_ranks(10.0 + 5.0 * rank, info)
    replicas.barrier(info)
    replicas.finish(info)
    q.put((rank, got))


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 15.0, 1: 15.0}


def test_single_process_is_passthrough():
    info = replicas.RankInfo(0, 1, 0)
    assert replicas.max_over_ranks(3.5, info) == 3.5
    replicas.barrier(info)        # no process group needed
    replicas.finish(info)


def test_rank_env_and_gpu_index():
    info = replicas.rank_info({"RANK": "3", "WORLD_SIZE": "8", "LOCAL_RANK": "3"})
    assert (info.rank, info.world, info.local_rank) == (3, 8, 3)
    assert replicas.physical_gpu_index(1, {"CUDA_VISIBLE_DEVICES": "4,5,6"}) == 5
    assert replicas.physical_gpu_index(2, {}) == 2
    assert replicas.physical_gpu_index(0, {"CUDA_VISIBLE_DEVICES": "GPU-abc"}) == 0
