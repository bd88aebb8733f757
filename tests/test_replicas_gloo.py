"""Replica aggregation over two gloo ranks on the CPU (the multi-GPU bench path
runs the same reduction over NCCL)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from speculative_moe_decoding_b200.replicas import replica_throughput, shard_sequences


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        tokens = [1000.0, 600.0][rank]
        ms = [250.0, 400.0][rank]
        q.put((rank, replica_throughput(tokens, ms), shard_sequences(5, rank, world)))
    finally:
        dist.destroy_process_group()


def test_two_rank_replica_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in procs:
        r, res, shard = q.get(timeout=120)
        out[r] = (res, shard)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        value, ms, tok = out[r][0]
        assert ms == 400.0 and tok == 1600.0
        assert value == pytest.approx(1600.0 / 0.4)
    assert out[0][1] == [0, 2, 4] and out[1][1] == [1, 3]


def test_single_process_is_local():
    assert replica_throughput(100.0, 50.0) == (2000.0, 50.0, 100.0)
