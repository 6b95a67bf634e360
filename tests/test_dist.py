"""Multi-rank host logic of bench.py on CPU: world_size 2 over gloo."""
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


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, w, l = bench.dist_env()
        t = bench.max_over_ranks(10.0 + 5.0 * rank)
        bench.barrier()
        q.put((rank, r, w, t, bench.rank_seed(1002, rank)))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[0] for g in got] == [0, 1] and [g[1] for g in got] == [0, 1]
    assert all(g[2] == 2 for g in got)
    assert all(g[3] == 15.0 for g in got)          # max over ranks, on every rank
    assert got[0][4] != got[1][4]                  # independent batch per rank


def test_alg_accounting():
    import bench
    # per token-head: q, k, g, v, beta, o in bf16
    assert bench.prefill_alg_bytes(1, 1, 1, 128, 128, False, False) == (3 * 128 + 128 + 1 + 128) * 2
    b = bench.decode_alg_bytes(256, 32, 128, 128)
    assert b == 256 * 32 * 132354
