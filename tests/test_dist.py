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


def test_clock_sampler_selects_the_process_gpu():
    """nvidia-smi numbers every GPU; CUDA numbers those in
    CUDA_VISIBLE_DEVICES.  The sampler must query the GPU the process uses."""
    import bench
    assert bench.smi_gpu_id(0, visible=None) == "0" or "CUDA_VISIBLE_DEVICES" in os.environ
    assert bench.smi_gpu_id(0, visible="") == "0"
    assert bench.smi_gpu_id(0, visible="5") == "5"
    assert bench.smi_gpu_id(1, visible="3, 6") == "6"
    assert bench.smi_gpu_id(0, visible="GPU-8a1c2f3e-aaaa-bbbb-cccc-0123456789ab") == \
        "GPU-8a1c2f3e-aaaa-bbbb-cccc-0123456789ab"
    assert bench.smi_gpu_id(2, visible="4") == "2"          # out of range: as given


def test_keep_busy_alternates_and_syncs():
    """The untimed load around the timed region: about the asked wall time,
    an even number of calls (so step(0) follows a call on the other input
    set), and a wait for the device every 8 calls and at the end."""
    import time
    import bench
    calls, syncs = [], []

    def step(i):
        calls.append(i)
        time.sleep(0.001)

    t0 = time.perf_counter()
    n = bench.keep_busy(step, 0.05, lambda: syncs.append(len(calls)))
    assert time.perf_counter() - t0 >= 0.05
    assert n == len(calls) and n % 2 == 0 and calls == list(range(n))
    assert calls[-1] % 2 == 1
    assert syncs[-1] == n and all(c % 8 == 0 for c in syncs[:-1])
    calls.clear()
    assert bench.keep_busy(step, 0.0, lambda: None) == 0 and calls == []
    n = bench.keep_busy(step, 0.01, lambda: None, first=5)
    assert n >= 2 and n % 2 == 0 and calls == list(range(5, 5 + n))
