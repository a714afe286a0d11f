"""Multi-rank host logic on CPU: world_size 2 over gloo (127.0.0.1)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from paged_kv_cache_439_b200 import dist as pdist
from paged_kv_cache_439_b200.workloads import make_custom


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each replica draws its own batch of the same shape
        wl = make_custom("r", [40, 17], 4, 2, 64, 16, "bf16", seed=pdist.replica_seed(5, rank))
        fingerprint = float(wl.q.float().sum())
        # per-rank "device time": rank 1 is the slowest
        my_ms = 10.0 + 5.0 * rank
        dist.barrier()
        mx = pdist.max_over_ranks(my_ms)
        rate = pdist.whole_job_rate(wl.kv_bytes(), 100, world, mx)
        q.put((rank, fingerprint, mx, rate, wl.kv_bytes()))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_max_timing():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    # both ranks see the slowest rank's time
    assert res[0][2] == res[1][2] == 15.0
    # same shape, different data per replica
    assert res[0][4] == res[1][4]
    assert res[0][1] != res[1][1]
    # whole-job rate: all ranks' bytes over the max time
    kv = res[0][4]
    assert res[0][3] == pytest.approx(kv * 100 * 2 / 0.015 / 1e9)


def test_single_process_identity():
    assert pdist.max_over_ranks(3.5) == 3.5
    with pytest.raises(ValueError):
        pdist.whole_job_rate(1, 1, 1, 0.0)
