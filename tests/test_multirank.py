"""Host-side logic of the N-GPU bench (independent replicas, weak scaling),
run as 2 gloo ranks on CPU: the max-over-ranks timing reduction, the barrier,
and the per-rank input seeds."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from kv_cache_quantization_hqmq_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
        bench.barrier(dist)
        w = W.WORKLOADS["tiny"]
        x = W.make_call_input(w.with_(input_seed=w.input_seed + 1000 * rank), 0, 0)
        gathered = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        q.put((rank, t, bool(torch.equal(gathered[0], gathered[1]))))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    # every rank sees the slowest rank's time; replicas code different caches
    assert [r[1] for r in res] == [15.0, 15.0]
    assert not res[0][2]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, None, "cpu") == 3.0
    bench.barrier(None)
