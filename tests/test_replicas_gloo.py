"""The multi-rank host logic of bench.py on CPU: two gloo ranks, barrier, and
the max-over-ranks timing reduction. The path itself has no collective."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        dist.barrier()
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms)
        q.put((rank, m, bench.whole_job_ms_per_layer(m, world)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_timing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [r[1] for r in res] == [15.0, 15.0]     # every rank sees the max
    assert [r[2] for r in res] == [7.5, 7.5]       # two layers per 15 ms step


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_ms_per_layer(8.0, 1) == 8.0


def test_head_split_host_logic():
    """--split heads: each rank keeps its KV-head range of the same layer (with
    the query heads and thresholds of those heads), and a layer takes the
    slowest rank's step instead of being one of `world` replicas."""
    import bench
    from block_sparse_long_score_b200.synth import make_problem
    prob = make_problem("c1", L=1024, hq=8, hkv=4)
    parts = [bench.local_heads(prob, r, 3) for r in range(3)]
    assert [(p.hq, p.hkv) for p in parts] == [(4, 2), (2, 1), (2, 1)]
    assert torch.equal(torch.cat([p.Q for p in parts], dim=1), prob.Q)
    assert torch.equal(torch.cat([p.K for p in parts], dim=1), prob.K)
    assert torch.equal(torch.cat([p.V for p in parts], dim=1), prob.V)
    assert list(np.concatenate([p.tau for p in parts])) == list(prob.tau)
    assert all(p.Q.is_contiguous() and p.K.is_contiguous() for p in parts)
    assert bench.whole_job_ms_per_layer(12.0, 4, "heads") == 12.0
    assert bench.whole_job_ms_per_layer(12.0, 4, "replicas") == 3.0
