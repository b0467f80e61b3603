"""The head-sharded split on CPU: two gloo ranks each run their range of KV
heads and all-gather O. The per-head step here is the oracle (this test runs
without a GPU); the GPU test of the same split is tests/test_gpu_shard.py.
What is checked is the host logic: the head ranges cover every head once, the
thresholds follow their heads, and the gather puts every head back in place."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_score_b200.shard import kv_head_range, run_heads


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


B, S = 16, 4


def _problem():
    g = torch.Generator().manual_seed(7)
    b, hq, hkv, L, d = 2, 6, 3, 64, 8
    Q = torch.randn(b, hq, L, d, generator=g, dtype=torch.float64)
    K = torch.randn(b, hkv, L, d, generator=g, dtype=torch.float64)
    V = torch.randn(b, hkv, L, d, generator=g, dtype=torch.float64)
    K[:, 1] *= 2.0
    tau = [0.5, 0.6, 0.7, 0.8, 0.9, 0.95]
    return Q, K, V, tau


def _oracle_step(q, k, v, t, o):
    """One batch-1 head range through the oracle: P, find_blocks, attention."""
    import oracle.xattn_oracle as O
    P = O.block_probs(q, k, B, S, True)
    _, lists = O.select_blocks(P, list(t), True)
    Os, _ = O.sparse_attention(q, k, v, B, True, lists)
    o.copy_(torch.from_numpy(Os))


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from block_sparse_long_score_b200.shard import gather_heads
    try:
        Q, K, V, tau = _problem()
        kv0, kv1 = kv_head_range(rank, world, K.shape[1])
        O_local = run_heads(_oracle_step, Q, K, V, tau, kv0, kv1)
        full = gather_heads(O_local, Q.shape[1], K.shape[1])
        q.put((rank, kv0, kv1, full.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_split_matches_the_whole_layer():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, qu)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(qu.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [(r[1], r[2]) for r in res] == [(0, 2), (2, 3)]   # 3 KV heads over 2 ranks
    Q, K, V, tau = _problem()
    whole = run_heads(_oracle_step, Q, K, V, tau, 0, K.shape[1]).numpy()
    for r in res:
        np.testing.assert_array_equal(r[3], whole)           # every rank holds all heads


@pytest.mark.parametrize("hkv,world", [(8, 1), (8, 2), (8, 3), (8, 8), (3, 5), (1, 2)])
def test_kv_head_ranges_cover_every_head_once(hkv, world):
    ranges = [kv_head_range(r, world, hkv) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == hkv
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0 and a0 <= a1
    sizes = [k1 - k0 for k0, k1 in ranges]
    assert max(sizes) - min(sizes) <= 1
