"""The benchmark's multi-process plumbing (rank layout, barrier, max over
ranks, per-rank batches) on 2 CPU ranks with the gloo backend."""
import os
import socket

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    import bench
    import workloads as W
    r, wsz, local = bench.dist_env()
    on = bench.init_dist("gloo", wsz)
    bench.barrier(on, torch.device("cpu"))
    m = bench.max_over_ranks(10.0 * (rank + 1), on, torch.device("cpu"))
    w = bench.rank_workload(W.WORKLOADS["llama7b"], rank)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, wsz, on, m, w.seed, w.B, w.Hkv))


def test_two_rank_plumbing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    ps = [ctx.Process(target=worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, on0, m0, s0, b0, h0), (r1, w1, on1, m1, s1, b1, h1) = res
    assert (r0, r1, w0, w1, on0, on1) == (0, 1, 2, 2, True, True)
    assert m0 == m1 == 20.0                      # max over ranks seen by both
    assert s0 != s1 and (b0, h0) == (b1, h1)     # own batch, same shapes


def test_single_process_is_not_distributed():
    import bench
    assert bench.init_dist("gloo", 1) is False
    assert bench.max_over_ranks(3.0, False, None) == 3.0
