"""Multi-rank host logic on CPU (gloo, world size 2): no GPU needed.

The path shards over independent sequences with no exchange on the data path: each
rank solves its own batch of the same shape (weak scaling), and the job's step time
is the max over ranks.  This checks the rank sharding and the max reduction.
"""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import oracle
    from nonlinear_rnn_solve_b200 import workloads as wl
    w = bench.rank_workload(wl.WORKLOADS["gru_b1_t1024_in4_h8"].resized(T=128), rank, world)
    inp = wl.generate(w)
    m = oracle.model_from_inputs("gru", inp)
    h, iters, _ = m.newton(inp["h0"], max_iters=w.T, tol=w.tol)
    err = float(np.abs(h - m.rollout(inp["h0"])).max())
    t = bench.max_over_ranks([1.0 + rank, 5.0 - rank])
    out[rank] = (w.seed, float(inp["x"].sum()), err, t)
    dist.destroy_process_group()


def test_two_ranks_shard_and_reduce():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    (s0, x0, e0, t0), (s1, x1, e1, t1) = out[0], out[1]
    assert s0 != s1 and x0 != x1          # independent sequences per rank
    assert e0 < 1e-9 and e1 < 1e-9        # each rank's solve is its rollout
    assert t0 == t1 == [2.0, 5.0]         # max over ranks, seen by every rank
