"""The multi-GPU path of bench.py is independent replicas: each rank times its
own batch and the job's time is the slowest rank.  This runs that aggregation
with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        mine = 10.0 + 5.0 * rank                 # rank 1 is the slow replica
        t = bench.max_over_ranks(mine, dist)
        dist.barrier()
        q.put((rank, t))
    finally:
        dist.destroy_process_group()


def test_replica_time_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(3.5, None) == 3.5


# ---------------------------------------------------------------------------
# Sequence parallelism (learned_token_group_b200.ulysses) with two gloo ranks:
# the CPU oracle stands in for the kernels on each rank, so the test checks the
# exchange itself (routing gathered, heads all-to-all and back) against the
# oracle's single-process block.
# ---------------------------------------------------------------------------
class _OracleOps:
    @staticmethod
    def route(x, W_r, b_r, M):
        import numpy as np
        import oracle
        gid, gate, _ = oracle.route(x.numpy(), W_r.numpy(), None if b_r is None else b_r.numpy())
        return torch.from_numpy(gid.astype(np.int32)), torch.from_numpy(gate)

    @staticmethod
    def block(q, k, v, group_id, gate, M, grid=None, window=None):
        import oracle
        out = oracle.group_attention(q.numpy(), k.numpy(), v.numpy(), group_id.numpy(), gate.numpy(), M)
        if window:
            out = 0.5 * (out + oracle.stga_attention(q.numpy(), k.numpy(), v.numpy(), *grid, window))
        return torch.from_numpy(out)


def _ulysses_worker(rank, world, port, q, case):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from learned_token_group_b200.ulysses import ulysses_layer
        x, W, q_, k_, v_, M, grid, window = case
        n = x.shape[0] // world
        sl = slice(rank * n, (rank + 1) * n)
        out, gid, gate = ulysses_layer(x[sl], W, None, q_[sl], k_[sl], v_[sl], M, grid, window, ops=_OracleOps)
        q.put((rank, out, gid, gate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("window", [None, (2, 2, 3)])
def test_ulysses_two_ranks_match_single_process(window):
    import numpy as np
    import oracle
    rng = np.random.default_rng(31)
    grid, M, H = (4, 3, 4), 3, 4            # N = 48 tokens, 4 heads -> 2 heads per rank
    N = grid[0] * grid[1] * grid[2]
    x = torch.from_numpy(rng.normal(size=(N, 6)))
    W = torch.from_numpy(rng.normal(size=(M, 6)))
    qkv = [torch.from_numpy(rng.normal(size=(N, H, 8))) for _ in range(3)]
    case = (x, W, *qkv, M, grid, window)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ulysses_worker, args=(r, 2, port, q, case)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict((r, (o, g, s)) for r, o, g, s in (q.get(timeout=120) for _ in range(2)))
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    ref = oracle.moga_layer(x.numpy(), W.numpy(), None, *(t.numpy() for t in qkv), M,
                            grid=grid if window else None, window=window)
    out = torch.cat([got[0][0], got[1][0]]).numpy()
    assert np.allclose(out, ref["out"], rtol=0, atol=1e-12)
    assert np.array_equal(torch.cat([got[0][1], got[1][1]]).numpy(), ref["group_id"])
    assert np.allclose(torch.cat([got[0][2], got[1][2]]).numpy(), ref["gate"], rtol=0, atol=1e-15)
