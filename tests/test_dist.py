"""Multi-process path on CPU (gloo, world size 2): batch sharding gives every
sequence to exactly one rank, the sharded results equal the single-process
results, and the timing reduction is the maximum over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from weight_state_recurrence_b200 import dist as wdist


def test_shard_partition():
    for total in (0, 1, 3, 4, 7, 64, 257):
        for world in (1, 2, 3, 8):
            ranges = [wdist.shard(total, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == total
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0 and a1 >= a0
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        wdist.shard(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import oracle
    from weight_state_recurrence_b200 import inputs
    wdist.init("gloo", timeout_s=60)
    B, H, N, d = 5, 2, 24, 8
    q, k, v = inputs.random_case(42, B, H, N, d, d)
    lam = torch.tensor([0.9, 1.0])
    b0, b1 = wdist.shard(B, world, rank)
    y, S, z = oracle.causal(q[b0:b1], k[b0:b1], v[b0:b1], lam, 1e-6, nthreads=1)
    parts = [None] * world
    torch.distributed.all_gather_object(parts, (b0, b1, y, S, z))
    t = wdist.max_over_ranks(float(rank + 1))
    wdist.barrier()
    if rank == 0:
        yf, Sf, zf = oracle.causal(q, k, v, lam, 1e-6, nthreads=1)
        ok = all(np.array_equal(yp, yf[a:b]) and np.array_equal(Sp, Sf[a:b]) and
                 np.array_equal(zp, zf[a:b]) for a, b, yp, Sp, zp in parts)
        covered = sorted(x for a, b, *_ in parts for x in range(a, b)) == list(range(B))
        out.put((ok, covered, t))
    wdist.finalize()


def test_two_rank_gloo_sharding():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    ok, covered, t = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert ok and covered and t == 2.0
