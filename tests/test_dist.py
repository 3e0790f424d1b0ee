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


# ------------------------------------------------ sequence parallelism
class OracleOps:
    """The three per-rank steps of the sequence-parallel forward, taken from
    the fp64 oracle: the state of a segment from zero is the final state of
    the recurrence over it (it does not depend on q), the scan is the
    recurrence of the carried state over whole segments, the output is the
    recurrence continued from a given state."""

    def state(self, k, v, lam):
        import oracle
        _, S, z = oracle.causal(k, k, v, lam, 0.0, nthreads=1)
        return torch.from_numpy(S), torch.from_numpy(z)

    def combine(self, seg_len, lam, S_init, z_init, dS, dz):
        G, B, H = dS.shape[:3]
        g = (torch.ones(H, dtype=torch.float64) if lam is None
             else lam.to(torch.float64) ** seg_len)
        run_S = torch.zeros_like(dS[0]) if S_init is None else S_init.to(torch.float64).clone()
        run_z = torch.zeros_like(dz[0]) if z_init is None else z_init.to(torch.float64).clone()
        for s in range(G):
            nS, nz = dS[s].clone(), dz[s].clone()
            dS[s], dz[s] = run_S, run_z
            run_S = g[None, :, None, None] * run_S + nS
            run_z = g[None, :, None] * run_z + nz

    def forward_from(self, q, k, v, lam, eps, S0, z0):
        import oracle
        return oracle.causal(q, k, v, lam, eps, S0=S0, z0=z0, nthreads=1)


def _seq_worker(rank, world, port, out, seg_len, N, with_init):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import oracle
    from weight_state_recurrence_b200 import inputs
    wdist.init("gloo", timeout_s=60)
    B, H, d = 2, 3, 8
    q, k, v = inputs.random_case(77, B, H, N, d, d)
    lam = torch.tensor([0.9, 1.0, 0.0])
    S_init = z_init = None
    if with_init:
        _, S_init, z_init = oracle.causal(*inputs.random_case(78, B, H, 5, d, d), lam, 1e-6)
        S_init, z_init = torch.from_numpy(S_init), torch.from_numpy(z_init)
    n0 = rank * seg_len
    n1 = min(N, n0 + seg_len)
    part = [t[:, :, n0:n1].contiguous() for t in (q, k, v)]
    y, S, z = wdist.seq_parallel_causal(*part, lam, 1e-6, world=world, rank=rank,
                                        seg_len=seg_len, ops=OracleOps(), S_init=S_init,
                                        z_init=z_init)
    parts = [None] * world
    torch.distributed.all_gather_object(parts, (n0, n1, y, S, z))
    if rank == 0:
        yf, Sf, zf = oracle.causal(q, k, v, lam, 1e-6, S0=S_init, z0=z_init, nthreads=1)
        scale = np.abs(yf).max()
        err_y = max(np.abs(yp - yf[:, :, a:b]).max() for a, b, yp, _, _ in parts) / scale
        _, _, _, S_last, z_last = parts[-1]
        err_S = np.abs(S_last - Sf).max() / np.abs(Sf).max()
        err_z = np.abs(z_last - zf).max() / np.abs(zf).max()
        covered = [x for a, b, *_ in parts for x in range(a, b)] == list(range(N))
        out.put((err_y, err_S, err_z, covered))
    wdist.finalize()


@pytest.mark.parametrize("world,seg_len,N,with_init", [(2, 20, 37, False), (2, 16, 32, True),
                                                       (3, 11, 30, True)])
def test_sequence_parallel_gloo(world, seg_len, N, with_init):
    """Sequences cut by token position over gloo ranks: own segment state,
    one all-gather, the scan, the continued forward; the pieces must equal the
    single-process recurrence over the whole sequence (fp64, so to rounding)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_seq_worker, args=(r, world, port, q, seg_len, N, with_init))
             for r in range(world)]
    for p in procs:
        p.start()
    err_y, err_S, err_z, covered = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert covered
    assert err_y < 1e-12 and err_S < 1e-12 and err_z < 1e-12, (err_y, err_S, err_z)


def test_sequence_parallel_rejects_short_middle_segment():
    with pytest.raises(ValueError):
        wdist.seq_parallel_causal(torch.zeros(1, 1, 3, 4), torch.zeros(1, 1, 3, 4),
                                  torch.zeros(1, 1, 3, 4), None, 1e-6, world=2, rank=0,
                                  seg_len=4, ops=OracleOps())
