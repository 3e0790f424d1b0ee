"""GPU parity of the pieces of the sequence-parallel causal forward: the
state-only pass (linattn_causal_state), the scan of segment states
(linattn_combine_states), and the whole per-rank sequence of
weight_state_recurrence_b200.dist.seq_parallel_causal on one GPU, with the
all-gather replaced by the stack of every rank's state (the ranks' kernels
never wait on one another, so one GPU can play them in turn)."""
import numpy as np
import pytest
import torch

import oracle
from weight_state_recurrence_b200 import dist as wdist
from weight_state_recurrence_b200 import inputs
from tests._compare import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def state(lib, k, v, lam):
    B, H, N, dk = k.shape
    dv = v.shape[-1]
    S = torch.empty(B, H, dk, dv, device=DEV)
    z = torch.empty(B, H, dk, device=DEV)
    lib.linattn_causal_state(k.to(DEV), v.to(DEV), None if lam is None else lam.to(DEV), S, z)
    torch.cuda.synchronize()
    return S, z


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, torch.bfloat16), (64, 64, torch.bfloat16),
                                         (128, 64, torch.bfloat16), (32, 32, torch.float32),
                                         (64, 16, torch.float32)])
@pytest.mark.parametrize("N", [1, 127, 300, 1000])
def test_state_pass(cuda_lib, dk, dv, dtype, N):
    q, k, v = inputs.random_case(4000 + N + dk, 2, 3, N, dk, dv, dtype, scale=dk ** -0.5)
    lam = torch.tensor([0.0, 0.95, 1.0])
    S, z = state(cuda_lib, k, v, lam)
    _, S_o, z_o = oracle.causal(q, k, v, lam, 1e-6)
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert_close("S", S, S_o, tol)
    assert_close("z", z, z_o, tol)


def test_state_pass_empty(cuda_lib):
    k = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16)
    S, z = state(cuda_lib, k, k, None)
    assert not S.any() and not z.any()


def numpy_scan(seg_len, lam, S_init, z_init, dS, dz):
    """carry_0 = (S_init, z_init) or zero, carry_{g+1} = lam^seg_len carry_g +
    dS_g; returns the carries (the recurrence of the carried state over whole
    segments), fp64."""
    G, B, H = dS.shape[:3]
    g = np.ones(H) if lam is None else np.asarray(lam, np.float64) ** seg_len
    run_S = np.zeros(dS.shape[1:]) if S_init is None else np.array(S_init, np.float64)
    run_z = np.zeros(dz.shape[1:]) if z_init is None else np.array(z_init, np.float64)
    cS, cz = np.empty(dS.shape), np.empty(dz.shape)
    for s in range(G):
        cS[s], cz[s] = run_S, run_z
        run_S = g[None, :, None, None] * run_S + dS[s]
        run_z = g[None, :, None] * run_z + dz[s]
    return cS, cz


@pytest.mark.parametrize("G,with_init", [(1, False), (2, True), (7, False), (64, True)])
def test_combine_states(cuda_lib, G, with_init):
    gen = torch.Generator().manual_seed(4100 + G)
    B, H, dk, dv, L = 2, 3, 64, 32, 300
    dS = torch.randn(G, B, H, dk, dv, generator=gen)
    dz = torch.rand(G, B, H, dk, generator=gen)
    lam = torch.tensor([0.999, 1.0, 0.0])
    S_init = torch.randn(B, H, dk, dv, generator=gen) if with_init else None
    z_init = torch.rand(B, H, dk, generator=gen) if with_init else None
    cS, cz = numpy_scan(L, lam.numpy(), None if S_init is None else S_init.numpy(),
                        None if z_init is None else z_init.numpy(), dS.double().numpy(),
                        dz.double().numpy())
    dS_d, dz_d = dS.to(DEV), dz.to(DEV)
    cuda_lib.linattn_combine_states(L, lam.to(DEV), None if S_init is None else S_init.to(DEV),
                                    None if z_init is None else z_init.to(DEV), dS_d, dz_d)
    torch.cuda.synchronize()
    assert_close("carried S", dS_d, cS, 1e-5)
    assert_close("carried z", dz_d, cz, 1e-5)


@pytest.mark.parametrize("world,seg_len,N,dtype", [(4, 512, 2000, torch.bfloat16),
                                                   (3, 128, 300, torch.bfloat16),
                                                   (2, 64, 100, torch.float32)])
def test_seq_parallel_on_one_gpu(cuda_lib, world, seg_len, N, dtype):
    """Every rank's steps of seq_parallel_causal with the library's kernels;
    the all-gather is played by stacking the states all ranks computed."""
    B, H, d = 2, 4, 128 if dtype == torch.bfloat16 else 32
    q, k, v = inputs.random_case(4200 + N, B, H, N, d, d, dtype, scale=d ** -0.5)
    lam = torch.tensor([0.9, 0.999, 1.0, 0.5])
    lamd = lam.to(DEV)
    ops = wdist.LibraryOps(cuda_lib)
    parts = []
    for r in range(world):
        n0, n1 = r * seg_len, min(N, (r + 1) * seg_len)
        parts.append([t[:, :, n0:n1].contiguous().to(DEV) for t in (q, k, v)])
    states = [ops.state(pk, pv, lamd) for _, pk, pv in parts]
    stacks = [torch.stack([s for s, _ in states]), torch.stack([z for _, z in states])]
    ys = []
    for r in range(world):
        calls = iter(stacks)
        y, S, z = wdist.seq_parallel_causal(*parts[r], lamd, 1e-6, world=world, rank=r,
                                            seg_len=seg_len, ops=ops,
                                            gather=lambda x, w: next(calls).clone())
        ys.append(y)
    torch.cuda.synchronize()
    y_o, S_o, z_o = oracle.causal(q, k, v, lam, 1e-6)
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert_close("y", torch.cat(ys, dim=2), y_o, tol)
    assert_close("S after the last rank", S, S_o, tol)
    assert_close("z after the last rank", z, z_o, tol)


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
