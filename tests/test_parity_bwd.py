"""GPU parity of linattn_bwd_causal (the backward of the causal forward)
against the fp64 gradient oracle (torch autograd of the masked form, pinned by
central differences in tests/test_oracle_grad.py), on identical seeded inputs.
Gate per gradient tensor: max|gpu - oracle| / max|oracle| <= 1e-4 for fp32
inputs and 2e-2 for bf16 inputs (fp32 arithmetic, bf16 outputs)."""
import numpy as np
import pytest
import torch

from oracle import grad as og
from weight_state_recurrence_b200 import inputs
from tests._compare import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def check_bwd(lib, B, H, N, dk, dv, dtype, lam, seed, tol, want_dlam=True, eps=1e-6):
    q, k, v = inputs.random_case(seed, B, H, N, dk, dv, dtype, scale=dk ** -0.5)
    g = torch.Generator().manual_seed(seed + 7)
    dy = torch.randn(B, H, N, dv, generator=g).to(dtype)
    lamd = None if lam is None else lam.to(DEV)
    dq, dkk, dvv, dl = lib.bwd_causal(q.to(DEV), k.to(DEV), v.to(DEV), dy.to(DEV), lamd, eps,
                                      want_dlam=want_dlam)
    torch.cuda.synchronize()
    lam_o = lam if lam is not None else (torch.ones(H) if want_dlam else None)
    _, dq_o, dk_o, dv_o, dl_o = og.causal_grad(q, k, v, lam_o, eps, dy)
    assert_close("dq", dq, dq_o, tol)
    assert_close("dk", dkk, dk_o, tol)
    assert_close("dv", dvv, dv_o, tol)
    if want_dlam:
        assert_close("dlambda", dl, dl_o, tol)


# When every token attends only to itself (N = 1, or lambda = 0), y_i = v_i w_i /
# (w_i + eps) and dphi(q_i) = S_i dnum_i + z_i dden_i is a difference of two
# O(1) terms whose exact value is proportional to eps: with eps = 1e-6 it lies
# below the fp32 resolution of those terms.  Those cases use eps = 0.5, where the
# gradient is a well-conditioned quantity.
SELF_ONLY_EPS = 0.5


@pytest.mark.parametrize("N", [1, 31, 32, 33, 100])
def test_bwd_fp32_lengths(cuda_lib, N):
    check_bwd(cuda_lib, 2, 2, N, 32, 32, torch.float32, torch.tensor([0.9, 1.0]), 1100 + N, 1e-4,
              eps=SELF_ONLY_EPS if N == 1 else 1e-6)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128), (128, 16)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bwd_shapes(cuda_lib, dk, dv, dtype):
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    check_bwd(cuda_lib, 1, 2, 70, dk, dv, dtype, torch.tensor([0.97, 0.6]), 1200 + dk + dv, tol)


@pytest.mark.parametrize("lamv", [0.0, 0.5, 1.0])
def test_bwd_decay_edges(cuda_lib, lamv):
    # lambda = 0: the oracle's dlambda is finite (running products); compare it too
    check_bwd(cuda_lib, 1, 1, 45, 64, 64, torch.float32, torch.tensor([lamv]), 1300, 1e-4,
              eps=SELF_ONLY_EPS if lamv == 0.0 else 1e-6)


def test_bwd_without_decay_and_without_dlambda(cuda_lib):
    check_bwd(cuda_lib, 2, 3, 50, 64, 64, torch.float32, None, 1400, 1e-4, want_dlam=False)
    check_bwd(cuda_lib, 1, 2, 50, 64, 64, torch.float32, None, 1401, 1e-4, want_dlam=True)


def test_bwd_decay_workload_shape(cuda_lib):
    """The causal_decay_d128 workload's head shape, lambda in [0.9, 0.999],
    four heads and 300 tokens (several chunks and a ragged tail)."""
    w = inputs.WORKLOADS["causal_decay_d128"]
    lam = inputs.decay(w, H=4)
    check_bwd(cuda_lib, 1, 4, 300, 128, 128, torch.bfloat16, lam, 1500, 2e-2)


@pytest.mark.parametrize("N,lam", [(4096, (0.9, 0.999)), (8192, (1.0,))])
def test_bwd_long_sequence(cuda_lib, N, lam):
    """Accumulation of the carried states over a long sequence: heads of the
    decay workload's shape (d = 128, bf16) and lambda range, 32 and 64 chunks
    of 128 tokens, against the gradient oracle's masked form."""
    lam = torch.tensor(lam, dtype=torch.float32)
    check_bwd(cuda_lib, 1, lam.numel(), N, 128, 128, torch.bfloat16, lam, 1600 + N, 2e-2)


def test_bwd_empty_sequence(cuda_lib):
    q = torch.zeros(1, 2, 0, 32, device=DEV)
    dq, dk, dv, dl = cuda_lib.bwd_causal(q, q, q, q, torch.ones(2, device=DEV), 1e-6,
                                         want_dlam=True)
    torch.cuda.synchronize()
    assert dq.numel() == 0 and not dl.any()


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
