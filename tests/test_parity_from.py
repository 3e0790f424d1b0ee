"""GPU parity of linattn_fwd_causal_from: the causal forward continued from a
caller-supplied state, against the fp64 oracle started from the same fp32
state (the state an oracle prefix run ends in, so its size and sign are those
of real use), and split-sequence consistency on the GPU itself."""
import numpy as np
import pytest
import torch

import oracle
from weight_state_recurrence_b200 import inputs
from weight_state_recurrence_b200.linattn import LinattnError
from tests._compare import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def prefix_state(q, k, v, lam, n0, eps=1e-6):
    """(S, z) after the first n0 tokens, from the oracle, rounded to fp32."""
    _, S0, z0 = oracle.causal(q[:, :, :n0], k[:, :, :n0], v[:, :, :n0], lam, eps)
    return torch.tensor(S0, dtype=torch.float32), torch.tensor(z0, dtype=torch.float32)


def check_from(lib, q, k, v, lam, n0, tol, eps=1e-6):
    S0, z0 = prefix_state(q, k, v, lam, n0, eps)
    qx, kx, vx = (t[:, :, n0:].contiguous() for t in (q, k, v))
    lamd = None if lam is None else lam.to(DEV)
    out, S, z = lib.fwd_causal(qx.to(DEV), kx.to(DEV), vx.to(DEV), lamd, eps,
                               S_init=S0.to(DEV), z_init=z0.to(DEV))
    torch.cuda.synchronize()
    y_o, S_o, z_o = oracle.causal(qx, kx, vx, lam, eps, S0=S0, z0=z0)
    assert_close("y", out, y_o, tol)
    assert_close("S_final", S, S_o, tol)
    assert_close("z_final", z, z_o, tol)


@pytest.mark.parametrize("N", [1, 129, 300])
@pytest.mark.parametrize("dv", [64, 128])
def test_tensor_core_path_from_state(cuda_lib, N, dv):
    q, k, v = inputs.random_case(900 + N + dv, 1, 3, 200 + N, 128, dv, torch.bfloat16,
                                 scale=128 ** -0.5)
    lam = torch.tensor([0.97, 0.5, 1.0], dtype=torch.float32)
    check_from(cuda_lib, q, k, v, lam, 200, 2e-2)


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 16), (128, 64), (16, 128)])
def test_cuda_core_path_from_state(cuda_lib, dk, dv):
    q, k, v = inputs.random_case(950 + dk + dv, 2, 2, 150, dk, dv, torch.float32,
                                 scale=dk ** -0.5)
    lam = torch.tensor([0.9, 1.0], dtype=torch.float32)
    check_from(cuda_lib, q, k, v, lam, 70, 1e-4)


def test_zero_decay_forgets_the_state(cuda_lib):
    q, k, v = inputs.random_case(960, 1, 2, 160, 128, 128, torch.bfloat16, scale=0.3)
    lam = torch.tensor([0.0, 0.0], dtype=torch.float32)
    check_from(cuda_lib, q, k, v, lam, 30, 2e-2)


def test_split_sequence_equals_one_call(cuda_lib):
    """prefill(n) then fwd_causal_from(rest) == prefill(all), on the GPU."""
    w = inputs.WORKLOADS["causal_decay_d128"]
    q, k, v = inputs.causal_inputs(w, B=1, H=4, N=1000)
    lam = inputs.decay(w, H=4).to(DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    y, S, z = cuda_lib.fwd_causal(qd, kd, vd, lam, w.eps)
    n = 333
    y1, S1, z1 = cuda_lib.fwd_causal(qd[:, :, :n].contiguous(), kd[:, :, :n].contiguous(),
                                     vd[:, :, :n].contiguous(), lam, w.eps)
    y2, S2, z2 = cuda_lib.fwd_causal(qd[:, :, n:].contiguous(), kd[:, :, n:].contiguous(),
                                     vd[:, :, n:].contiguous(), lam, w.eps, S_init=S1, z_init=z1)
    torch.cuda.synchronize()
    y_o, S_o, z_o = oracle.causal(q, k, v, lam.cpu(), w.eps)
    assert_close("split y", torch.cat([y1, y2], 2), y_o, 2e-2)
    assert_close("one-call y", y, y_o, 2e-2)
    assert_close("split S", S2, S_o, 2e-2)
    assert_close("split z", z2, z_o, 2e-2)
    assert_close("split vs one call", torch.cat([y1, y2], 2), y.double().cpu().numpy(), 2e-2)


def test_empty_sequence_copies_the_state(cuda_lib):
    q = torch.zeros(1, 2, 0, 128, dtype=torch.bfloat16, device=DEV)
    v = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device=DEV)
    S0 = torch.randn(1, 2, 128, 64, device=DEV)
    z0 = torch.rand(1, 2, 128, device=DEV)
    out, S, z = cuda_lib.fwd_causal(q, q, v, None, 1e-6, S_init=S0, z_init=z0)
    torch.cuda.synchronize()
    assert torch.equal(S, S0) and torch.equal(z, z0)


def test_state_arguments_are_checked(cuda_lib):
    q = torch.zeros(1, 1, 8, 32, dtype=torch.float32, device=DEV)
    S0 = torch.zeros(1, 1, 32, 32, device=DEV)
    z0 = torch.zeros(1, 1, 32, device=DEV)
    out = torch.empty_like(q)
    with pytest.raises(LinattnError):      # z_init missing
        cuda_lib.linattn_fwd_causal_from(q, q, q, None, 1e-6, S0, None, out)
    with pytest.raises(LinattnError):      # the starting state aliases the final one
        cuda_lib.linattn_fwd_causal_from(q, q, q, None, 1e-6, S0, z0, out, S0, z0)


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
