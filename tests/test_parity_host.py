"""GPU checks of fwd_causal_host, the causal forward on host tensors whose
batch pieces are copied in, computed and copied out on overlapping streams:
its results must equal the device call on the same inputs bit for bit (every
(b, h) is computed by the same kernel either way), and the oracle's."""
import pytest
import torch

import oracle
from weight_state_recurrence_b200 import inputs
from tests._compare import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("dtype,dk,pieces", [(torch.bfloat16, 128, 3), (torch.bfloat16, 128, 6),
                                             (torch.bfloat16, 128, None),
                                             (torch.float32, 32, 5)])
def test_host_pipeline_matches_device_call(cuda_lib, dtype, dk, pieces):
    # pieces: whole sequences (3), one head each (6), the default (runs of up
    # to 4 heads: one head each here), and 5 requested (whole sequences)
    B, H, N, dv = 3, 2, 700, 128 if dk == 128 else 32
    q, k, v = inputs.random_case(4100 + dk + (pieces or 0), B, H, N, dk, dv, dtype, scale=dk ** -0.5)
    lam = torch.tensor([0.95, 0.999])
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    y_h, S_h, z_h = cuda_lib.fwd_causal_host(hq, hk, hv, lam.to(DEV), 1e-6, pieces=pieces)
    assert not y_h.is_cuda and not S_h.is_cuda
    y_d, S_d, z_d = cuda_lib.fwd_causal(q.to(DEV), k.to(DEV), v.to(DEV), lam.to(DEV), 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(y_h, y_d.cpu())
    assert torch.equal(S_h, S_d.cpu())
    assert torch.equal(z_h, z_d.cpu())
    y_o, S_o, z_o = oracle.causal(q, k, v, lam, 1e-6)
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    assert_close("y", y_h, y_o, tol)
    assert_close("S", S_h, S_o, tol)
    assert_close("z", z_h, z_o, tol)


def test_host_pipeline_single_sequence(cuda_lib):
    # B = 1: the overlap comes from runs of heads alone
    B, H, N, d = 1, 8, 300, 64
    q, k, v = inputs.random_case(4200, B, H, N, d, d, torch.bfloat16, scale=d ** -0.5)
    y_h, S_h, z_h = cuda_lib.fwd_causal_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                                             None, 1e-6, pieces=4)
    y_d, S_d, z_d = cuda_lib.fwd_causal(q.to(DEV), k.to(DEV), v.to(DEV), None, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(y_h, y_d.cpu()) and torch.equal(S_h, S_d.cpu()) and torch.equal(z_h, z_d.cpu())


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
