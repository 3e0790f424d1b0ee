"""GPU parity of linattn_fwd_global_cross (queries of one length attending to
keys / values of another) against the fp64 oracle's cross form."""
import pytest
import torch

import oracle
from weight_state_recurrence_b200 import inputs
from tests._compare import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def check_cross(lib, B, H, Nq, Nk, dk, dv, dtype, seed, tol, eps=1e-6):
    q, _, _ = inputs.random_case(seed, B, H, Nq, dk, dv, dtype, scale=dk ** -0.5)
    _, k, v = inputs.random_case(seed + 1, B, H, Nk, dk, dv, dtype, scale=dk ** -0.5)
    out, KV, ks = lib.fwd_global_cross(q.to(DEV), k.to(DEV), v.to(DEV), eps)
    torch.cuda.synchronize()
    y_o, KV_o, ks_o = oracle.global_cross(q, k, v, eps)
    if Nq:
        assert_close("y", out, y_o, tol)
    if Nk:
        assert_close("KV", KV, KV_o, tol)
        assert_close("ksum", ks, ks_o, tol)
    else:
        assert not KV.any() and not ks.any() and not out.any()


@pytest.mark.parametrize("Nq,Nk", [(300, 1000), (1000, 129), (128, 128), (1, 4096), (77, 0)])
def test_tensor_core_path_cross(cuda_lib, Nq, Nk):
    check_cross(cuda_lib, 2, 4, Nq, Nk, 64, 64, torch.bfloat16, 1600 + Nq + Nk, 2e-2)


@pytest.mark.parametrize("dk,dv", [(32, 32), (128, 64), (16, 128)])
def test_cuda_core_path_cross(cuda_lib, dk, dv):
    check_cross(cuda_lib, 2, 3, 90, 150, dk, dv, torch.float32, 1700 + dk + dv, 1e-4)


def test_empty_queries(cuda_lib):
    check_cross(cuda_lib, 1, 2, 0, 200, 64, 64, torch.bfloat16, 1800, 2e-2)


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
