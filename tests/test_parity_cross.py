"""GPU parity of linattn_fwd_global_cross (queries of one length attending to
keys / values of another) and of linattn_fwd_global_masked (the same with a
key padding mask) against the fp64 oracle's cross and masked forms."""
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


def random_padding(seed, B, Nk):
    """Padding rows of every kind: scattered keys, a padded tail, all padding
    (when B > 2), none."""
    g = torch.Generator().manual_seed(seed)
    pad = torch.rand(B, Nk, generator=g) < 0.3
    if B > 1:
        pad[1] = False
        pad[1, Nk // 2:] = True
    if B > 2:
        pad[2] = True
    if B > 3:
        pad[3] = False
    return pad


def check_masked(lib, B, H, Nq, Nk, dk, dv, dtype, seed, tol, eps=1e-6):
    q, _, _ = inputs.random_case(seed, B, H, Nq, dk, dv, dtype, scale=dk ** -0.5)
    _, k, v = inputs.random_case(seed + 1, B, H, Nk, dk, dv, dtype, scale=dk ** -0.5)
    pad = random_padding(seed + 2, B, Nk)
    out, KV, ks = lib.fwd_global_masked(q.to(DEV), k.to(DEV), v.to(DEV), pad.to(DEV), eps)
    torch.cuda.synchronize()
    y_o, KV_o, ks_o = oracle.global_masked(q, k, v, pad, eps)
    assert_close("y", out, y_o, tol)
    assert_close("KV", KV, KV_o, tol)
    assert_close("ksum", ks, ks_o, tol)
    if B > 2:   # a sequence whose keys are all padding
        assert not KV[2].any() and not ks[2].any() and not out[2].any()


@pytest.mark.parametrize("Nq,Nk", [(300, 1000), (128, 128), (200, 129)])
def test_tensor_core_path_masked(cuda_lib, Nq, Nk):
    check_masked(cuda_lib, 4, 4, Nq, Nk, 64, 64, torch.bfloat16, 1900 + Nq + Nk, 2e-2)


@pytest.mark.parametrize("dk,dv,dtype", [(32, 32, torch.float32), (128, 64, torch.float32),
                                         (64, 64, torch.bfloat16)])
def test_cuda_core_path_masked(cuda_lib, dk, dv, dtype):
    # H = 3 (odd) sends bf16 d = 64 to the CUDA-core kernels as well
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    check_masked(cuda_lib, 4, 3, 90, 150, dk, dv, dtype, 2000 + dk + dv, tol)


def test_masked_without_mask_is_cross(cuda_lib):
    """No mask: the same kernels as the cross form.  The KV kernel's CTAs add
    their partial sums with float atomics, so the order of those adds (and the
    last bits) may differ between calls: equal up to that rounding."""
    q, k, v = inputs.random_case(2100, 2, 4, 200, 64, 64, torch.bfloat16, scale=0.125)
    a = cuda_lib.fwd_global_masked(q.to(DEV), k.to(DEV), v.to(DEV), None, 1e-6)
    b = cuda_lib.fwd_global_cross(q.to(DEV), k.to(DEV), v.to(DEV), 1e-6)
    torch.cuda.synchronize()
    # KV and ksum (fp32) to rounding; y (bf16) to a bf16 step or two
    for name, x, y, tol in zip(("y", "KV", "ksum"), a, b, (8e-3, 1e-5, 1e-5)):
        assert_close(f"masked vs cross {name}", x, y.double().cpu().numpy(), tol)


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
