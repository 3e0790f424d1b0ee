"""linattn_fwd_causal_noalloc: the causal forward whose segment-parallel form
takes its scratch from a static device array of the library instead of a
caller workspace.  CPU: the symbol and its argument checks.  GPU: parity with
the oracle on a segmented case and on the tensor-core path, and back-to-back
calls reusing the scratch."""
import ctypes

import pytest
import torch

import oracle
from weight_state_recurrence_b200 import inputs, linattn
from tests._compare import assert_close

DEV = "cuda:0"


def test_no_alloc_symbol_and_checks():
    lib = linattn.load()
    assert hasattr(lib, "linattn_fwd_causal_noalloc")
    d = linattn.linattn_dims(1, 1, 8, 64, 64, 0)
    f = ctypes.c_void_p(0x7F0000000000)
    out = ctypes.c_void_p(0x7F0000100000)
    # NULL q, a misaligned output and an unsupported d_k fail before any launch
    assert lib.linattn_fwd_causal_noalloc(ctypes.byref(d), None, f, f, None, 1e-6, out, None,
                                          None, None) == linattn.LINATTN_ERR_INVALID
    assert lib.linattn_fwd_causal_noalloc(ctypes.byref(d), f, f, f, None, 1e-6,
                                          ctypes.c_void_p(0x7F0000100008), None, None,
                                          None) == linattn.LINATTN_ERR_INVALID
    d.dk = 48
    assert lib.linattn_fwd_causal_noalloc(ctypes.byref(d), f, f, f, None, 1e-6, out, None,
                                          None, None) == linattn.LINATTN_ERR_UNSUPPORTED


def run(lib, q, k, v, lam, eps):
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    out = torch.empty(B, H, N, dv, dtype=v.dtype, device=DEV)
    S = torch.empty(B, H, dk, dv, device=DEV)
    z = torch.empty(B, H, dk, device=DEV)
    lib.linattn_fwd_causal_noalloc(q.to(DEV), k.to(DEV), v.to(DEV),
                                   None if lam is None else lam.to(DEV), eps, out, S, z)
    return out, S, z


SCRATCH_BYTES = 16 << 20   # the library's static scratch array


@pytest.mark.gpu
def test_no_alloc_segmented_workload(cuda_lib):
    """causal_d64 (16 heads): the tensor-core path cuts it into segments
    whose states fit the scratch.  The no-allocation call must give exactly
    the bits of the same segmented call with a caller workspace, which differ
    from the single pass (other summation order), so the scratch was used."""
    w = inputs.WORKLOADS["causal_d64"]
    q, k, v = inputs.causal_inputs(w)
    need = cuda_lib.linattn_fwd_causal_workspace(w.B, w.H, w.N, w.d, w.d, w.dtype)
    assert 0 < need <= SCRATCH_BYTES
    out, S, z = run(cuda_lib, q, k, v, None, w.eps)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    out_ws = torch.empty_like(out)
    S_ws, z_ws = torch.empty_like(S), torch.empty_like(z)
    cuda_lib.linattn_fwd_causal_ws(q.to(DEV), k.to(DEV), v.to(DEV), None, w.eps, None, None,
                                   out_ws, S_ws, z_ws, ws)
    out_1, S_1, _ = cuda_lib.fwd_causal(q.to(DEV), k.to(DEV), v.to(DEV), None, w.eps)
    torch.cuda.synchronize()
    assert torch.equal(out, out_ws) and torch.equal(S, S_ws) and torch.equal(z, z_ws)
    assert not torch.equal(S, S_1)
    y_o, S_o, z_o = oracle.causal(q, k, v, None, w.eps)
    assert_close("y", out, y_o, 2e-2)
    assert_close("S_final", S, S_o, 2e-2)
    assert_close("z_final", z, z_o, 2e-2)


@pytest.mark.gpu
def test_no_alloc_back_to_back_calls_share_the_scratch(cuda_lib):
    outs = []
    cases = []
    for seed in (2001, 2002):
        q, k, v = inputs.random_case(seed, 1, 2, 1500, 32, 32, torch.float32, scale=32 ** -0.5)
        lam = torch.tensor([0.99, 1.0])
        cases.append((q, k, v, lam))
        outs.append(run(cuda_lib, q, k, v, lam, 1e-6))   # same stream: ordered
    torch.cuda.synchronize()
    for (q, k, v, lam), (out, S, z) in zip(cases, outs):
        y_o, S_o, _ = oracle.causal(q, k, v, lam, 1e-6)
        assert_close("y", out, y_o, 1e-4)
        assert_close("S_final", S, S_o, 1e-4)


@pytest.mark.gpu
def test_no_alloc_tensor_core_path(cuda_lib):
    q, k, v = inputs.random_case(2003, 1, 2, 300, 128, 128, torch.bfloat16, scale=128 ** -0.5)
    lam = torch.tensor([0.97, 0.9])
    out, S, z = run(cuda_lib, q, k, v, lam, 1e-6)
    torch.cuda.synchronize()
    y_o, S_o, _ = oracle.causal(q, k, v, lam, 1e-6)
    assert_close("y", out, y_o, 2e-2)
    assert_close("S_final", S, S_o, 2e-2)


@pytest.mark.gpu
def test_no_alloc_no_device_errors(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
