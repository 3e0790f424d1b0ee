"""GPU parity of the segment-parallel causal forward (linattn_fwd_causal_ws):
the sequence cut into segments run at once from scanned starting states must
give the recurrence's outputs and final state, against the fp64 oracle."""
import pytest
import torch

import oracle
from weight_state_recurrence_b200 import inputs
from weight_state_recurrence_b200.linattn import (LINATTN_KERNEL_CUDA_CORES, LINATTN_OP_CAUSAL,
                                                   kernel_choice)
from tests._compare import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run_ws(lib, q, k, v, lam, eps, S0=None, z0=None, ws_bytes=None):
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    need = lib.linattn_fwd_causal_workspace(B, H, N, dk, dv, q.dtype)
    nbytes = need if ws_bytes is None else ws_bytes
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=DEV) if nbytes else None
    out = torch.empty(B, H, N, dv, dtype=v.dtype, device=DEV)
    S = torch.empty(B, H, dk, dv, device=DEV)
    z = torch.empty(B, H, dk, device=DEV)
    lib.linattn_fwd_causal_ws(q.to(DEV), k.to(DEV), v.to(DEV),
                              None if lam is None else lam.to(DEV), eps,
                              None if S0 is None else S0.to(DEV),
                              None if z0 is None else z0.to(DEV), out, S, z, ws)
    torch.cuda.synchronize()
    return need, out, S, z


def test_causal_d64_workload_segmented_cuda_cores(cuda_lib):
    """The causal_d64 workload (16 heads, 4096 tokens, d = 64, bf16) on the
    CUDA-core path (chosen explicitly: bf16 with d_k = 64 normally takes the
    tensor cores), cut into segments."""
    w = inputs.WORKLOADS["causal_d64"]
    q, k, v = inputs.causal_inputs(w)
    with kernel_choice(LINATTN_OP_CAUSAL, LINATTN_KERNEL_CUDA_CORES):
        need, out, S, z = run_ws(cuda_lib, q, k, v, None, w.eps)
    assert need > 0
    y_o, S_o, z_o = oracle.causal(q, k, v, None, w.eps)
    assert_close("y", out, y_o, 2e-2)
    assert_close("S_final", S, S_o, 2e-2)
    assert_close("z_final", z, z_o, 2e-2)


@pytest.mark.parametrize("N", [256, 1000, 3001])
def test_fp32_segmented_from_state(cuda_lib, N):
    q, k, v = inputs.random_case(1900 + N, 1, 2, N + 50, 32, 32, torch.float32, scale=32 ** -0.5)
    lam = torch.tensor([0.999, 1.0], dtype=torch.float32)
    _, S0, z0 = oracle.causal(q[:, :, :50], k[:, :, :50], v[:, :, :50], lam, 1e-6)
    S0 = torch.tensor(S0, dtype=torch.float32)
    z0 = torch.tensor(z0, dtype=torch.float32)
    qx, kx, vx = (t[:, :, 50:].contiguous() for t in (q, k, v))
    need, out, S, z = run_ws(cuda_lib, qx, kx, vx, lam, 1e-6, S0, z0)
    assert need > 0
    y_o, S_o, z_o = oracle.causal(qx, kx, vx, lam, 1e-6, S0=S0, z0=z0)
    assert_close("y", out, y_o, 1e-4)
    assert_close("S_final", S, S_o, 1e-4)
    assert_close("z_final", z, z_o, 1e-4)


def test_small_decay_segments(cuda_lib):
    q, k, v = inputs.random_case(1950, 1, 1, 2000, 64, 16, torch.float32, scale=0.125)
    lam = torch.tensor([0.3], dtype=torch.float32)
    need, out, S, z = run_ws(cuda_lib, q, k, v, lam, 1e-6)
    assert need > 0
    y_o, S_o, z_o = oracle.causal(q, k, v, lam, 1e-6)
    assert_close("y", out, y_o, 1e-4)
    assert_close("S_final", S, S_o, 1e-4)


def test_small_workspace_runs_the_single_pass(cuda_lib):
    w = inputs.WORKLOADS["causal_d64"]
    q, k, v = inputs.causal_inputs(w, B=1, H=2, N=1024)
    with kernel_choice(LINATTN_OP_CAUSAL, LINATTN_KERNEL_CUDA_CORES):
        need, out, S, z = run_ws(cuda_lib, q, k, v, None, w.eps, ws_bytes=64)
    assert need > 64
    y_o, S_o, _ = oracle.causal(q, k, v, None, w.eps)
    assert_close("y", out, y_o, 2e-2)
    assert_close("S_final", S, S_o, 2e-2)


def test_workspace_query(cuda_lib):
    ws = cuda_lib.linattn_fwd_causal_workspace
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # tensor-core path, 16 heads: about one segment per SM, 128-token multiples
    G = -(-32 // -(-32 // (sms // 16)))
    assert ws(2, 8, 4096, 64, 64, torch.bfloat16) == 16 * G * (64 * 64 + 64) * 4
    # 64 heads on 148 SMs: two segments (the first beside the state pass)
    assert ws(4, 16, 16384, 128, 128, torch.bfloat16) == (64 * 2 * (128 * 128 + 128) * 4
                                                           if sms >= 128 else 0)
    assert ws(8, 16, 16384, 128, 128, torch.bfloat16) == 0   # 128 heads: one pass
    assert ws(2, 8, 4096, 32, 32, torch.bfloat16) > 0        # 16 heads on CUDA cores: segmented
    assert ws(2, 8, 4096, 64, 64, torch.float32) > 0         # likewise
    with kernel_choice(LINATTN_OP_CAUSAL, LINATTN_KERNEL_CUDA_CORES):
        assert ws(2, 8, 4096, 64, 64, torch.bfloat16) > 0    # CUDA cores chosen: segmented
    assert ws(64, 64, 4096, 64, 64, torch.float32) == 0      # enough heads already
    assert ws(1, 1, 100, 64, 64, torch.float32) == 0         # too short to cut
    assert ws(1, 1, 4096, 48, 64, torch.float32) == 0        # unsupported: no plan


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
