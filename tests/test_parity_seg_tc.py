"""GPU parity of the segmented tensor-core causal forward: every sequence cut
into G segments, each segment's own state from the tensor-core state pass,
the starting states from the combine scan, then all segments at once
(fast-weight article §4.1 note and §5.2: blocks in parallel, the state carried
across them).  Against the fp64 oracle's plain recurrence, with no kernel
forced except the segment count."""
import math

import pytest
import torch

import oracle
from weight_state_recurrence_b200 import inputs
from weight_state_recurrence_b200.linattn import (LINATTN_KERNEL_AUTO, LINATTN_OP_CAUSAL,
                                                   kernel_choice)
from tests._compare import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run_ws(lib, q, k, v, lam, eps, S0=None, z0=None):
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    need = lib.linattn_fwd_causal_workspace(B, H, N, dk, dv, q.dtype)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=DEV)
    out = torch.empty(B, H, N, dv, dtype=v.dtype, device=DEV)
    S = torch.empty(B, H, dk, dv, device=DEV)
    z = torch.empty(B, H, dk, device=DEV)
    lib.linattn_fwd_causal_ws(q.to(DEV), k.to(DEV), v.to(DEV),
                              None if lam is None else lam.to(DEV), eps,
                              None if S0 is None else S0.to(DEV),
                              None if z0 is None else z0.to(DEV), out, S, z, ws)
    torch.cuda.synchronize()
    return need, out, S, z


def expected_G(N, G):
    """Segments the library makes when asked for at most G: whole chunks of
    128 tokens, ceil(chunks / G) per segment; for two, the first segment
    (which runs beside the state pass) takes ceil(chunks / 1.6)."""
    nch = -(-N // 128)
    per = math.ceil(nch / 1.6) if G == 2 else -(-nch // G)
    return -(-nch // per)


def check(lib, q, k, v, lam, eps, G, S0=None, z0=None, tol=2e-2):
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    with kernel_choice(LINATTN_OP_CAUSAL, LINATTN_KERNEL_AUTO, segments=G):
        need, out, S, z = run_ws(lib, q, k, v, lam, eps, S0, z0)
    g = expected_G(N, G)
    assert need == (B * H * g * (dk * dv + dk) * 4 if g > 1 else 0)
    y_o, S_o, z_o = oracle.causal(q, k, v, lam, eps, S0=S0, z0=z0)
    assert_close("y", out, y_o, tol)
    assert_close("S_final", S, S_o, tol)
    assert_close("z_final", z, z_o, tol)


@pytest.mark.parametrize("G", [2, 3, 5])
@pytest.mark.parametrize("N", [1024, 1000, 1153])
def test_segments_decay_edges(cuda_lib, G, N):
    """lambda in {0, 0.9, 1} (explicit and factored decay), several segments,
    a ragged last chunk in the last segment."""
    q, k, v = inputs.random_case(3000 + G * 7 + N, 2, 3, N, 128, 128, torch.bfloat16,
                                 scale=128 ** -0.5)
    lam = torch.tensor([0.0, 0.9, 1.0])
    check(cuda_lib, q, k, v, lam, 1e-6, G)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_segments_shapes(cuda_lib, dk, dv):
    q, k, v = inputs.random_case(3100 + dk + dv, 1, 2, 777, dk, dv, torch.bfloat16,
                                 scale=dk ** -0.5)
    lam = torch.tensor([0.97, 0.5])
    check(cuda_lib, q, k, v, lam, 1e-6, 4)


def test_segments_from_a_starting_state(cuda_lib):
    q, k, v = inputs.random_case(3200, 1, 2, 900 + 60, 128, 128, torch.bfloat16,
                                 scale=128 ** -0.5)
    lam = torch.tensor([0.999, 0.6])
    _, S0, z0 = oracle.causal(q[:, :, :60], k[:, :, :60], v[:, :, :60], lam, 1e-6)
    S0 = torch.tensor(S0, dtype=torch.float32)
    z0 = torch.tensor(z0, dtype=torch.float32)
    qx, kx, vx = (t[:, :, 60:].contiguous() for t in (q, k, v))
    check(cuda_lib, qx, kx, vx, lam, 1e-6, 3, S0=S0, z0=z0)


def test_causal_d64_workload_auto_segments(cuda_lib):
    """The causal_d64 workload (B=2, H=8, N=4096, d=64, no decay) as the
    library plans it: 16 heads cut into about one segment per SM."""
    w = inputs.WORKLOADS["causal_d64"]
    q, k, v = inputs.causal_inputs(w)
    need, out, S, z = run_ws(cuda_lib, q, k, v, None, w.eps)
    assert need > 0
    y_o, S_o, z_o = oracle.causal(q, k, v, None, w.eps)
    assert_close("y", out, y_o, w.tol)
    assert_close("S_final", S, S_o, w.tol)
    assert_close("z_final", z, z_o, w.tol)


def test_headline_workload_two_segments_sampled(cuda_lib):
    """The causal_decay_d128 workload at full size (B=4, H=16, N=16384,
    d=128) cut into two segments per sequence, sampled heads against the
    oracle."""
    w = inputs.WORKLOADS["causal_decay_d128"]
    q, k, v = inputs.causal_inputs(w)
    lam = inputs.decay(w)
    with kernel_choice(LINATTN_OP_CAUSAL, LINATTN_KERNEL_AUTO, segments=2):
        need, out, S, z = run_ws(cuda_lib, q, k, v, lam, w.eps)
    assert need == w.B * w.H * 2 * (128 * 128 + 128) * 4
    for b, h in [(0, 0), (1, 9), (3, 15)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        y_o, S_o, z_o = oracle.causal(q[sl], k[sl], v[sl], lam[h:h + 1], w.eps)
        assert_close(f"y[{b},{h}]", out[sl], y_o, w.tol)
        assert_close(f"S_final[{b},{h}]", S[sl], S_o, w.tol)
        assert_close(f"z_final[{b},{h}]", z[sl], z_o, w.tol)


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0


def test_output_16_byte_aligned_only(cuda_lib):
    """y written to a buffer that is 16- but not 32-byte aligned (the
    kernel's 32-byte stores need the wider alignment and fall back)."""
    q, k, v = inputs.random_case(3300, 1, 2, 300, 128, 128, torch.bfloat16, scale=128 ** -0.5)
    lam = torch.tensor([0.95, 1.0])
    raw = torch.empty(q.numel() + 8, dtype=torch.bfloat16, device=DEV)
    off = 8 if raw.data_ptr() % 32 == 0 else 0   # 8 bf16 = 16 bytes
    out = raw[off:off + q.numel()].view(q.shape)
    assert out.data_ptr() % 32 == 16
    S = torch.empty(1, 2, 128, 128, device=DEV)
    z = torch.empty(1, 2, 128, device=DEV)
    cuda_lib.linattn_fwd_causal(q.to(DEV), k.to(DEV), v.to(DEV), lam.to(DEV), 1e-6, out, S, z)
    torch.cuda.synchronize()
    y_o, S_o, z_o = oracle.causal(q, k, v, lam, 1e-6)
    assert_close("y", out, y_o, 2e-2)
    assert_close("S_final", S, S_o, 2e-2)


@pytest.mark.parametrize("G", [1, 2, 3])
@pytest.mark.parametrize("with_init", [False, True])
def test_factored_frames(cuda_lib, G, with_init):
    """Factored decay keeps the state relative to a frame of
    R = floor(64 / (128 log2(1/lambda))) chunks and renormalises at its end:
    lambda = 0.7 (R = 1: every chunk, k weights near 2^66), 0.75 (R = 1),
    0.85 (R = 2), 0.9 (R = 3), 0.99 (R = 34: one frame here), 0.9999; ten
    chunks with a ragged last one, in one pass or cut into segments."""
    N = 128 * 9 + 37
    q, k, v = inputs.random_case(3400 + G + 10 * with_init, 1, 6, N, 128, 128, torch.bfloat16,
                                 scale=128 ** -0.5)
    lam = torch.tensor([0.7, 0.75, 0.85, 0.9, 0.99, 0.9999])
    S0 = z0 = None
    if with_init:
        gen = torch.Generator().manual_seed(3450 + G)
        S0 = torch.randn(1, 6, 128, 128, generator=gen) * 0.05
        z0 = torch.rand(1, 6, 128, generator=gen) + 0.5
    check(cuda_lib, q, k, v, lam, 1e-6, G, S0=S0, z0=z0)
