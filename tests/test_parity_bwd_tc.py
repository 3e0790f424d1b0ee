"""GPU parity of the tensor-core backward (linattn_bwd_causal for bf16 with
d_k = d_v = 128: the forward-recompute pass, the dlambda pass and the reverse
pass) against the fp64 gradient oracle (pinned by central differences in
tests/test_oracle_grad.py) on identical seeded inputs.

Gate per gradient tensor: max|gpu - oracle| / max|oracle| <= 2e-2, the bf16
tolerance of the forward: the operands of every product are bf16 (phi(q),
phi(k), v, dnum, the score tiles and the carried states rounded once, relative
2^-9 each) and every sum is accumulated in fp32."""
import ctypes

import pytest
import torch

from oracle import grad as og
from weight_state_recurrence_b200 import inputs
from weight_state_recurrence_b200.linattn import (LINATTN_KERNEL_AUTO, LINATTN_KERNEL_CUDA_CORES,
                                                   LINATTN_OP_BACKWARD, kernel_choice)
from tests._compare import assert_close, max_rel

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 2e-2
D = 128
# a token that attends only to itself makes dphi(q) proportional to eps (see
# tests/test_parity_bwd.py); those cases use a well-conditioned eps
SELF_ONLY_EPS = 0.5


def run(lib, q, k, v, dy, lam, eps, want_dlam, phi=0, kernel=LINATTN_KERNEL_AUTO):
    with kernel_choice(LINATTN_OP_BACKWARD, kernel):
        out = lib.bwd_causal(q.to(DEV), k.to(DEV), v.to(DEV), dy.to(DEV),
                             None if lam is None else lam.to(DEV), eps, want_dlam=want_dlam,
                             phi=phi)
    torch.cuda.synchronize()
    return out


def check(lib, B, H, N, lam, seed, want_dlam=True, eps=1e-6):
    q, k, v = inputs.random_case(seed, B, H, N, D, D, torch.bfloat16, scale=D ** -0.5)
    g = torch.Generator().manual_seed(seed + 7)
    dy = torch.randn(B, H, N, D, generator=g).to(torch.bfloat16)
    dq, dk, dv, dl = run(lib, q, k, v, dy, lam, eps, want_dlam)
    lam_o = lam if lam is not None else (torch.ones(H) if want_dlam else None)
    _, dq_o, dk_o, dv_o, dl_o = og.causal_grad(q, k, v, lam_o, eps, dy)
    pairs = [("dq", dq, dq_o), ("dk", dk, dk_o), ("dv", dv, dv_o)]
    if want_dlam:
        pairs.append(("dlambda", dl, dl_o))
    errs = {name: max_rel(a, b) for name, a, b in pairs}
    assert max(errs.values()) <= TOL, errs


@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 257, 640])
def test_lengths(cuda_lib, N):
    """One chunk, a ragged second chunk, exact multiples of the chunk and
    several chunks."""
    check(cuda_lib, 1, 2, N, torch.tensor([0.9, 0.999]), 4100 + N,
          eps=SELF_ONLY_EPS if N == 1 else 1e-6)


@pytest.mark.parametrize("lamv", [0.0, 0.3, 0.7, 0.95, 1.0])
def test_decay_values(cuda_lib, lamv):
    """lambda = 0 (each token sees itself only), small decays whose powers
    underflow inside a chunk, the headline range and no decay."""
    check(cuda_lib, 1, 1, 300, torch.tensor([lamv]), 4200,
          eps=SELF_ONLY_EPS if lamv == 0.0 else 1e-6)


def test_batch_heads_and_no_dlambda(cuda_lib):
    check(cuda_lib, 2, 3, 200, torch.tensor([0.9, 0.95, 0.999]), 4300, want_dlam=False)
    check(cuda_lib, 2, 2, 200, None, 4301, want_dlam=True)
    check(cuda_lib, 1, 2, 200, None, 4302, want_dlam=False)


def test_split_and_unsplit_forward_pass(cuda_lib):
    """The forward pass runs as two CTAs per head (the second from the state
    the state pass leaves at the split point) while the heads leave SMs
    idle, and as one CTA per head once they fill the GPU: an odd split point
    (5 chunks), and 160 heads over 3 chunks (no split)."""
    check(cuda_lib, 1, 2, 600, torch.tensor([0.95, 1.0]), 4350)
    check(cuda_lib, 10, 16, 300, inputs.decay(inputs.WORKLOADS["causal_decay_d128"], H=16), 4360)
    # without dlambda the reverse pass is split too (its earlier half from the
    # reverse state pass's adjoint): odd and even split points
    check(cuda_lib, 1, 2, 600, torch.tensor([0.95, 1.0]), 4370, want_dlam=False)
    check(cuda_lib, 1, 3, 1100, torch.tensor([0.5, 0.9, 0.999]), 4380, want_dlam=False)


@pytest.mark.parametrize("room", ["full", "stash", "none"])
def test_workspace_entry_point(cuda_lib, room):
    """linattn_bwd_causal_ws: with the queried workspace (split forward pass),
    with only the per-token stash (unsplit), and with none (the stash in the
    dk rows, the passes in order) the gradients are the same."""
    from weight_state_recurrence_b200 import linattn as L
    B, H, N = 1, 3, 700
    q, k, v = inputs.random_case(4700, B, H, N, D, D, torch.bfloat16, scale=D ** -0.5)
    dy = torch.randn(B, H, N, D, generator=torch.Generator().manual_seed(4701)).to(torch.bfloat16)
    lam = torch.tensor([0.9, 0.99, 1.0])
    need = L.linattn_bwd_causal_workspace(B, H, N, D, D, torch.bfloat16)
    assert need >= B * H * N * 8
    nbytes = {"full": need, "stash": B * H * N * 8, "none": 0}[room]
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=DEV)[:nbytes] if nbytes else None
    args = (q.to(DEV), k.to(DEV), v.to(DEV), dy.to(DEV), lam.to(DEV), 1e-6)
    if ws is None:
        # the ws entry point with (NULL, 0)
        d = L.linattn_dims(B, H, N, D, D, L.LINATTN_BF16, 0)
        dq, dk, dv = (torch.empty_like(args[0]), torch.empty_like(args[1]),
                      torch.empty_like(args[2]))
        dl = torch.empty(H, device=DEV)
        rc = L.load().linattn_bwd_causal_ws(ctypes.byref(d), *(L._ptr(t) for t in args[:3]),
                                            L._ptr(args[4]), 1e-6, L._ptr(args[3]), L._ptr(dq),
                                            L._ptr(dk), L._ptr(dv), L._ptr(dl), None, 0, None)
        assert rc == 0
    else:
        dq, dk, dv, dl = cuda_lib.bwd_causal(*args[:4], args[4], 1e-6, want_dlam=True,
                                             workspace=ws)
    torch.cuda.synchronize()
    _, dq_o, dk_o, dv_o, dl_o = og.causal_grad(q, k, v, lam, 1e-6, dy)
    errs = {n: max_rel(a, b) for n, a, b in
            (("dq", dq, dq_o), ("dk", dk, dk_o), ("dv", dv, dv_o), ("dlambda", dl, dl_o))}
    assert max(errs.values()) <= TOL, errs


def test_identity_features(cuda_lib):
    """phi = identity on positive feature vectors (phi' = 1)."""
    B, H, N = 1, 2, 300
    g = torch.Generator().manual_seed(4400)
    fq = (torch.rand(B, H, N, D, generator=g) * 0.2 + 0.01).to(torch.bfloat16)
    fk = (torch.rand(B, H, N, D, generator=g) * 0.2 + 0.01).to(torch.bfloat16)
    v = torch.randn(B, H, N, D, generator=g).to(torch.bfloat16)
    dy = torch.randn(B, H, N, D, generator=g).to(torch.bfloat16)
    lam = torch.tensor([0.97, 1.0])
    dq, dk, dv, dl = run(cuda_lib, fq, fk, v, dy, lam, 1e-6, True, phi=1)
    _, dq_o, dk_o, dv_o, dl_o = og.causal_grad(fq, fk, v, lam, 1e-6, dy, identity=True)
    assert_close("dq", dq, dq_o, TOL)
    assert_close("dk", dk, dk_o, TOL)
    assert_close("dv", dv, dv_o, TOL)
    assert_close("dlambda", dl, dl_o, TOL)


def test_matches_cuda_core_backward_at_length(cuda_lib):
    """At 4096 tokens (32 chunks) the tensor-core passes against the fp32
    CUDA-core backward (itself held to the oracle at 1e-4 in fp32) on the
    same bf16 inputs, for the headline decay range."""
    B, H, N = 1, 4, 4096
    q, k, v = inputs.random_case(4500, B, H, N, D, D, torch.bfloat16, scale=D ** -0.5)
    g = torch.Generator().manual_seed(4507)
    dy = torch.randn(B, H, N, D, generator=g).to(torch.bfloat16)
    lam = inputs.decay(inputs.WORKLOADS["causal_decay_d128"], H=H)
    tc = run(cuda_lib, q, k, v, dy, lam, 1e-6, True)
    ref = run(cuda_lib, q, k, v, dy, lam, 1e-6, True, kernel=LINATTN_KERNEL_CUDA_CORES)
    for name, a, b in zip(("dq", "dk", "dv", "dlambda"), tc, ref):
        assert_close(name, a, b.double().cpu(), TOL)


def test_repeatable(cuda_lib):
    """dq, dk, dv come from fixed-order sums: two calls agree bit for bit."""
    q, k, v = inputs.random_case(4600, 1, 2, 700, D, D, torch.bfloat16, scale=D ** -0.5)
    dy = torch.randn(1, 2, 700, D, generator=torch.Generator().manual_seed(4601)).to(torch.bfloat16)
    lam = torch.tensor([0.9, 0.99])
    a = run(cuda_lib, q, k, v, dy, lam, 1e-6, False)
    b = run(cuda_lib, q, k, v, dy, lam, 1e-6, False)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
