"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle
on identical seeded inputs.

Gate per output tensor: max|gpu - oracle| / max|oracle| <= 2e-2 for bf16
inputs (fp32 state) and 1e-4 for fp32 inputs; no non-finite values.
Reduced sizes are compared element by element over every head; the full
workload sizes run in the launch configuration the benchmark times and are
compared on sampled heads (every token and every output of those heads).
"""
import numpy as np
import pytest
import torch

import oracle
from weight_state_recurrence_b200 import inputs
from weight_state_recurrence_b200.linattn import (LINATTN_KERNEL_CUDA_CORES,
                                                   LINATTN_KERNEL_TC_PAIRED, LINATTN_OP_CAUSAL,
                                                   LINATTN_OP_GLOBAL, kernel_choice)
from tests._compare import assert_close

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS
DEV = "cuda:0"


def run_causal(lib, q, k, v, lam, eps):
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    lamd = lam.to(DEV) if lam is not None else None
    out, S, z = lib.fwd_causal(qd, kd, vd, lamd, eps)
    torch.cuda.synchronize()
    return out, S, z


def check_causal(lib, q, k, v, lam, eps, tol, heads=None):
    out, S, z = run_causal(lib, q, k, v, lam, eps)
    if heads is None:
        y_o, S_o, z_o = oracle.causal(q, k, v, lam, eps)
        assert_close("y", out, y_o, tol)
        assert_close("S_final", S, S_o, tol)
        assert_close("z_final", z, z_o, tol)
        return
    for (b, h) in heads:
        lam_h = None if lam is None else lam[h:h + 1]
        sl = (slice(b, b + 1), slice(h, h + 1))
        y_o, S_o, z_o = oracle.causal(q[sl], k[sl], v[sl], lam_h, eps)
        assert_close(f"y[{b},{h}]", out[sl], y_o, tol)
        assert_close(f"S_final[{b},{h}]", S[sl], S_o, tol)
        assert_close(f"z_final[{b},{h}]", z[sl], z_o, tol)


def test_library_loads(cuda_lib):
    assert cuda_lib.linattn_version() >= 100
    assert cuda_lib.linattn_device_status(clear=True) == 0


# ------------------------------------------------------------ workload sizes
def test_tiny_f32_full(cuda_lib):
    w = W["tiny_f32"]
    q, k, v = inputs.causal_inputs(w)
    check_causal(cuda_lib, q, k, v, inputs.decay(w), w.eps, w.tol)


def test_causal_d64_full(cuda_lib):
    w = W["causal_d64"]
    q, k, v = inputs.causal_inputs(w)
    check_causal(cuda_lib, q, k, v, inputs.decay(w), w.eps, w.tol)


def test_causal_decay_d128_reduced(cuda_lib):
    w = W["causal_decay_d128"]
    # several chunks and a ragged tail, every head of a 2 x 16 batch
    q, k, v = inputs.causal_inputs(w, B=2, N=1000)
    check_causal(cuda_lib, q, k, v, inputs.decay(w), w.eps, w.tol)


def test_causal_decay_d128_full_sampled(cuda_lib):
    w = W["causal_decay_d128"]
    q, k, v = inputs.causal_inputs(w)
    heads = [(0, 0), (1, 7), (2, 15), (3, 3)]
    check_causal(cuda_lib, q, k, v, inputs.decay(w), w.eps, w.tol, heads=heads)


def test_global_d64_full(cuda_lib):
    w = W["global_d64"]
    q, k, v = inputs.causal_inputs(w)
    out, KV, ks = cuda_lib.fwd_global(q.to(DEV), k.to(DEV), v.to(DEV), w.eps)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (3, 5), (7, 11)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        y_o, KV_o, ks_o = oracle.global_attn(q[sl], k[sl], v[sl], w.eps)
        assert_close(f"y[{b},{h}]", out[sl], y_o, w.tol)
        assert_close(f"KV[{b},{h}]", KV[sl], KV_o, w.tol)
        assert_close(f"ksum[{b},{h}]", ks[sl], ks_o, w.tol)


def _decode_run(lib, w, B, steps, heads=None, N=None):
    """Prefill the decode state through the causal kernel, then run `steps`
    decode steps; compare every step's y and the final state with the oracle
    on the selected heads (all heads when `heads` is None)."""
    lam = inputs.decay(w)
    qp, kp, vp = inputs.causal_inputs(w, B=B, N=N)
    yp, S, z = lib.fwd_causal(qp.to(DEV), kp.to(DEV), vp.to(DEV), lam.to(DEV), w.eps)
    lamd = lam.to(DEV)
    if heads is None:
        sel = (slice(None), slice(None))
        lam_sel = lam
    else:
        bs, hs = zip(*heads)
        sel = (list(bs), list(hs))
        lam_sel = None
    # oracle prefix state for the selected heads
    if heads is None:
        _, S_o, z_o = oracle.causal(qp, kp, vp, lam, w.eps)
    else:
        S_o, z_o = [], []
        for b, h in heads:
            sl = (slice(b, b + 1), slice(h, h + 1))
            _, s_, z_ = oracle.causal(qp[sl], kp[sl], vp[sl], lam[h:h + 1], w.eps)
            S_o.append(s_[0, 0])
            z_o.append(z_[0, 0])
        S_o, z_o = np.stack(S_o)[None], np.stack(z_o)[None]
        lam_sel = torch.stack([lam[h] for _, h in heads])
    torch.cuda.synchronize()
    assert_close("prefix S", S[sel] if heads is not None else S, S_o[0] if heads is not None else S_o, w.tol)
    for s in range(steps):
        q, k, v = inputs.decode_step_inputs(w, s, B=B)
        y = lib.decode_step(q.to(DEV), k.to(DEV), v.to(DEV), S, z, lamd, w.eps)
        if heads is None:
            y_o, S_o, z_o = oracle.decode_step(q, k, v, S_o, z_o, lam, w.eps)
            assert_close(f"y step {s}", y, y_o, w.tol)
        else:
            qs, ks_, vs = q[sel][None], k[sel][None], v[sel][None]
            y_o, S_o, z_o = oracle.decode_step(qs, ks_, vs, S_o, z_o, lam_sel, w.eps)
            assert_close(f"y step {s}", y[sel][None], y_o, w.tol)
    torch.cuda.synchronize()
    if heads is None:
        assert_close("S after steps", S, S_o, w.tol)
        assert_close("z after steps", z, z_o, w.tol)
    else:
        assert_close("S after steps", S[sel][None], S_o, w.tol)
        assert_close("z after steps", z[sel][None], z_o, w.tol)


def test_decode_reduced_all_heads(cuda_lib):
    _decode_run(cuda_lib, W["decode_d128"], B=4, steps=48)


def test_decode_d128_as_stated(cuda_lib):
    """The decode workload exactly as stated: 256 sequences x 32 heads, the
    state prefilled from 512 tokens through the causal forward, then 1024
    decode steps, each launched over all 8192 heads (the benchmark's launch
    configuration).  Every step's y of five sampled heads, and their S, z
    after the last step, against the oracle."""
    w = W["decode_d128"]
    _decode_run(cuda_lib, w, B=w.B, steps=w.steps,
                heads=[(0, 0), (17, 31), (128, 5), (200, 9), (255, 16)])


# ------------------------------------------------------------ edge cases
@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 300])
@pytest.mark.parametrize("lamv", [0.0, 0.5, 0.97, 1.0])
def test_causal_tc_edges(cuda_lib, N, lamv):
    q, k, v = inputs.random_case(50 + N, 1, 2, N, 128, 128, torch.bfloat16, scale=0.3)
    lam = torch.tensor([lamv, 0.9], dtype=torch.float32)
    check_causal(cuda_lib, q, k, v, lam, 1e-6, 2e-2)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 32), (64, 64), (64, 32), (32, 128),
                                   (128, 64), (128, 16)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_causal_shapes(cuda_lib, dk, dv, dtype):
    q, k, v = inputs.random_case(dk * 3 + dv, 2, 3, 77, dk, dv, dtype, scale=dk ** -0.5)
    lam = torch.tensor([0.95, 1.0, 0.6], dtype=torch.float32)
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    check_causal(cuda_lib, q, k, v, lam, 1e-6, tol)


def test_causal_other_kernels_second_opinion(cuda_lib):
    """The CUDA-core kernel and the paired tensor-core kernel on the product
    kernel's inputs."""
    w = W["causal_decay_d128"]
    q, k, v = inputs.causal_inputs(w, B=1, H=4, N=700)
    lam = inputs.decay(w, H=4)
    out_tc, S_tc, z_tc = run_causal(cuda_lib, q, k, v, lam, w.eps)
    with kernel_choice(LINATTN_OP_CAUSAL, LINATTN_KERNEL_CUDA_CORES):
        out_s, S_s, z_s = run_causal(cuda_lib, q, k, v, lam, w.eps)
    with kernel_choice(LINATTN_OP_CAUSAL, LINATTN_KERNEL_TC_PAIRED):
        out_p, S_p, z_p = run_causal(cuda_lib, q, k, v, lam, w.eps)
    y_o, S_o, z_o = oracle.causal(q, k, v, lam, w.eps)
    for name, (y, S, z) in {"simt": (out_s, S_s, z_s), "tc": (out_tc, S_tc, z_tc),
                            "paired": (out_p, S_p, z_p)}.items():
        assert_close(f"y {name}", y, y_o, 2e-2)
        assert_close(f"S {name}", S, S_o, 2e-2)
        assert_close(f"z {name}", z, z_o, 2e-2)


def test_causal_empty_and_zero_heads(cuda_lib):
    q = torch.zeros(2, 3, 0, 128, dtype=torch.bfloat16, device=DEV)
    v = torch.zeros(2, 3, 0, 64, dtype=torch.bfloat16, device=DEV)
    out = torch.empty_like(v)
    S = torch.full((2, 3, 128, 64), 7.0, device=DEV)
    z = torch.full((2, 3, 128), 7.0, device=DEV)
    cuda_lib.linattn_fwd_causal(q, q, v, None, 1e-6, out, S, z)
    torch.cuda.synchronize()
    assert not S.any() and not z.any()
    q0 = torch.zeros(0, 3, 10, 128, dtype=torch.bfloat16, device=DEV)
    v0 = torch.zeros(0, 3, 10, 128, dtype=torch.bfloat16, device=DEV)
    cuda_lib.linattn_fwd_causal(q0, q0, v0, None, 1e-6, torch.empty_like(v0))


def test_prefill_then_decode_equals_prefill(cuda_lib):
    q, k, v = inputs.random_case(77, 2, 4, 300, 128, 128, torch.bfloat16, scale=128 ** -0.5)
    lam = torch.tensor([0.99, 0.9, 1.0, 0.5])
    lamd = lam.to(DEV)
    y_full, S_full, z_full = run_causal(cuda_lib, q, k, v, lam, 1e-6)
    n = 260
    y1, S, z = run_causal(cuda_lib, q[:, :, :n].contiguous(), k[:, :, :n].contiguous(),
                          v[:, :, :n].contiguous(), lam, 1e-6)
    ys = []
    for i in range(n, 300):
        ys.append(cuda_lib.decode_step(q[:, :, i].contiguous().to(DEV),
                                       k[:, :, i].contiguous().to(DEV),
                                       v[:, :, i].contiguous().to(DEV), S, z, lamd, 1e-6))
    torch.cuda.synchronize()
    y_o, S_o, z_o = oracle.causal(q, k, v, lam, 1e-6)
    assert_close("decode tail", torch.stack(ys, 2), y_o[:, :, n:], 2e-2)
    assert_close("S resume", S, S_o, 2e-2)
    assert_close("z resume", z, z_o, 2e-2)
    assert_close("S one-shot", S_full, S_o, 2e-2)


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (64, 16)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_global_shapes(cuda_lib, dk, dv, dtype):
    q, k, v = inputs.random_case(dk + dv, 2, 3, 1111, dk, dv, dtype, scale=dk ** -0.5)
    out, KV, ks = cuda_lib.fwd_global(q.to(DEV), k.to(DEV), v.to(DEV), 1e-6)
    torch.cuda.synchronize()
    y_o, KV_o, ks_o = oracle.global_attn(q, k, v, 1e-6)
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert_close("y", out, y_o, tol)
    assert_close("KV", KV, KV_o, tol)
    assert_close("ksum", ks, ks_o, tol)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 64), (128, 128), (128, 32)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_shapes(cuda_lib, dk, dv, dtype):
    B, H = 3, 5
    g = torch.Generator().manual_seed(dk * 7 + dv)
    S0 = torch.randn(B, H, dk, dv, generator=g) * 0.1
    z0 = torch.rand(B, H, dk, generator=g) + 0.5
    lam = torch.linspace(0.0, 1.0, H)
    S, z = S0.to(DEV), z0.to(DEV)
    lamd = lam.to(DEV)
    S_o, z_o = S0.double().numpy(), z0.double().numpy()
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    for s in range(5):
        q, k, v = inputs.qkv((B, H, dk), (B, H, dv), 900 + s, dk ** -0.5, dtype)
        y = cuda_lib.decode_step(q.to(DEV), k.to(DEV), v.to(DEV), S, z, lamd, 1e-6)
        y_o, S_o, z_o = oracle.decode_step(q, k, v, S_o, z_o, lam, 1e-6)
        assert_close(f"y step {s}", y, y_o, tol)
    assert_close("S", S, S_o, tol)
    assert_close("z", z, z_o, tol)


def test_convex_hull_on_gpu(cuda_lib):
    q, k, v = inputs.random_case(5, 1, 2, 400, 128, 128, torch.bfloat16, scale=0.2)
    lam = torch.tensor([0.9, 1.0])
    out, _, _ = run_causal(cuda_lib, q, k, v, lam, 0.0)
    vv = v.double()
    lo = torch.cummin(vv, dim=2).values
    hi = torch.cummax(vv, dim=2).values
    y = out.double().cpu()
    slack = 2e-2 * vv.abs().max()
    assert bool((y >= lo - slack).all()) and bool((y <= hi + slack).all())



@pytest.mark.parametrize("N", [1, 100, 128, 129, 1111, 4096])
def test_global_tc_edges(cuda_lib, N):
    """Tensor-core global path (bf16, d = 64, even H): ragged and tiny N."""
    q, k, v = inputs.random_case(300 + N, 2, 4, N, 64, 64, torch.bfloat16, scale=0.125)
    out, KV, ks = cuda_lib.fwd_global(q.to(DEV), k.to(DEV), v.to(DEV), 1e-6)
    torch.cuda.synchronize()
    y_o, KV_o, ks_o = oracle.global_attn(q, k, v, 1e-6)
    assert_close("y", out, y_o, 2e-2)
    assert_close("KV", KV, KV_o, 2e-2)
    assert_close("ksum", ks, ks_o, 2e-2)


def test_global_simt_second_opinion(cuda_lib):
    q, k, v = inputs.random_case(17, 1, 6, 3000, 64, 64, torch.bfloat16, scale=0.125)
    out_tc, KV_tc, _ = cuda_lib.fwd_global(q.to(DEV), k.to(DEV), v.to(DEV), 1e-6)
    with kernel_choice(LINATTN_OP_GLOBAL, LINATTN_KERNEL_CUDA_CORES):
        out_s, KV_s, _ = cuda_lib.fwd_global(q.to(DEV), k.to(DEV), v.to(DEV), 1e-6)
    torch.cuda.synchronize()
    y_o, KV_o, _ = oracle.global_attn(q, k, v, 1e-6)
    assert_close("y tc", out_tc, y_o, 2e-2)
    assert_close("y simt", out_s, y_o, 2e-2)
    assert_close("KV tc", KV_tc, KV_o, 2e-2)
    assert_close("KV simt", KV_s, KV_o, 1e-4)


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(clear=False) == 0
