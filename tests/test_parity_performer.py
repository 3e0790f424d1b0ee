"""GPU parity of the Performer path (linear-attention note §4.2): the random
feature kernels against the fp64 feature oracle, and the attention calls in
identity mode (dims.phi = LINATTN_PHI_IDENTITY) on those features against the
numpy recurrence on features, from raw q, k, v and omega.

The inputs follow the Performer workload recipe (q, k with scale 1/(2 sqrt d),
orthogonal omega), where the trig estimate is well conditioned; extra cases
use larger inputs so the arguments omega.x reach tens of radians."""
import math

import numpy as np
import pytest
import torch

from oracle import performer as P
from weight_state_recurrence_b200 import inputs
from weight_state_recurrence_b200.linattn import (LINATTN_KERNEL_AUTO, LINATTN_KERNEL_CUDA_CORES,
                                                   LINATTN_OP_PERFORMER, kernel_choice)
from tests._compare import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
IDENT = 1
KERNELS = {"softmax": 0, "gaussian": 1}
# Features are bounded by their row's scale g(x)/sqrt(m) and rounded once to
# bf16 (relative 2^-9); omega.x is accumulated in fp32 from the same bf16
# values the oracle sees, and sin/cos are good to ~4e-7.  So the error of a
# feature is a few 1e-3 of the row scale: gate 5e-3 of the largest feature.
BF16_FEAT_TOL = 5e-3


def draw(seed, shape, scale, dtype):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(dtype)


# --------------------------------------------------------------- features
def check_features(lib, rows, d, m, kernel, dtype, scale, seed, tol, simt=False):
    x = draw(seed, (rows, d), scale, dtype)
    w = inputs.performer_omega(m, d, seed + 1, True, dtype)
    with kernel_choice(LINATTN_OP_PERFORMER,
                       LINATTN_KERNEL_CUDA_CORES if simt else LINATTN_KERNEL_AUTO):
        f = lib.performer_features(x.to(DEV), w.to(DEV), KERNELS[kernel])
    torch.cuda.synchronize()
    assert f.shape == (rows, 2 * m) and f.dtype == dtype
    if rows:
        assert_close(f"features {kernel}", f, P.features(x, w, kernel), tol)


@pytest.mark.parametrize("d,m", [(128, 64), (128, 32), (64, 64), (64, 32)])
@pytest.mark.parametrize("kernel", ["softmax", "gaussian"])
def test_tensor_core_features(cuda_lib, d, m, kernel):
    # 1000 rows: 7 full tiles of 128 and a ragged tail of 104
    check_features(cuda_lib, 1000, d, m, kernel, torch.bfloat16, 0.5 / math.sqrt(d),
                   2000 + d + m, BF16_FEAT_TOL)


@pytest.mark.parametrize("scale", [1.0, 8.0])
def test_tensor_core_features_large_arguments(cuda_lib, scale):
    # d = 128: omega.x ~ N(0, 128 scale^2), tens (scale 1) to hundreds (scale 8)
    # of radians, through every quadrant of the argument reduction
    check_features(cuda_lib, 777, 128, 64, "gaussian", torch.bfloat16, scale, 2100, BF16_FEAT_TOL)


def test_tensor_core_features_many_tiles(cuda_lib):
    # more tiles than CTAs: every CTA walks its range through the whole ring
    check_features(cuda_lib, 148 * 128 * 5 + 3, 128, 64, "softmax", torch.bfloat16,
                   0.5 / math.sqrt(128), 2200, BF16_FEAT_TOL)


@pytest.mark.parametrize("d,m,dtype,tol", [(32, 16, torch.bfloat16, BF16_FEAT_TOL),
                                           (128, 8, torch.bfloat16, BF16_FEAT_TOL),
                                           (64, 64, torch.float32, 1e-4),
                                           (16, 32, torch.float32, 1e-4)])
def test_cuda_core_features(cuda_lib, d, m, dtype, tol):
    check_features(cuda_lib, 333, d, m, "softmax", dtype, 0.5 / math.sqrt(d), 2300 + d + m, tol)
    check_features(cuda_lib, 333, d, m, "gaussian", dtype, 1.0, 2400 + d + m, tol)


def test_forced_cuda_core_features_bf16(cuda_lib):
    check_features(cuda_lib, 500, 128, 64, "softmax", torch.bfloat16, 0.5 / math.sqrt(128), 2500,
                   BF16_FEAT_TOL, simt=True)


def test_zero_rows(cuda_lib):
    check_features(cuda_lib, 0, 128, 64, "softmax", torch.bfloat16, 1.0, 2600, 2e-2)


# ------------------------------------------------------- attention on features
def perf_case(B, H, N, d, m, dv, dtype, seed):
    q = draw(seed, (B, H, N, d), 0.5 / math.sqrt(d), dtype)
    k = draw(seed + 1, (B, H, N, d), 0.5 / math.sqrt(d), dtype)
    v = draw(seed + 2, (B, H, N, dv), 1 / math.sqrt(dv), dtype)
    w = inputs.performer_omega(m, d, seed + 3, True, dtype)
    return q, k, v, w


@pytest.mark.parametrize("dv,lam", [(128, "decay"), (64, "decay"), (128, None)])
def test_performer_causal_tensor_core(cuda_lib, dv, lam):
    # m = 64: 128 features, so the bf16 causal kernel runs on the tensor cores
    B, H, N = 2, 2, 700
    q, k, v, w = perf_case(B, H, N, 128, 64, dv, torch.bfloat16, 2700 + dv)
    L = torch.tensor([0.95, 0.999]) if lam else None
    out, S, z = cuda_lib.performer_causal(q.to(DEV), k.to(DEV), v.to(DEV), w.to(DEV),
                                          None if L is None else L.to(DEV), 1e-6)
    torch.cuda.synchronize()
    y_o, S_o, z_o = P.causal_feat(P.features(q, w), P.features(k, w), v, L, 1e-6)
    assert_close("y", out, y_o, 2e-2)
    assert_close("S", S, S_o, 2e-2)
    assert_close("z", z, z_o, 2e-2)


@pytest.mark.parametrize("kernel", ["softmax", "gaussian"])
def test_performer_causal_fp32(cuda_lib, kernel):
    B, H, N = 1, 3, 300
    q, k, v, w = perf_case(B, H, N, 64, 32, 32, torch.float32, 2800)
    L = torch.tensor([0.9, 0.99, 1.0])
    fq = cuda_lib.performer_features(q.to(DEV), w.to(DEV), KERNELS[kernel])
    fk = cuda_lib.performer_features(k.to(DEV), w.to(DEV), KERNELS[kernel])
    out, S, z = cuda_lib.fwd_causal(fq, fk, v.to(DEV), L.to(DEV), 1e-6, phi=IDENT)
    torch.cuda.synchronize()
    y_o, S_o, z_o = P.causal_feat(P.features(q, w, kernel), P.features(k, w, kernel), v, L, 1e-6)
    assert_close("y", out, y_o, 1e-4)
    assert_close("S", S, S_o, 1e-4)
    assert_close("z", z, z_o, 1e-4)


def test_identity_causal_segmented_with_signed_features(cuda_lib):
    # few heads and a long sequence: the segment-parallel CUDA-core path, on
    # arbitrary signed features (eps large enough to keep the denominator away
    # from zero)
    B, H, N, f, dv = 1, 2, 3000, 32, 32
    fq = draw(2900, (B, H, N, f), 1.0, torch.float32).abs() * 0.2 + draw(2901, (B, H, N, f), 0.05,
                                                                          torch.float32)
    fk = draw(2902, (B, H, N, f), 1.0, torch.float32).abs() * 0.2 + draw(2903, (B, H, N, f), 0.05,
                                                                          torch.float32)
    v = draw(2904, (B, H, N, dv), 1.0, torch.float32)
    L = torch.tensor([0.999, 0.9])
    S0 = draw(2905, (B, H, f, dv), 0.1, torch.float32)
    z0 = draw(2906, (B, H, f), 0.1, torch.float32).abs() + 1.0
    assert cuda_lib.linattn_fwd_causal_workspace(B, H, N, f, dv, torch.float32, IDENT) > 0
    out, S, z = cuda_lib.fwd_causal(fq.to(DEV), fk.to(DEV), v.to(DEV), L.to(DEV), 0.5,
                                    S_init=S0.to(DEV), z_init=z0.to(DEV), phi=IDENT)
    torch.cuda.synchronize()
    y_o, S_o, z_o = P.causal_feat(fq, fk, v, L, 0.5, S0, z0)
    assert_close("y", out, y_o, 1e-4)
    assert_close("S", S, S_o, 1e-4)
    assert_close("z", z, z_o, 1e-4)


@pytest.mark.parametrize("dtype,d,m,tol", [(torch.bfloat16, 64, 32, 2e-2),
                                           (torch.float32, 32, 16, 1e-4)])
def test_performer_global(cuda_lib, dtype, d, m, tol):
    # bf16 with 64 features and dv = 64 (an even head count) runs on the tensor cores
    B, H, Nq, Nk = 2, 2, 300, 900
    q, _, _, w = perf_case(B, H, Nq, d, m, 2 * m, dtype, 3000 + d)
    _, k, v, _ = perf_case(B, H, Nk, d, m, 2 * m, dtype, 3100 + d)
    fq = cuda_lib.performer_features(q.to(DEV), w.to(DEV))
    fk = cuda_lib.performer_features(k.to(DEV), w.to(DEV))
    out, KV, ks = cuda_lib.fwd_global_cross(fq, fk, v.to(DEV), 1e-6, phi=IDENT)
    torch.cuda.synchronize()
    y_o, KV_o, ks_o = P.global_feat(P.features(q, w), P.features(k, w), v, 1e-6)
    assert_close("y", out, y_o, tol)
    assert_close("KV", KV, KV_o, tol)
    assert_close("ksum", ks, ks_o, tol)


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, 2e-2), (torch.float32, 1e-4)])
def test_performer_decode(cuda_lib, dtype, tol):
    B, H, d, m, dv = 3, 4, 128, 64, 64
    q, k, v, w = perf_case(B, H, 5, d, m, dv, dtype, 3200)
    L = torch.linspace(0.9, 1.0, H)
    fq_all = P.features(q, w)
    fk_all = P.features(k, w)
    S = torch.zeros(B, H, 2 * m, dv, device=DEV)
    z = torch.zeros(B, H, 2 * m, device=DEV)
    S_o = np.zeros((B, H, 2 * m, dv))
    z_o = np.zeros((B, H, 2 * m))
    for t in range(5):
        fq = cuda_lib.performer_features(q[:, :, t].contiguous().to(DEV), w.to(DEV))
        fk = cuda_lib.performer_features(k[:, :, t].contiguous().to(DEV), w.to(DEV))
        y = cuda_lib.decode_step(fq, fk, v[:, :, t].contiguous().to(DEV), S, z, L.to(DEV), 1e-6,
                                 phi=IDENT)
        y_o, S_o, z_o = P.decode_feat(fq_all[:, :, t], fk_all[:, :, t], v[:, :, t], S_o, z_o, L,
                                      1e-6)
        torch.cuda.synchronize()
        assert_close(f"y step {t}", y, y_o, tol)
    assert_close("S", S, S_o, tol)
    assert_close("z", z, z_o, tol)


def test_performer_full_size_sampled_rows(cuda_lib):
    """The Performer workload at full size (4 x 16 heads, 16384 tokens, d =
    128, m = 64), in the configuration the benchmark times; y checked on
    sampled rows of three heads against the unrolled sum on their features."""
    q, k, v, lam, w = inputs.performer_inputs("performer_d128", device=DEV)
    out, S, z = cuda_lib.performer_causal(q, k, v, w, lam.to(DEV), 1e-6, want_state=False)
    torch.cuda.synchronize()
    w_c = w.cpu()
    N = q.shape[2]
    heads = [(0, 0), (1, 7), (3, 15)]
    idx = [0, 1, 127, 128, 129, 4095, N - 129, N - 1]
    for b, h in heads:
        fq = P.features(q[b, h].cpu(), w_c)[None, None]
        fk = P.features(k[b, h].cpu(), w_c)[None, None]
        vh = v[b, h].cpu()[None, None]
        ref = P.causal_feat_rows(fq, fk, vh, lam[h:h + 1].numpy(), 1e-6, [(0, 0, i) for i in idx])
        assert_close(f"y head {(b, h)}", out[b, h, idx], ref, 2e-2)


@pytest.mark.parametrize("dtype,tol", [(torch.float32, 1e-4), (torch.bfloat16, 2e-2)])
def test_identity_backward(cuda_lib, dtype, tol):
    """Gradients with respect to the features (phi = identity) against the
    gradient oracle in identity mode, on Performer features of seeded q, k."""
    B, H, N, d, m, dv = 1, 2, 150, 64, 32, 32
    q, k, v, w = perf_case(B, H, N, d, m, dv, torch.float32, 3300)
    fq = torch.as_tensor(P.features(q, w)).to(dtype)
    fk = torch.as_tensor(P.features(k, w)).to(dtype)
    v = v.to(dtype)
    dy = draw(3301, (B, H, N, dv), 1.0, dtype)
    L = torch.tensor([0.97, 1.0])
    dq, dk, dvv, dl = cuda_lib.bwd_causal(fq.to(DEV), fk.to(DEV), v.to(DEV), dy.to(DEV),
                                          L.to(DEV), 1e-6, want_dlam=True, phi=IDENT)
    torch.cuda.synchronize()
    from oracle import grad as og
    _, dq_o, dk_o, dv_o, dl_o = og.causal_grad(fq, fk, v, L, 1e-6, dy, identity=True)
    assert_close("dq", dq, dq_o, tol)
    assert_close("dk", dk, dk_o, tol)
    assert_close("dv", dvv, dv_o, tol)
    assert_close("dlambda", dl, dl_o, tol)


def test_no_device_errors_recorded(cuda_lib):
    assert cuda_lib.linattn_device_status(True) == 0
