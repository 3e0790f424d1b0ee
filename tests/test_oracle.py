"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: exact
rational arithmetic, the O(N^2) masked-weight form, the non-causal closed
form, library routines (ELU, matmul, cumsum) and invariants of the method.
The last group plants mistakes in a copy of the oracle's C source and checks
that the pins catch them.
"""
import json
import math
import os
import shutil
import subprocess
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from weight_state_recurrence_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def phi_np(x):
    # elu(x) + 1 via the library routine, in float64
    return (torch.nn.functional.elu(torch.as_tensor(x, dtype=torch.float64), alpha=1.0)
            + 1.0).numpy()


def brute_causal(q, k, v, lam, eps):
    """Masked-weight form ([FW] §3.1 triangular mask, [LN] §3 before the sum
    swap, decay unrolled): y_i = sum_{j<=i} w_ij v_j / (sum_{j<=i} w_ij + eps),
    w_ij = lam^(i-j) phi(q_i).phi(k_j)."""
    B, H, N, dk = q.shape
    y = np.zeros(v.shape[:-1] + (v.shape[-1],))
    for b in range(B):
        for h in range(H):
            L = 1.0 if lam is None else float(lam[h])
            fq, fk = phi_np(q[b, h]), phi_np(k[b, h])
            W = fq @ fk.T                                   # [N, N]
            i = np.arange(N)[:, None]
            j = np.arange(N)[None, :]
            dec = np.where(j <= i, np.power(L, np.maximum(i - j, 0).astype(np.float64)), 0.0)
            Wm = W * dec
            y[b, h] = (Wm @ v[b, h]) / (Wm.sum(1, keepdims=True) + eps)
    return y


def final_state(k, v, lam):
    """S_N = sum_j lam^(N-1-j) phi(k_j) v_j^T as a weighted GEMM and
    z_N = sum_j lam^(N-1-j) phi(k_j)."""
    B, H, N, dk = k.shape
    S = np.zeros((B, H, dk, v.shape[-1]))
    z = np.zeros((B, H, dk))
    for b in range(B):
        for h in range(H):
            L = 1.0 if lam is None else float(lam[h])
            w = np.power(L, (N - 1 - np.arange(N)).astype(np.float64))
            fk = phi_np(k[b, h])
            S[b, h] = (fk * w[:, None]).T @ v[b, h]
            z[b, h] = (fk * w[:, None]).sum(0)
    return S, z


def rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def rand(seed, B, H, N, dk, dv, scale=1.0):
    q, k, v = inputs.random_case(seed, B, H, N, dk, dv, scale=scale)
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


# --------------------------------------------------------------------------
def test_golden_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_n2_d4.json")))
    q = np.array(g["q"], float)[None, None]
    k = np.array(g["k"], float)[None, None]
    v = np.array(g["v"], float)[None, None]
    lam = np.array([g["lambda"]])
    y, S, z = oracle.causal(q, k, v, lam, eps=g["eps"])
    assert np.allclose(y[0, 0], g["causal_y"], rtol=0, atol=1e-15)
    assert np.allclose(S[0, 0], g["causal_S"], rtol=0, atol=1e-15)
    assert np.allclose(z[0, 0], g["causal_z"], rtol=0, atol=1e-15)
    yg, KV, ks = oracle.global_attn(q, k, v, eps=g["eps"])
    assert np.allclose(yg[0, 0], g["global_y"], rtol=0, atol=1e-15)
    assert np.allclose(KV[0, 0], g["global_KV"], rtol=0, atol=1e-15)
    assert np.allclose(ks[0, 0], g["global_ks"], rtol=0, atol=1e-15)


def test_feature_map_is_elu_plus_one():
    x = np.concatenate([np.linspace(-40, 40, 4001), [0.0, -0.0, 1e-300, -1e-300, -745.0,
                                                     -800.0, 1e6]])
    got = oracle.feature_map(x)
    ref = phi_np(x)   # library elu(x)+1 = (exp(x)-1)+1: absolute accuracy near 0
    assert np.all(got >= 0)
    assert np.all(np.abs(got - ref) <= 4e-16 * np.maximum(np.abs(ref), 1.0))
    # for x <= 0 the oracle takes exp(x) directly: relative accuracy everywhere
    neg = x <= 0
    e = np.array([math.exp(t) for t in x[neg]])
    nz = e > 0
    assert np.all(np.abs(got[neg][nz] - e[nz]) <= 2e-16 * e[nz])
    assert np.all(got[neg][~nz] == 0.0)
    # for x > 0 it is exactly x + 1
    assert np.array_equal(got[~neg], x[~neg] + 1.0)
    # the two branches meet at 0 (phi(0) = 1) and phi is positive there
    assert oracle.feature_map(np.array([0.0]))[0] == 1.0


@pytest.mark.parametrize("N", [1, 2, 3, 7, 64])
@pytest.mark.parametrize("d", [4, 8, 32])
@pytest.mark.parametrize("lamv", [0.0, 0.5, 0.9, 1.0])
def test_causal_matches_masked_bruteforce(N, d, lamv):
    q, k, v = rand(100 + N * 7 + d, 2, 3, N, d, d)
    lam = np.array([lamv, 1.0, 0.3 * lamv + 0.2])
    for eps in (0.0, 1e-6):
        y, S, z = oracle.causal(q, k, v, lam, eps=eps)
        assert rel(y, brute_causal(q, k, v, lam, eps)) < 1e-12
        S_ref, z_ref = final_state(k, v, lam)
        assert rel(S, S_ref) < 1e-12
        assert rel(z, z_ref) < 1e-12


def test_causal_dk_ne_dv():
    q, k, v = rand(7, 1, 2, 33, 8, 5)
    lam = np.array([0.8, 1.0])
    y, S, z = oracle.causal(q, k, v, lam, eps=1e-6)
    assert y.shape == (1, 2, 33, 5) and S.shape == (1, 2, 8, 5) and z.shape == (1, 2, 8)
    assert rel(y, brute_causal(q, k, v, lam, 1e-6)) < 1e-12


def _frac_phi(x):
    assert x >= 0
    return x + 1 if x > 0 else Fraction(1)


def test_causal_exact_rational():
    """Exact brute force in rational arithmetic; inputs >= 0 keep phi exact."""
    rng = np.random.default_rng(11)
    N, dk, dv = 9, 3, 4
    qi = rng.integers(0, 4, (N, dk))
    ki = rng.integers(0, 4, (N, dk))
    vi = rng.integers(-5, 6, (N, dv))
    lamF, epsF = Fraction(3, 4), Fraction(1, 1000)
    fq = [[_frac_phi(Fraction(int(a))) for a in r] for r in qi]
    fk = [[_frac_phi(Fraction(int(a))) for a in r] for r in ki]
    y_exact = []
    for i in range(N):
        num = [Fraction(0)] * dv
        den = Fraction(0)
        for j in range(i + 1):
            w = lamF ** (i - j) * sum(a * b for a, b in zip(fq[i], fk[j]))
            den += w
            for c in range(dv):
                num[c] += w * int(vi[j][c])
        y_exact.append([n / (den + epsF) for n in num])
    y, _, _ = oracle.causal(qi[None, None].astype(float), ki[None, None].astype(float),
                            vi[None, None].astype(float), np.array([0.75]), eps=0.001)
    ref = np.array([[float(t) for t in r] for r in y_exact])
    assert rel(y[0, 0], ref) < 1e-14


def test_global_closed_form_and_reorder():
    q, k, v = rand(21, 2, 2, 50, 8, 6)
    eps = 1e-6
    y, KV, ks = oracle.global_attn(q, k, v, eps=eps)
    for b in range(2):
        for h in range(2):
            fq, fk = phi_np(q[b, h]), phi_np(k[b, h])
            W = fq @ fk.T                          # un-reordered pairwise weights
            y_ref = (W @ v[b, h]) / (W.sum(1, keepdims=True) + eps)
            assert rel(y[b, h], y_ref) < 1e-12
            assert rel(KV[b, h], fk.T @ v[b, h]) < 1e-12   # phi(K)^T V
            assert rel(ks[b, h], fk.sum(0)) < 1e-12


def test_global_cross_brute_force():
    """Nq queries against Nk keys of another sequence: the double sum
    y_i = sum_j (phi(q_i).phi(k_j)) v_j / (sum_j phi(q_i).phi(k_j) + eps), and
    Nq = Nk reduces to the self form."""
    q, _, _ = rand(21, 2, 3, 7, 5, 4)
    _, k, v = rand(22, 2, 3, 11, 5, 4)
    eps = 1e-3
    y, KV, ks = oracle.global_cross(q, k, v, eps)
    fq, fk = phi_np(q), phi_np(k)
    w = np.einsum("bhid,bhjd->bhij", fq, fk)
    assert rel(y, np.einsum("bhij,bhjv->bhiv", w, v) / (w.sum(-1, keepdims=True) + eps)) < 1e-13
    assert rel(KV, np.einsum("bhjd,bhjv->bhdv", fk, v)) < 1e-13 and rel(ks, fk.sum(2)) < 1e-13
    y2, _, _ = oracle.global_cross(q, q, v[:, :, :7], eps)
    y3, _, _ = oracle.global_attn(q, q, v[:, :, :7], eps)
    assert np.array_equal(y2, y3)
    y0, KV0, ks0 = oracle.global_cross(q, k[:, :, :0], v[:, :, :0], eps)
    assert not y0.any() and not KV0.any() and not ks0.any()


def test_global_masked_pins():
    """Key padding mask ([LN] §6 key_padding_mask): the double sum over the
    keys that are not padding; the same as the cross form on those keys alone
    (per sequence); no padding gives the cross form; all padding gives
    KV = ks = 0 and y = 0."""
    q, _, _ = rand(23, 3, 2, 6, 5, 4)
    _, k, v = rand(24, 3, 2, 13, 5, 4)
    eps = 1e-3
    pad = np.zeros((3, 13), dtype=np.uint8)
    pad[0, [0, 4, 12]] = 1          # a few padding keys
    pad[1, 7:] = 1                  # a padded tail
    pad[2, :] = 1                   # all padding
    y, KV, ks = oracle.global_masked(q, k, v, pad, eps)
    fq, fk = phi_np(q), phi_np(k)
    keep = (pad == 0).astype(np.float64)[:, None, :]          # [B, 1, Nk]
    w = np.einsum("bhid,bhjd->bhij", fq, fk) * keep[:, :, None, :]
    assert rel(y, np.einsum("bhij,bhjv->bhiv", w, v) / (w.sum(-1, keepdims=True) + eps)) < 1e-13
    assert rel(KV, np.einsum("bhjd,bhjv->bhdv", fk * keep[..., None], v)) < 1e-13
    assert rel(ks, (fk * keep[..., None]).sum(2)) < 1e-13
    for b in range(2):
        idx = np.nonzero(pad[b] == 0)[0]
        yc, KVc, ksc = oracle.global_cross(q[b:b + 1], k[b:b + 1, :, idx], v[b:b + 1, :, idx], eps)
        assert rel(y[b:b + 1], yc) < 1e-14 and rel(KV[b:b + 1], KVc) < 1e-14
        assert rel(ks[b:b + 1], ksc) < 1e-14
    assert not KV[2].any() and not ks[2].any() and not y[2].any()
    y0, KV0, ks0 = oracle.global_masked(q, k, v, None, eps)
    yx, KVx, ksx = oracle.global_cross(q, k, v, eps)
    assert np.array_equal(y0, yx) and np.array_equal(KV0, KVx) and np.array_equal(ks0, ksx)


def test_causal_last_token_equals_global_without_decay():
    q, k, v = rand(5, 1, 3, 40, 8, 8)
    y, S, z = oracle.causal(q, k, v, None, eps=1e-6)
    yg, KV, ks = oracle.global_attn(q, k, v, eps=1e-6)
    assert rel(y[:, :, -1], yg[:, :, -1]) < 1e-13
    assert rel(S, KV) < 1e-13 and rel(z, ks) < 1e-13


@pytest.mark.parametrize("lamv", [0.0, 0.7, 1.0])
def test_convex_hull_invariant(lamv):
    q, k, v = rand(9, 1, 2, 60, 8, 8)
    lam = np.array([lamv, lamv])
    y, _, _ = oracle.causal(q, k, v, lam, eps=0.0)
    lo = np.minimum.accumulate(v, axis=2)
    hi = np.maximum.accumulate(v, axis=2)
    tol = 1e-12 * np.max(np.abs(v))
    assert np.all(y >= lo - tol) and np.all(y <= hi + tol)
    # with eps > 0 the output is W/(W+eps) times a hull point: the hull
    # widened to include 0
    y2, _, _ = oracle.causal(q, k, v, lam, eps=0.5)
    assert np.all(y2 >= np.minimum(lo, 0) - tol) and np.all(y2 <= np.maximum(hi, 0) + tol)


def test_decode_loop_equals_causal_bitwise():
    q, k, v = rand(3, 2, 2, 12, 8, 8)
    lam = np.array([0.9, 1.0])
    y, S, z = oracle.causal(q, k, v, lam, eps=1e-6)
    St = np.zeros((2, 2, 8, 8))
    zt = np.zeros((2, 2, 8))
    for i in range(12):
        yi, St, zt = oracle.decode_step(q[:, :, i], k[:, :, i], v[:, :, i], St, zt, lam, 1e-6)
        assert np.array_equal(yi, y[:, :, i])
    assert np.array_equal(St, S) and np.array_equal(zt, z)


def test_prefill_then_decode_equals_prefill():
    q, k, v = rand(4, 1, 2, 20, 8, 8)
    lam = np.array([0.95, 0.5])
    y, S, z = oracle.causal(q, k, v, lam, eps=1e-6)
    n = 13
    y1, S1, z1 = oracle.causal(q[:, :, :n], k[:, :, :n], v[:, :, :n], lam, eps=1e-6)
    y2, S2, z2 = oracle.causal(q[:, :, n:], k[:, :, n:], v[:, :, n:], lam, eps=1e-6,
                               S0=S1, z0=z1)
    assert np.array_equal(np.concatenate([y1, y2], 2), y)
    assert np.array_equal(S2, S) and np.array_equal(z2, z)


def test_initial_state_single_token_closed_form():
    """One token from a given (S0, z0): S1 = lam S0 + phi(k) v^T, z1 = lam z0 +
    phi(k), y = phi(q) S1 / (phi(q) z1 + eps), written out with numpy."""
    q, k, v = rand(13, 1, 1, 1, 6, 4)
    rng = np.random.default_rng(14)
    S0 = rng.standard_normal((1, 1, 6, 4))
    z0 = rng.random((1, 1, 6)) + 0.5
    lam, eps = 0.8, 1e-3
    y, S, z = oracle.causal(q, k, v, np.array([lam]), eps=eps, S0=S0, z0=z0)
    fq, fk = phi_np(q[0, 0, 0]), phi_np(k[0, 0, 0])
    S1 = lam * S0[0, 0] + np.outer(fk, v[0, 0, 0])
    z1 = lam * z0[0, 0] + fk
    assert rel(S[0, 0], S1) < 1e-14 and rel(z[0, 0], z1) < 1e-14
    assert rel(y[0, 0, 0], fq @ S1 / (fq @ z1 + eps)) < 1e-14


def test_single_token_and_constant_values():
    q, k, v = rand(8, 1, 1, 1, 8, 4)
    eps = 1e-3
    y, _, _ = oracle.causal(q, k, v, None, eps=eps)
    w = float(phi_np(q[0, 0, 0]) @ phi_np(k[0, 0, 0]))
    assert rel(y[0, 0, 0], v[0, 0, 0] * w / (w + eps)) < 1e-14
    # constant values: y_i = c W_i / (W_i + eps)
    q, k, _ = rand(9, 1, 1, 30, 8, 4)
    c = np.array([1.5, -2.0, 0.25, 3.0])
    v = np.broadcast_to(c, (1, 1, 30, 4)).copy()
    lam = np.array([0.8])
    y, _, _ = oracle.causal(q, k, v, lam, eps=eps)
    fq, fk = phi_np(q[0, 0]), phi_np(k[0, 0])
    for i in range(30):
        Wi = sum(0.8 ** (i - j) * float(fq[i] @ fk[j]) for j in range(i + 1))
        assert rel(y[0, 0, i], c * Wi / (Wi + eps)) < 1e-13


def test_cumsum_form_without_decay():
    """[FW] §4.1 trains with a cumsum of outer products (no decay); restated
    in torch fp64 with the normaliser, it must agree with the recurrence."""
    q, k, v = rand(12, 1, 2, 25, 6, 5)
    eps = 1e-6
    y, _, _ = oracle.causal(q, k, v, None, eps=eps)
    for h in range(2):
        fq = torch.nn.functional.elu(torch.tensor(q[0, h])) + 1
        fk = torch.nn.functional.elu(torch.tensor(k[0, h])) + 1
        vv = torch.tensor(v[0, h])
        S = torch.cumsum(fk[:, :, None] * vv[:, None, :], dim=0)     # [N, dk, dv]
        zc = torch.cumsum(fk, dim=0)
        num = torch.einsum("nd,ndv->nv", fq, S)
        den = (fq * zc).sum(-1, keepdim=True) + eps
        assert rel(y[0, h], (num / den).numpy()) < 1e-12


def test_empty_sequence_gives_initial_state():
    q = np.zeros((1, 2, 0, 4))
    v = np.zeros((1, 2, 0, 3))
    y, S, z = oracle.causal(q, q, v, None)
    assert y.shape == (1, 2, 0, 3) and not S.any() and not z.any()


# --------------------------------------------------------------------------
# Planted mistakes: each mutation of the oracle's source must be caught by
# the brute-force / closed-form pins above.
MUTATIONS = {
    "decay_not_applied_to_z": ("z[a] = lam * z[a] + fk[a];", "z[a] = z[a] + fk[a];"),
    "read_before_update": None,  # handled by moving the read (exclusive output)
    "phi_minus_one": ("return x > 0.0 ? x + 1.0 : exp(x);", "return x > 0.0 ? x : exp(x);"),
    "eps_dropped": ("den += c->eps;\n            double *yi = y",
                    "double *yi = y"),
    "state_transposed": ("Sa[b] = lam * Sa[b] + fk[a] * vi[b];",
                         "Sa[b] = lam * Sa[b] + fk[b % dk] * vi[a % dv];"),
    "global_missing_ks": ("ks[a] += f[a];", "ks[a] += 1.0;"),
}


def _build_mutant(tmp_path, name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "linattn_oracle.c")).read()
    if name == "read_before_update":
        a = "        /* state update: decay, then add the outer product phi(k_i) v_i^T */"
        b = "        /* read: numerator phi(q_i)^T S_i and denominator phi(q_i)^T z_i + eps */"
        i0, i1 = src.index(a), src.index(b)
        i2 = src.index("    }\n    if (c->S_out)", i1)
        upd, read = src[i0:i1], src[i1:i2]
        src = src[:i0] + read + upd + src[i2:]
    else:
        old, new = MUTATIONS[name]
        assert old in src, name
        src = src.replace(old, new)
    d = tmp_path / name
    d.mkdir()
    shutil.copy(os.path.join(os.path.dirname(oracle.__file__), "__init__.py"), d / "__init__.py")
    (d / "linattn_oracle.c").write_text(src)
    import importlib.util
    spec = importlib.util.spec_from_file_location(f"mutant_{name}", d / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistakes(tmp_path, name):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    m = _build_mutant(tmp_path, name)
    q, k, v = rand(31, 1, 2, 16, 6, 6, scale=0.7)
    lam = np.array([0.8, 0.6])
    eps = 0.05
    caught = False
    y, S, z = m.causal(q, k, v, lam, eps=eps)
    caught |= rel(y, brute_causal(q, k, v, lam, eps)) > 1e-9
    S_ref, z_ref = final_state(k, v, lam)
    caught |= rel(S, S_ref) > 1e-9 or rel(z, z_ref) > 1e-9
    yg, KV, ks = m.global_attn(q, k, v, eps=eps)
    fk = phi_np(k[0, 0])
    caught |= rel(ks[0, 0], fk.sum(0)) > 1e-9
    assert caught, f"mutation {name} went unnoticed"
