"""Pins for the Performer oracle (CPU only).

The feature map is pinned by what the linear-attention note §4.2 says it is
for: with many random features, phi(x).phi(y) must converge to exp(x.y)
(h = 1) or to the Gaussian kernel exp(-|x-y|^2/2) (h(x) = exp(-|x|^2/2)),
within a bound computed from the estimator's exact variance.  An exact
special case (a scaled permutation as omega, x = 0) pins the layout.  The
attention-on-features functions are pinned against the C oracle by feeding
them elu + 1 features, and end to end against softmax-kernel attention.
The last test plants plausible mistakes in copies of the feature map and
checks that the pins catch each one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import performer as P
from weight_state_recurrence_b200 import inputs


def elu1(x):
    return (torch.nn.functional.elu(torch.as_tensor(x, dtype=torch.float64)) + 1.0).numpy()


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------ feature map
def pin_layout(feat):
    """omega = 2 * (rows of a 5-cycle permutation matrix), m = d = 5: phi_l is
    g/sqrt(5) cos(2 x_pi(l)) for l < 5 and the sines after, computed with
    scalar math.cos/math.sin/math.exp; x = 0 gives [1/sqrt(m)] * m then zeros."""
    d = 5
    perm = [2, 4, 1, 0, 3]
    w = np.zeros((d, d))
    for l, c in enumerate(perm):
        w[l, c] = 2.0
    x = np.array([0.3, -0.7, 0.25, 1.1, -0.4])
    n2 = sum(t * t for t in x)
    ok = True
    for kernel, g in (("softmax", math.exp(n2 / 2)), ("gaussian", 1.0)):
        want = [g / math.sqrt(d) * math.cos(2 * x[c]) for c in perm] + \
               [g / math.sqrt(d) * math.sin(2 * x[c]) for c in perm]
        ok &= np.allclose(feat(x, w, kernel), want, rtol=1e-13, atol=1e-15)
        z = feat(np.zeros(d), w, kernel)
        ok &= np.allclose(z, [1 / math.sqrt(d)] * d + [0.0] * d, rtol=0, atol=1e-15)
    return bool(ok)


def _mc_pairs():
    r = _rng(11)
    d = 6
    return d, [(0.35 * r.standard_normal(d), 0.35 * r.standard_normal(d)) for _ in range(3)]


def pin_softmax_limit(feat, orthogonal):
    """phi(x).phi(y) -> exp(x.y) with m = 120000 features.  The estimate is
    G/m sum_l cos(omega_l.(x-y)), G = exp((|x|^2+|y|^2)/2); for iid omega its
    standard deviation is G (1 - exp(-s2)) / sqrt(2m), s2 = |x-y|^2; the
    orthogonal draw has no larger variance.  Gate: 8 sigma."""
    d, pairs = _mc_pairs()
    m = 120000
    w = inputs.performer_omega(m, d, 21, orthogonal, torch.float64).numpy()
    for x, y in pairs:
        est = float(feat(x, w, "softmax") @ feat(y, w, "softmax"))
        s2 = float(np.sum((x - y) ** 2))
        G = math.exp((x @ x + y @ y) / 2)
        sigma = G * (1 - math.exp(-s2)) / math.sqrt(2 * m)
        if not abs(est - math.exp(float(x @ y))) < 8 * sigma:
            return False
    return True


def pin_gaussian_limit(feat, orthogonal):
    """phi(x).phi(y) -> exp(-|x-y|^2/2) with h(x) = exp(-|x|^2/2); sigma as above with G = 1."""
    d, pairs = _mc_pairs()
    m = 120000
    w = inputs.performer_omega(m, d, 22, orthogonal, torch.float64).numpy()
    for x, y in pairs:
        est = float(feat(x, w, "gaussian") @ feat(y, w, "gaussian"))
        s2 = float(np.sum((x - y) ** 2))
        sigma = (1 - math.exp(-s2)) / math.sqrt(2 * m)
        if not abs(est - math.exp(-s2 / 2)) < 8 * sigma:
            return False
    return True


def test_feature_layout_exact():
    assert pin_layout(P.features)


@pytest.mark.parametrize("orthogonal", [False, True])
def test_feature_softmax_kernel_limit(orthogonal):
    assert pin_softmax_limit(P.features, orthogonal)


@pytest.mark.parametrize("orthogonal", [False, True])
def test_feature_gaussian_kernel_limit(orthogonal):
    assert pin_gaussian_limit(P.features, orthogonal)


def test_feature_shapes_and_batching():
    r = _rng(3)
    x = r.standard_normal((2, 3, 7, 8)) * 0.3
    w = r.standard_normal((5, 8))
    f = P.features(x, w, "softmax")
    assert f.shape == (2, 3, 7, 10)
    # row-wise map: batching changes nothing
    np.testing.assert_allclose(f[1, 2, 4], P.features(x[1, 2, 4], w, "softmax"), rtol=1e-13)


def test_orthogonal_draw_blocks():
    """Rows inside each block of d are orthogonal; every row is marginally
    N(0, I_d): the mean squared norm over many rows is close to d."""
    d, m = 16, 16 * 400
    w = inputs.performer_omega(m, d, 5, True, torch.float64).numpy()
    for b in range(0, m, d):
        G = w[b:b + d] @ w[b:b + d].T
        off = G - np.diag(np.diag(G))
        assert np.max(np.abs(off)) < 1e-9 * np.max(np.diag(G))
    # chi^2_d rows: mean d, sd sqrt(2d/m') over m' rows
    assert abs(np.mean(np.sum(w * w, 1)) - d) < 6 * math.sqrt(2 * d / m)
    # partial last block
    assert inputs.performer_omega(20, 16, 5, True, torch.float64).shape == (20, 16)


# ------------------------------------------------------- attention on features
def _case(seed, B, H, N, dk, dv):
    q, k, v = inputs.random_case(seed, B, H, N, dk, dv, torch.float32)
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


@pytest.mark.parametrize("with_lam,with_init", [(False, False), (True, False), (True, True)])
def test_causal_feat_matches_c_oracle_on_elu_features(with_lam, with_init):
    q, k, v = _case(31, 2, 3, 37, 8, 5)
    lam = np.array([0.9, 0.5, 0.0]) if with_lam else None
    S0 = z0 = None
    if with_init:
        r = _rng(4)
        S0 = np.abs(r.standard_normal((2, 3, 8, 5)))
        z0 = np.abs(r.standard_normal((2, 3, 8))) + 0.5
    y, S, z = P.causal_feat(elu1(q), elu1(k), v, lam, 1e-3, S0, z0)
    yo, So, zo = oracle.causal(q, k, v, lam, 1e-3, S0, z0)
    np.testing.assert_allclose(y, yo, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(S, So, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(z, zo, rtol=1e-11, atol=1e-13)


def test_global_and_decode_feat_match_c_oracle_on_elu_features():
    q, k, v = _case(32, 2, 2, 19, 8, 4)
    qc = q[:, :, :7]
    y, KV, ks = P.global_feat(elu1(qc), elu1(k), v, 1e-4)
    yo, KVo, kso = oracle.global_cross(qc, k, v, 1e-4)
    np.testing.assert_allclose(y, yo, rtol=1e-12)
    np.testing.assert_allclose(KV, KVo, rtol=1e-12)
    np.testing.assert_allclose(ks, kso, rtol=1e-12)
    r = _rng(5)
    S = np.abs(r.standard_normal((2, 2, 8, 4)))
    z = np.abs(r.standard_normal((2, 2, 8))) + 0.1
    lam = np.array([0.7, 1.0])
    y1, S1, z1 = P.decode_feat(elu1(q[:, :, 0]), elu1(k[:, :, 0]), v[:, :, 0], S, z, lam, 1e-4)
    yo, So, zo = oracle.decode_step(q[:, :, 0], k[:, :, 0], v[:, :, 0], S, z, lam, 1e-4)
    np.testing.assert_allclose(y1, yo, rtol=1e-12)
    np.testing.assert_allclose(S1, So, rtol=1e-12)
    np.testing.assert_allclose(z1, zo, rtol=1e-12)


def test_rows_form_matches_recurrence_with_signed_features():
    r = _rng(6)
    B, H, N, f, dv = 2, 2, 40, 6, 3
    fq = r.standard_normal((B, H, N, f))
    fk = r.standard_normal((B, H, N, f))
    v = r.standard_normal((B, H, N, dv))
    lam = np.array([0.95, 0.6])
    y, _, _ = P.causal_feat(fq, fk, v, lam, 0.5)
    rows = [(0, 0, 0), (1, 1, 39), (0, 1, 17), (1, 0, 5)]
    np.testing.assert_allclose(P.causal_feat_rows(fq, fk, v, lam, 0.5, rows),
                               np.stack([y[b, h, i] for b, h, i in rows]), rtol=1e-10)


def test_performer_attention_converges_to_softmax_kernel_attention():
    """With 200000 features, the Performer recurrence approaches decayed
    softmax-kernel attention y_i = sum_j lam^(i-j) e^(q_i.k_j) v_j /
    sum_j lam^(i-j) e^(q_i.k_j), written as a plain double loop."""
    r = _rng(7)
    N, d, dv, lam = 6, 4, 3, 0.9
    q = 0.3 * r.standard_normal((1, 1, N, d))
    k = 0.3 * r.standard_normal((1, 1, N, d))
    v = r.standard_normal((1, 1, N, dv))
    w = inputs.performer_omega(200000, d, 8, True, torch.float64).numpy()
    y, _, _ = P.causal_feat(P.features(q, w), P.features(k, w), v, np.array([lam]), 0.0)
    for i in range(N):
        num = np.zeros(dv)
        den = 0.0
        for j in range(i + 1):
            a = lam ** (i - j) * math.exp(float(q[0, 0, i] @ k[0, 0, j]))
            num += a * v[0, 0, j]
            den += a
        np.testing.assert_allclose(y[0, 0, i], num / den, atol=5e-3)


# ------------------------------------------------------------ planted mistakes
def _mutant(kind):
    def feat(x, w, kernel="softmax"):
        x, w = np.asarray(x, float), np.asarray(w, float)
        m = w.shape[0]
        u = x @ w if kind == "transposed" else x @ w.T
        n2 = np.sum(x * x, axis=-1, keepdims=True)
        if kernel == "softmax":
            g = np.exp((-0.5 if kind == "exp_sign" else 0.5) * n2)
        else:
            g = np.ones_like(n2)
        sc = 1.0 / m if kind == "scale" else 1.0 / np.sqrt(m)
        c, s = np.cos(u), np.sin(u)
        if kind == "swap_halves":
            c, s = s, c
        if kind == "cos_twice":
            s = c
        return g * sc * np.concatenate([c, s], axis=-1)
    return feat


@pytest.mark.parametrize("kind", ["exp_sign", "scale", "swap_halves", "cos_twice", "transposed"])
def test_pins_catch_planted_mistakes(kind):
    feat = _mutant(kind)
    if kind == "transposed":
        # only defined where omega is square; the layout pin uses m = d
        caught = not pin_layout(feat)
    else:
        caught = (not pin_layout(feat) or not pin_softmax_limit(feat, False)
                  or not pin_gaussian_limit(feat, False))
    assert caught
