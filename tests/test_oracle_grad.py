"""Pins of the gradient oracle (CPU): its forward equals the C oracle's, and
every gradient equals central differences of the C oracle's forward (an
independent code path), on tiny inputs, with and without decay."""
import numpy as np
import pytest

import oracle
from oracle import grad as og


def rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape) * 0.7


def loss(q, k, v, lam, eps, dy):
    y, _, _ = oracle.causal(q, k, v, lam, eps)
    return float((y * dy).sum())


@pytest.mark.parametrize("lamv", [None, (0.9, 0.6)])
def test_forward_matches_c_oracle(lamv):
    q, k, v = rand(1, 2, 2, 9, 4), rand(2, 2, 2, 9, 4), rand(3, 2, 2, 9, 3)
    lam = None if lamv is None else np.array(lamv)
    y_c, _, _ = oracle.causal(q, k, v, lam, 1e-3)
    y_g, *_ = og.causal_grad(q, k, v, lam, 1e-3, np.zeros_like(y_c))
    assert np.abs(y_g - y_c).max() <= 1e-13 * np.abs(y_c).max()


@pytest.mark.parametrize("lamv", [None, (0.85, 1.0)])
def test_gradients_match_central_differences(lamv):
    q, k, v = rand(4, 1, 2, 6, 3), rand(5, 1, 2, 6, 3), rand(6, 1, 2, 6, 2)
    dy = rand(7, 1, 2, 6, 2)
    lam = None if lamv is None else np.array(lamv)
    eps = 1e-2
    _, dq, dk, dv, dlam = og.causal_grad(q, k, v, lam, eps, dy)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            fd[idx] = (loss(**{**args, name: xp}, lam=lam, eps=eps, dy=dy) -
                       loss(**{**args, name: xm}, lam=lam, eps=eps, dy=dy)) / (2 * h)
        assert np.abs(fd - g).max() <= 1e-6 * max(1.0, np.abs(g).max()), name
    if lam is not None:
        for hh in range(2):
            lp, lm = lam.copy(), lam.copy()
            lp[hh] += h
            lm[hh] -= h
            fd = (loss(q, k, v, lp, eps, dy) - loss(q, k, v, lm, eps, dy)) / (2 * h)
            assert abs(fd - dlam[hh]) <= 1e-6 * max(1.0, abs(dlam[hh]))


def test_zero_decay_has_finite_gradients():
    q, k, v = rand(8, 1, 1, 5, 3), rand(9, 1, 1, 5, 3), rand(10, 1, 1, 5, 3)
    dy = rand(11, 1, 1, 5, 3)
    y, dq, dk, dv, dlam = og.causal_grad(q, k, v, np.array([0.0]), 1e-3, dy)
    for a in (y, dq, dk, dv, dlam):
        assert np.isfinite(a).all()
    # with lambda = 0 every token attends only to itself: y_i = v_i w/(w + eps)
    w = (og._phi(__import__("torch").tensor(q)) * og._phi(__import__("torch").tensor(k))).sum(-1)
    w = w.numpy()[..., None]
    assert np.abs(y - v * w / (w + 1e-3)).max() < 1e-13


def test_identity_mode_gradients_match_central_differences_of_feature_recurrence():
    """q and k as signed feature vectors: gradients of the masked form with phi =
    identity equal central differences of oracle/performer.py's token-by-token
    recurrence (numpy, no autograd)."""
    from oracle import performer as P
    q, k, v = rand(12, 1, 2, 6, 3), rand(13, 1, 2, 6, 3), rand(14, 1, 2, 6, 2)
    q, k = q + 1.5, k + 1.5            # mostly positive scores, some signed features
    dy = rand(15, 1, 2, 6, 2)
    lam = np.array([0.8, 1.0])
    eps = 0.5

    def L(qq, kk, vv, ll):
        return float((P.causal_feat(qq, kk, vv, ll, eps)[0] * dy).sum())

    y, dq, dk, dv, dlam = og.causal_grad(q, k, v, lam, eps, dy, identity=True)
    np.testing.assert_allclose(y, P.causal_feat(q, k, v, lam, eps)[0], rtol=1e-12)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("lam", lam, dlam)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            a = {"qq": q, "kk": k, "vv": v, "ll": lam}
            key = {"q": "qq", "k": "kk", "v": "vv", "lam": "ll"}[name]
            fd[idx] = (L(**{**a, key: xp}) - L(**{**a, key: xm})) / (2 * h)
        assert np.abs(fd - g).max() <= 1e-6 * max(1.0, np.abs(g).max()), name
