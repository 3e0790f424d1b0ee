"""Performer random-feature oracle (fp64, CPU).

TEST INFRASTRUCTURE ONLY, under the same rule as the rest of ``oracle/``:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s baseline legs
may use it; the product never imports it, and this module imports nothing
from the product.

Feature map (linear-attention note §4.2).  For a projection Omega [m, d]
whose rows omega_l are N(0, I_d) draws (passed in, never drawn here):

    phi(x) = g(x) / sqrt(m) * [cos(omega_1.x) .. cos(omega_m.x),
                               sin(omega_1.x) .. sin(omega_m.x)]      (2m values)

with g(x) = exp(|x|^2 / 2) h(x).  The note's h is optional:
  * kernel "softmax":  h = 1, so phi(x).phi(y) estimates exp(x.y);
  * kernel "gaussian": h(x) = exp(-|x|^2/2), the note's example, so
    phi(x).phi(y) estimates the Gaussian kernel exp(-|x-y|^2/2).
The tests pin both limits by Monte Carlo.

Attention on features.  The fast-weight recurrence (fast-weight article
§2.1, §3.2, §4.2) with q and k replaced by given feature vectors fq, fk:

    S_i = lambda S_{i-1} + fk_i v_i^T,   z_i = lambda z_{i-1} + fk_i,
    y_i = fq_i^T S_i / (fq_i^T z_i + eps).

It is written here with numpy, independently of the C oracle; the tests pin
it against the C oracle by feeding it elu + 1 features.  Trig features can be
negative, so nothing here assumes a positive denominator.
"""
from __future__ import annotations

import numpy as np

KERNELS = ("softmax", "gaussian")


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu").to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def features(x, omega, kernel="softmax"):
    """phi(x) for x ``[..., d]`` and omega ``[m, d]``: ``[..., 2m]``, the m
    cosines first, then the m sines (linear-attention note §4.2)."""
    if kernel not in KERNELS:
        raise ValueError(kernel)
    x, w = _f64(x), _f64(omega)
    m = w.shape[0]
    u = x @ w.T                                            # omega_l . x
    if kernel == "softmax":
        g = np.exp(0.5 * np.sum(x * x, axis=-1, keepdims=True))
    else:
        g = np.ones(x.shape[:-1] + (1,))
    return (g / np.sqrt(m)) * np.concatenate([np.cos(u), np.sin(u)], axis=-1)


def causal_feat(fq, fk, v, lam=None, eps=1e-6, S0=None, z0=None):
    """The causal recurrence on features, token by token, every (b, h) at once.
    fq, fk ``[B, H, N, f]``, v ``[B, H, N, dv]``, lam ``[H]`` or None.
    Returns ``(y [B,H,N,dv], S_N [B,H,f,dv], z_N [B,H,f])``."""
    fq, fk, v = _f64(fq), _f64(fk), _f64(v)
    B, H, N, f = fq.shape
    dv = v.shape[-1]
    L = np.ones(H) if lam is None else _f64(lam)
    S = np.zeros((B, H, f, dv)) if S0 is None else _f64(S0).copy()
    z = np.zeros((B, H, f)) if z0 is None else _f64(z0).copy()
    y = np.empty((B, H, N, dv))
    for i in range(N):
        S = L[None, :, None, None] * S + fk[:, :, i, :, None] * v[:, :, i, None, :]
        z = L[None, :, None] * z + fk[:, :, i]
        num = np.einsum("bhf,bhfv->bhv", fq[:, :, i], S)
        den = np.einsum("bhf,bhf->bh", fq[:, :, i], z) + eps
        y[:, :, i] = num / den[..., None]
    return y, S, z


def causal_feat_rows(fq, fk, v, lam, eps, rows):
    """y_i for sampled (b, h, i) triples only, from the unrolled sum
    y_i = sum_{j<=i} lam^(i-j) (fq_i.fk_j) v_j / (sum_{j<=i} lam^(i-j) fq_i.fk_j + eps)
    (fast-weight article §3.1 triangular-mask form).  Returns ``[len(rows), dv]``."""
    fq, fk, v = _f64(fq), _f64(fk), _f64(v)
    out = []
    for b, h, i in rows:
        L = 1.0 if lam is None else float(_f64(lam)[h])
        w = fk[b, h, : i + 1] @ fq[b, h, i]                   # fq_i . fk_j, j <= i
        w = w * np.power(L, np.arange(i, -1, -1, dtype=np.float64))
        out.append((w @ v[b, h, : i + 1]) / (w.sum() + eps))
    return np.stack(out) if out else np.zeros((0, v.shape[-1]))


def global_feat(fq, fk, v, eps=1e-6):
    """Non-causal form on features: y = fq (fk^T V) / (fq (fk^T 1) + eps), with
    separate query and key lengths allowed.  Returns ``(y, KV, ksum)``."""
    fq, fk, v = _f64(fq), _f64(fk), _f64(v)
    KV = np.einsum("bhnf,bhnv->bhfv", fk, v)
    ks = fk.sum(axis=2)
    num = np.einsum("bhnf,bhfv->bhnv", fq, KV)
    den = np.einsum("bhnf,bhf->bhn", fq, ks) + eps
    return num / den[..., None], KV, ks


def decode_feat(fq, fk, v, S, z, lam=None, eps=1e-6):
    """One recurrent step on features ``[B, H, f]`` from state (S, z); the
    inputs are not modified.  Returns ``(y [B,H,dv], S_new, z_new)``."""
    fq, fk, v = _f64(fq), _f64(fk), _f64(v)
    H = fq.shape[1]
    L = np.ones(H) if lam is None else _f64(lam)
    S = L[None, :, None, None] * _f64(S) + fk[..., :, None] * v[..., None, :]
    z = L[None, :, None] * _f64(z) + fk
    y = np.einsum("bhf,bhfv->bhv", fq, S) / (np.einsum("bhf,bhf->bh", fq, z) + eps)[..., None]
    return y, S, z
