"""Gradient oracle (fp64, CPU) of the causal forward.

TEST INFRASTRUCTURE ONLY, under the same rule as the rest of ``oracle/``:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s baseline legs
may use it; the product never imports it.

The forward is written in its masked O(N^2) form: the recurrence
S_i = lambda S_{i-1} + phi(k_i) v_i^T, z_i = lambda z_{i-1} + phi(k_i),
y_i = phi(q_i)^T S_i / (phi(q_i)^T z_i + eps) of the fast-weight article
(§2.1, §3.2, §4.2), unrolled into the triangular-mask form of its §3.1:

    y_i = sum_{j<=i} lambda^(i-j) (phi(q_i).phi(k_j)) v_j
          / (sum_{j<=i} lambda^(i-j) phi(q_i).phi(k_j) + eps),

with phi(x) = x + 1 for x > 0 and e^x otherwise (elu + 1).  torch autograd on
that expression gives the gradients of L = sum(dy * y) with respect to q, k,
v and the per-head lambda (summed over the batch).  The tests pin it with
central differences of the C oracle's forward, which shares no code with it.
With ``identity`` q and k are feature vectors already (phi is the identity,
as for random features); that mode is pinned by central differences of the
numpy recurrence on features in ``oracle/performer.py``.
"""
from __future__ import annotations

import numpy as np
import torch


def _phi(x: torch.Tensor) -> torch.Tensor:
    # exp only of min(x, 0): the branch torch.where does not select must stay
    # finite, or its zero gradient times inf would give NaN
    return torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))


def _decay_mask(lam: torch.Tensor, N: int) -> torch.Tensor:
    """[H, N, N] with lambda_h^(i-j) for j <= i and 0 above the diagonal.
    Powers are running products, so lambda = 0 gives 0^0 = 1 on the diagonal."""
    H = lam.shape[0]
    ones = torch.ones(H, 1, dtype=lam.dtype)
    pw = torch.cat([ones, torch.cumprod(lam[:, None].expand(H, max(N - 1, 0)), dim=1)], dim=1)
    i = torch.arange(N)
    diff = (i[:, None] - i[None, :]).clamp(min=0)
    W = pw[:, diff]                                   # [H, N, N]
    return torch.where((i[:, None] >= i[None, :])[None], W, torch.zeros((), dtype=lam.dtype))


def causal_forward(q, k, v, lam, eps, identity=False):
    """y [B, H, N, dv] of the masked form (torch float64, differentiable)."""
    N = q.shape[-2]
    W = _decay_mask(lam, N)[None]                     # [1, H, N, N]
    f = (lambda x: x) if identity else _phi
    A = (f(q) @ f(k).transpose(-1, -2)) * W
    return (A @ v) / (A.sum(-1, keepdim=True) + eps)


def causal_grad(q, k, v, lam, eps, dy, identity=False):
    """Returns numpy float64 (y, dq, dk, dv, dlam) for L = sum(dy * y).
    ``lam`` [H] or None (no decay: dlam is then None); ``identity``: q and k
    are feature vectors (no elu + 1)."""
    t = lambda a: torch.as_tensor(np.asarray(a, dtype=np.float64) if not torch.is_tensor(a)
                                  else a.detach().to(torch.float64).cpu().numpy())
    qd, kd, vd, dyd = (t(a).clone().requires_grad_(True) for a in (q, k, v, dy))
    H = qd.shape[1]
    want_lam = lam is not None
    lamd = t(lam).clone().requires_grad_(True) if want_lam else torch.ones(H, dtype=torch.float64)
    y = causal_forward(qd, kd, vd, lamd, float(eps), identity)
    (y * dyd.detach()).sum().backward()
    dlam = lamd.grad.numpy() if want_lam else None
    return (y.detach().numpy(), qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy(), dlam)
