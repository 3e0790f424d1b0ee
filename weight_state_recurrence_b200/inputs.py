"""Seeded synthetic workloads.

This module only draws random numbers and shapes tensors; it holds none of
the method's arithmetic.  Both the CUDA path (tests, bench) and the oracle
(tests, CPU baseline) take their inputs from here, so both sides see the
same bit patterns.

Recipe (shared by every workload): a ``torch.Generator`` seeded with the
workload's seed draws q, then k, then v with ``torch.randn(shape,
dtype=float32)``; each is multiplied by the workload's scale (1/sqrt(d) for
the bf16 workloads, 1 for the fp32 one) and rounded once to the workload's
dtype (round-to-nearest-even).  Per-head decay values are produced in fp32.

The five workloads mirror the pages' statement of the problem: the elu+1
feature map, an optional per-head decay and the normaliser, in the causal,
global and decode forms.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    op: str                 # "causal" | "global" | "decode"
    B: int
    H: int
    N: int                  # sequence length (decode: prefix length)
    d: int                  # d_k = d_v
    dtype: torch.dtype
    scale: float
    seed: int
    eps: float = 1e-6
    lam: str = "none"       # "none" | "linspace" | "const"
    lam_lo: float = 1.0
    lam_hi: float = 1.0
    steps: int = 0          # decode steps
    tol: float = 2e-2       # max relative error gate against the oracle
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return self.B * self.N


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", "causal", 1, 1, 256, 32, torch.float32, 1.0, 1,
                         tol=1e-4),
    "causal_d64": Workload("causal_d64", "causal", 2, 8, 4096, 64, torch.bfloat16,
                           1 / math.sqrt(64), 2),
    "causal_decay_d128": Workload("causal_decay_d128", "causal", 4, 16, 16384, 128,
                                  torch.bfloat16, 1 / math.sqrt(128), 3, lam="linspace",
                                  lam_lo=0.9, lam_hi=0.999),
    "global_d64": Workload("global_d64", "global", 8, 12, 8192, 64, torch.bfloat16,
                           1 / math.sqrt(64), 4),
    "decode_d128": Workload("decode_d128", "decode", 256, 32, 512, 128, torch.bfloat16,
                            1 / math.sqrt(128), 5, lam="const", lam_lo=0.999,
                            lam_hi=0.999, steps=1024),
}

# Per-step seeds of the decode workload: step s draws from seed STEP_SEED0 + s.
STEP_SEED0 = 1000


def _draw(gen, shape, scale, dtype, device):
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    if scale != 1.0:
        x = x * scale
    return x.to(dtype).contiguous()


def qkv(shape_q, shape_v, seed, scale, dtype, device="cpu"):
    """q, k with shape ``shape_q`` and v with ``shape_v``, drawn in that
    order from one generator seeded with ``seed``."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    q = _draw(gen, shape_q, scale, dtype, device)
    k = _draw(gen, shape_q, scale, dtype, device)
    v = _draw(gen, shape_v, scale, dtype, device)
    return q, k, v


def decay(w: Workload, H: int | None = None):
    """Per-head decay as an fp32 tensor ``[H]``, or None for no decay.
    "linspace": H values evenly spaced over [lam_lo, lam_hi], endpoints
    included; "const": every head lam_lo."""
    H = w.H if H is None else H
    if w.lam == "none":
        return None
    if w.lam == "linspace":
        return torch.linspace(w.lam_lo, w.lam_hi, H, dtype=torch.float32)
    if w.lam == "const":
        return torch.full((H,), w.lam_lo, dtype=torch.float32)
    raise ValueError(w.lam)


def causal_inputs(w: Workload, B=None, H=None, N=None, device="cpu"):
    """q, k, v ``[B, H, N, d]`` for a causal or global workload (the sizes
    may be overridden for reduced-size parity cases)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    shape = (B, H, N, w.d)
    return qkv(shape, shape, w.seed, w.scale, w.dtype, device)


def decode_step_inputs(w: Workload, step: int, B=None, H=None, device="cpu"):
    """q, k, v ``[B, H, d]`` for decode step ``step`` (seed STEP_SEED0+step)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    shape = (B, H, w.d)
    return qkv(shape, shape, STEP_SEED0 + step, w.scale, w.dtype, device)


def random_case(seed, B, H, N, dk, dv, dtype=torch.float32, scale=1.0, device="cpu"):
    """Generic seeded case for edge-shape tests (d_k may differ from d_v)."""
    return qkv((B, H, N, dk), (B, H, N, dv), seed, scale, dtype, device)


# Performer workload: the fast-weight recurrence on random trig features
# (linear-attention note §4.2) of q and k.  Raw q, k are N(0, 1/(4d)) (scale
# 1/(2 sqrt d)), so |omega.(q-k)| stays near 0.7 rad and the m = 64 estimate of
# the kernel is well conditioned; v is N(0, 1/d) like the other bf16 workloads.
PERFORMER = {
    "performer_d128": dict(B=4, H=16, N=16384, d=128, m=64, seed=6, lam_lo=0.9,
                           lam_hi=0.999, dtype=torch.bfloat16),
}


def performer_omega(m, d, seed, orthogonal=True, dtype=torch.float32, device="cpu"):
    """Projection ``[m, d]`` for the Performer feature map: every row is
    marginally N(0, I_d) (linear-attention note §4.2: omega drawn from the
    standard normal, with a fixed seed shared by all processes).

    ``orthogonal`` draws the rows in blocks of d that are mutually orthogonal
    (the note's orthogonalised omega): each block is Q^T of the QR factors of a
    d x d Gaussian matrix, with Q's columns sign-fixed by diag(R) so the block
    is Haar-distributed, and each row rescaled by the norm of an independent
    N(0, I_d) vector.  The last block keeps its first m mod d rows.  The
    result is rounded once to ``dtype``."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    if not orthogonal:
        w = torch.randn((m, d), generator=gen, dtype=torch.float64)
    else:
        blocks = []
        for _ in range((m + d - 1) // d):
            G = torch.randn((d, d), generator=gen, dtype=torch.float64)
            Q, R = torch.linalg.qr(G)
            Q = Q * torch.sign(torch.diagonal(R))[None, :]
            norms = torch.randn((d, d), generator=gen, dtype=torch.float64).norm(dim=1)
            blocks.append(Q.T * norms[:, None])
        w = torch.cat(blocks, 0)[:m]
    return w.to(dtype).contiguous().to(device)


def performer_inputs(name, B=None, H=None, N=None, device="cpu"):
    """q, k ``[B, H, N, d]``, v ``[B, H, N, d]``, lambda ``[H]`` and omega
    ``[m, d]`` (same dtype as q) of a Performer workload."""
    p = PERFORMER[name]
    B = p["B"] if B is None else B
    H = p["H"] if H is None else H
    N = p["N"] if N is None else N
    d = p["d"]
    gen = torch.Generator(device=device)
    gen.manual_seed(int(p["seed"]))
    shape = (B, H, N, d)
    q = _draw(gen, shape, 0.5 / math.sqrt(d), p["dtype"], device)
    k = _draw(gen, shape, 0.5 / math.sqrt(d), p["dtype"], device)
    v = _draw(gen, shape, 1.0 / math.sqrt(d), p["dtype"], device)
    lam = torch.linspace(p["lam_lo"], p["lam_hi"], H, dtype=torch.float32)
    omega = performer_omega(p["m"], d, p["seed"] + 1, True, p["dtype"], device)
    return q, k, v, lam, omega
