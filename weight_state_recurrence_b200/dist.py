"""Process-per-GPU plumbing: the batch-sharded path and the sequence-parallel
causal forward.

Every (batch, head) pair is independent in all three forms of the method (the
state of one head never reads another head's tokens), so several GPUs split
the batch: rank r owns sequences [start, stop) of the global batch and never
exchanges data with the other ranks.  The only collectives are for timing:
a barrier around the timed region and the maximum of the per-rank times.

Long sequences can instead be split by token position (``seq_parallel_causal``):
rank r holds one segment of every sequence.  This is the segment scan of the
fast-weight article (§4.1 note, §5.2: blocks computed in parallel, the state
carried across them) one level above the chunks, and it has one real exchange:
each rank's own segment state (d_k*d_v + d_k fp32 per head) is all-gathered,
every rank scans the gathered states into its starting state, and then runs
its segment's forward from that state.

Ranks are launched one per GPU (torchrun); NCCL is used on GPUs and gloo on
CPU (tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def shard(total: int, world: int, rank: int) -> tuple[int, int]:
    """Balanced contiguous range [start, stop) of `total` items for `rank`."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def env_world() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0, device=None) -> None:
    """Join the process group named by the environment (no-op for one rank)."""
    world, rank, _ = env_world()
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if device is not None else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def barrier() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device="cpu") -> float:
    """Largest value of `x` over all ranks (x itself for one rank)."""
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class LibraryOps:
    """The three steps of the sequence-parallel forward on this rank's GPU,
    each one call of the C library (``weight_state_recurrence_b200.linattn``)."""

    def __init__(self, lib, stream=None):
        self.lib = lib
        self.stream = stream

    def state(self, k, v, lam):
        B, H, _, dk = k.shape
        dv = v.shape[-1]
        S = torch.empty(B, H, dk, dv, dtype=torch.float32, device=k.device)
        z = torch.empty(B, H, dk, dtype=torch.float32, device=k.device)
        self.lib.linattn_causal_state(k, v, lam, S, z, self.stream)
        return S, z

    def combine(self, seg_len, lam, S_init, z_init, dS, dz):
        self.lib.linattn_combine_states(seg_len, lam, S_init, z_init, dS, dz, self.stream)

    def forward_from(self, q, k, v, lam, eps, S0, z0):
        B, H, _, dk = q.shape
        dv = v.shape[-1]
        out = torch.empty_like(v)
        S = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
        z = torch.empty(B, H, dk, dtype=torch.float32, device=q.device)
        self.lib.linattn_fwd_causal_from(q, k, v, lam, eps, S0, z0, out, S, z, self.stream)
        return out, S, z


def gather_stack(x: torch.Tensor, world: int) -> torch.Tensor:
    """[world, *x.shape]: x from every rank, in rank order (one all-gather)."""
    if world == 1:
        return x[None].clone()
    outt = torch.empty((world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
    if x.is_cuda:
        dist.all_gather_into_tensor(outt, x.contiguous())
    else:
        dist.all_gather(list(outt.unbind(0)), x.contiguous())
    return outt


def seq_parallel_causal(q, k, v, lam, eps, *, world: int, rank: int, seg_len: int, ops,
                        S_init=None, z_init=None, gather=gather_stack):
    """Causal forward of sequences cut by token position across `world`
    ranks: this rank holds tokens [rank*seg_len, rank*seg_len + n) of every
    sequence (q, k [B, H, n, dk], v [B, H, n, dv]; n = seg_len except
    possibly on the last rank).  Steps:

    1. own state: (dS, dz) of this rank's tokens from a zero start;
    2. exchange: one all-gather of (dS, dz) into slots [world, B, H, ...];
    3. combine: slot g becomes the state at the start of segment g,
       carry_{g+1} = lambda^seg_len carry_g + dS_g, carry_0 = (S_init, z_init);
    4. output: this rank's tokens from slot `rank`.

    Returns (y, S_end, z_end): y of this rank's tokens and the state after its
    last token (on the last rank, the state after the whole sequence)."""
    if q.shape[2] != seg_len and rank != world - 1:
        raise ValueError("only the last rank may hold fewer than seg_len tokens")
    dS, dz = ops.state(k, v, lam)
    dS_all = gather(dS, world)
    dz_all = gather(dz, world)
    ops.combine(seg_len, lam, S_init, z_init, dS_all, dz_all)
    return ops.forward_from(q, k, v, lam, eps, dS_all[rank].contiguous(),
                            dz_all[rank].contiguous())


def finalize() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
