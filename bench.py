"""Benchmark: causal linear-attention forward tokens/s at N=16K, d=128 (plus
decode and global legs), as a fraction of the B200 roofline.

One step = one causal forward (linattn_fwd_causal) over the
causal_decay_d128 workload: B=4 sequences x H=16 heads x N=16384 tokens,
d_k = d_v = 128, bf16 q/k/v ~ N(0,1)/sqrt(128), per-head decay
lambda_h = linspace(0.9, 0.999, 16), fp32 state, outputs y, S_final, z_final.
Under torchrun every rank runs its own batch of that size (the batch axis is
sharded: heads and sequences are independent, so there is no data-path
collective; weak scaling).  Timing: W untimed steps, then K steps between a
barrier + synchronize on both sides, CUDA events on the launch stream, max
over ranks.  Inputs (805 MB per step) are larger than the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--no-e2e] [--no-legs] [--no-cpu-baseline]
                  [--only causal|decode|global|backward|segmented|performer]
                  [--batch B] [--dec-batch B]
                  [--dec-steps T]
The last four options shrink or isolate a leg for profiler captures; the
reported benchmark always uses the full workloads (their defaults).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_state_recurrence_b200 import dist as wdist  # noqa: E402
from weight_state_recurrence_b200 import inputs  # noqa: E402

METRIC = "causal linear-attn fwd tokens/s (N=16K,d=128) + decode tok/s, % roofline"
WL = inputs.WORKLOADS["causal_decay_d128"]
WL_DEC = inputs.WORKLOADS["decode_d128"]
WL_GLB = inputs.WORKLOADS["global_d64"]


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def causal_bytes(B, H, N, dk, dv, es=2):
    """Algorithmic HBM bytes of one causal forward: q, k, v read once, y
    written once, S_final / z_final written once (fp32)."""
    return B * H * N * (2 * dk + 2 * dv) * es + B * H * (dk * dv + dk) * 4


def causal_mma_flops(B, H, N, dk, dv):
    """MMA flops the segmented tensor-core causal kernel executes per launch
    (C = 128 tokens per chunk, one CTA per head with the whole dv).  Per chunk
    and head: the score tile 128x128xdk, the carried term 128xdvxdk, the state
    update 128xdvx128 (its M is the 128 rows of d_k, zero-padded for
    dk = 64) and the intra term 128xdvx128."""
    C = 128
    chunks = -(-N // C)
    per = 2 * C * (C * dk + dv * dk + dv * 128 + dv * C)
    return B * H * chunks * per


def decode_bytes(B, H, dk, dv, es=2):
    """Per step: S read + written (fp32), z read + written, q/k/v read, y written."""
    return B * H * (2 * dk * dv * 4 + 2 * dk * 4 + (2 * dk + 2 * dv) * es)


def global_bytes(B, H, N, dk, dv, es=2):
    return B * H * N * (2 * dk + 2 * dv) * es + B * H * (dk * dv + dk) * 4


def traffic_record(kernel):
    """DRAM bytes per launch from the committed ncu summary, valid only while
    the kernel source is unchanged (sha256 of the sources it was taken on)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    h = hashlib.sha256()
    for rel in rec.get("sources", []):
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        except OSError:
            return None
    if h.hexdigest() != rec.get("sha256"):
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """SM clock and throttle-reason samples during the timed region, polled
    through NVML every ~1 ms (nvidia-smi at its 100 ms minimum as a fallback)."""

    def __init__(self, index):
        self.index = index
        self.samples = []          # (sm_mhz, reasons bitmask)
        self.max_mhz = None
        self.stop = threading.Event()
        self.nvml = None
        self.proc = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def poll():
                while not self.stop.is_set():
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                             get_reasons(h)))
                    except Exception:
                        pass
                    time.sleep(0.001)
            self.t = threading.Thread(target=poll, daemon=True)
            self.t.start()
        except Exception:
            self.nvml = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.index),
                     "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.t = threading.Thread(target=self._read_smi, daemon=True)
                self.t.start()
            except Exception:
                self.proc = None
        return self

    def _read_smi(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            try:
                self.max_mhz = float(f[1])
                self.samples.append((float(f[0]), int(f[2], 16)))
            except (ValueError, IndexError):
                continue

    def __exit__(self, *a):
        self.stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    # NVML clocks-event-reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mask = 0
        for _, r in self.samples:
            mask |= int(r)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for b, n in self.REASONS.items() if mask & b),
                "samples": len(self.samples)}


def dist_setup():
    world, rank, local = wdist.env_world()
    torch.cuda.set_device(local)
    wdist.init("nccl", timeout_s=120, device=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    wdist.barrier()


def max_over_ranks(x, world):
    return wdist.max_over_ranks(x, device="cuda")


def time_steps(fn, steps, warmup, world, stream):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1), world)


# ---------------------------------------------------------------- legs
def causal_leg(lib, args, world, rank, stream, hbm, tc_peak):
    B, H, N, d = args.batch or WL.B, WL.H, WL.N, WL.d
    dev = torch.device("cuda")
    q, k, v = inputs.qkv((B, H, N, d), (B, H, N, d), WL.seed * 1000 + rank, WL.scale,
                         WL.dtype, device=dev)
    lam = inputs.decay(WL).to(dev)
    out = torch.empty_like(v)
    S = torch.empty(B, H, d, d, device=dev)
    z = torch.empty(B, H, d, device=dev)

    # the product call: linattn_fwd_causal_ws with the workspace the library
    # asks for (the segment plan it picks, or --segments forced), i.e. the
    # state pass and the forward launched as its dependent
    with lib.kernel_choice(lib.LINATTN_OP_CAUSAL, lib.LINATTN_KERNEL_AUTO, args.segments):
        need = lib.linattn_fwd_causal_workspace(B, H, N, d, d, WL.dtype)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    seg_launches = 2 if need > 0 else 1

    ops = wdist.LibraryOps(lib, stream)

    def step():
        if args.seq_parallel:
            # this rank holds tokens [rank N, (rank + 1) N) of sequences of
            # world * N tokens: own segment state, one all-gather, the scan,
            # then the segment's forward from its starting state
            wdist.seq_parallel_causal(q, k, v, lam, WL.eps, world=world, rank=rank, seg_len=N,
                                      ops=ops)
        else:
            lib.linattn_fwd_causal_ws(q, k, v, lam, WL.eps, None, None, out, S, z, ws, stream)

    with torch.cuda.stream(stream):
        with ClockSampler(torch.cuda.current_device()) as clk:
            with lib.kernel_choice(lib.LINATTN_OP_CAUSAL, lib.LINATTN_KERNEL_AUTO, args.segments):
                ms = time_steps(step, args.steps, args.warmup, world, stream)
    assert lib.linattn_device_status(clear=True, stream=stream) == 0, "device error flag set"
    per_launch_s = ms / 1e3 / args.steps
    tokens = B * N * world * args.steps
    value = tokens / (ms / 1e3)
    alg = causal_bytes(B, H, N, d, d)
    flops = causal_mma_flops(B, H, N, d, d)
    # DRAM bytes of one step: the forward, plus the state pass when the step has one
    traffic = traffic_record("causal_seg_tc_kernel")
    if traffic is not None and seg_launches == 2:
        sp = traffic_record("causal_seg_state_tc_kernel")
        traffic = None if sp is None else traffic + sp
    roof = {"bound": "hbm", "achieved": alg / per_launch_s / 1e9, "peak": hbm, "unit": "GB/s",
            "frac": alg / per_launch_s / 1e9 / hbm, "traffic": traffic,
            "algorithmic_bytes_per_launch": alg,
            "kernel": ("causal_seg_state_tc_kernel + causal_seg_tc_kernel (overlapped; timed as one step)"
                       if seg_launches == 2 else "causal_seg_tc_kernel"),
            "tensor": {"mma_tflops": flops / per_launch_s / 1e12, "peak": tc_peak,
                       "frac": flops / per_launch_s / 1e12 / tc_peak,
                       "mma_flops_per_launch": flops}}
    launches = args.steps * (3 if args.seq_parallel else seg_launches)
    res = {"ms_per_step": ms / args.steps, "value": value, "roofline": roof,
           "clocks": clk.summary(), "gpu_launches": launches}

    if args.e2e and not args.seq_parallel:
        # through the public API with host buffers (fwd_causal_host): every
        # step copies q, k, v in from pinned host memory and y, S_final,
        # z_final back, four heads at a time on overlapping streams
        hq, hk, hv = (t.to("cpu").pin_memory() for t in (q, k, v))
        hy = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hS = torch.empty(S.shape, dtype=S.dtype, pin_memory=True)
        hz = torch.empty(z.shape, dtype=z.dtype, pin_memory=True)
        del q, k, v, out
        torch.cuda.empty_cache()

        def e2e_step():
            lib.fwd_causal_host(hq, hk, hv, lam, WL.eps, hy, hS, hz)

        ksteps = max(1, min(args.steps, 5))
        with torch.cuda.stream(stream):
            ms_e = time_steps(e2e_step, ksteps, 1, world, stream)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        d2h = sum(t.numel() * t.element_size() for t in (hy, hS, hz))
        res["e2e"] = {"value": B * N * world * ksteps / (ms_e / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "steps": ksteps, "ms_per_step": ms_e / ksteps,
                      "api": "fwd_causal_host (pieces of 4 heads)"}
    else:
        del q, k, v, out
    torch.cuda.empty_cache()
    return res


def decode_leg(lib, args, world, rank, stream, hbm):
    """256 sequences x 32 heads, d=128, state from a 512-token prefill, then
    1024 decode steps captured in one CUDA graph (inputs pre-staged)."""
    w = WL_DEC
    B, H, d, T = args.dec_batch or w.B, w.H, w.d, args.dec_steps or w.steps
    dev = torch.device("cuda")
    lam = inputs.decay(w).to(dev)
    qp, kp, vp = inputs.qkv((B, H, w.N, d), (B, H, w.N, d), w.seed * 1000 + rank, w.scale,
                            w.dtype, device=dev)
    S = torch.empty(B, H, d, d, device=dev)
    z = torch.empty(B, H, d, device=dev)
    yp = torch.empty_like(vp)
    lib.linattn_fwd_causal(qp, kp, vp, lam, w.eps, yp, S, z, stream)
    del qp, kp, vp, yp
    g = torch.Generator(device=dev)
    g.manual_seed(inputs.STEP_SEED0 + rank)
    qs = (torch.randn(T, B, H, d, generator=g, device=dev) * w.scale).to(w.dtype)
    ks = (torch.randn(T, B, H, d, generator=g, device=dev) * w.scale).to(w.dtype)
    vs = (torch.randn(T, B, H, d, generator=g, device=dev) * w.scale).to(w.dtype)
    ys = torch.empty_like(vs)
    torch.cuda.synchronize()

    def all_steps():
        for s in range(T):
            lib.linattn_decode_step(qs[s], ks[s], vs[s], lam, w.eps, S, z, ys[s], stream)

    with torch.cuda.stream(stream):
        all_steps()  # warm-up outside capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            all_steps()
        reps = 3
        ms = time_steps(graph.replay, reps, 1, world, stream)
    assert lib.linattn_device_status(clear=True, stream=stream) == 0
    del graph
    step_s = ms / 1e3 / (reps * T)
    alg = decode_bytes(B, H, d, d)
    state = B * H * (2 * d * d * 4 + 2 * d * 4)
    res = {"value": B * world / step_s, "unit": "tokens/s", "ms_per_step": step_s * 1e3,
           "steps_per_graph": T,
           "roofline": {"bound": "hbm", "achieved": alg / step_s / 1e9, "peak": hbm,
                        "unit": "GB/s", "frac": alg / step_s / 1e9 / hbm,
                        "state_frac": state / step_s / 1e9 / hbm,
                        "traffic": traffic_record("decode_step_kernel"),
                        "algorithmic_bytes_per_launch": alg, "kernel": "decode_step_kernel"},
           "gpu_launches": (reps + 1) * T}
    del qs, ks, vs, ys, S, z
    torch.cuda.empty_cache()
    return res


def global_leg(lib, args, world, rank, stream, hbm):
    w = WL_GLB
    B, H, N, d = w.B, w.H, w.N, w.d
    dev = torch.device("cuda")
    q, k, v = inputs.qkv((B, H, N, d), (B, H, N, d), w.seed * 1000 + rank, w.scale, w.dtype,
                         device=dev)
    out = torch.empty_like(v)
    KV = torch.empty(B, H, d, d, device=dev)
    ks = torch.empty(B, H, d, device=dev)

    def step():
        lib.linattn_fwd_global(q, k, v, w.eps, out, KV, ks, stream)

    with torch.cuda.stream(stream):
        ms = time_steps(step, args.steps, args.warmup, world, stream)
    per = ms / 1e3 / args.steps
    alg = global_bytes(B, H, N, d, d)
    res = {"value": B * N * world / per, "unit": "tokens/s", "ms_per_step": per * 1e3,
           "roofline": {"bound": "hbm", "achieved": alg / per / 1e9, "peak": hbm,
                        "unit": "GB/s", "frac": alg / per / 1e9 / hbm,
                        "algorithmic_bytes_per_launch": alg}}
    del q, k, v, out
    torch.cuda.empty_cache()
    return res


def tiny_leg(lib, args, world, rank, stream, hbm):
    """The tiny_f32 workload (B=1, H=1, N=256, d=32, fp32, no decay) on its
    kernel (the CUDA-core causal kernel: fp32 inputs).  A single head of 256
    tokens is latency-bound; the time is reported as the workload asks, with
    the HBM fraction for completeness."""
    w = inputs.WORKLOADS["tiny_f32"]
    B, H, N, d = w.B, w.H, w.N, w.d
    dev = torch.device("cuda")
    q, k, v = inputs.qkv((B, H, N, d), (B, H, N, d), w.seed * 1000 + rank, w.scale, w.dtype,
                         device=dev)
    out = torch.empty_like(v)
    S = torch.empty(B, H, d, d, device=dev)
    z = torch.empty(B, H, d, device=dev)

    def step():
        lib.linattn_fwd_causal(q, k, v, None, w.eps, out, S, z, stream)

    with torch.cuda.stream(stream):
        ms = time_steps(step, args.steps, args.warmup, world, stream)
    per = ms / 1e3 / args.steps
    alg = causal_bytes(B, H, N, d, d, es=4)
    return {"workload": "tiny_f32: B=1 x H=1 x N=256, d=32, fp32, no decay",
            "value": B * N * world / per, "unit": "tokens/s", "ms_per_step": per * 1e3,
            "kernel": "causal_simt_kernel (fp32)",
            "roofline": {"bound": "latency", "achieved": alg / per / 1e9, "peak": hbm,
                         "unit": "GB/s", "frac": alg / per / 1e9 / hbm,
                         "algorithmic_bytes_per_launch": alg}}


def seg_leg(lib, args, world, rank, stream, hbm):
    """The causal_d64 workload (B=2, H=8, N=4096, d=64, bf16, no decay): the
    product path (the tensor-core kernel cut into about one segment per SM,
    with its state pass, through linattn_fwd_causal_ws), the
    same kernel in one pass (16 CTAs), and for comparison the CUDA-core kernel
    in one pass and segmented."""
    w = inputs.WORKLOADS["causal_d64"]
    B, H, N, d = w.B, w.H, w.N, w.d
    dev = torch.device("cuda")
    q, k, v = inputs.qkv((B, H, N, d), (B, H, N, d), w.seed * 1000 + rank, w.scale, w.dtype,
                         device=dev)
    out = torch.empty_like(v)
    S = torch.empty(B, H, d, d, device=dev)
    z = torch.empty(B, H, d, device=dev)
    need_tc = lib.linattn_fwd_causal_workspace(B, H, N, d, d, w.dtype)
    with lib.kernel_choice(lib.LINATTN_OP_CAUSAL, lib.LINATTN_KERNEL_CUDA_CORES):
        need_cc = lib.linattn_fwd_causal_workspace(B, H, N, d, d, w.dtype)
    ws = torch.empty(max(need_tc, need_cc, 16), dtype=torch.uint8, device=dev)
    res = {"workload": "causal_d64: B=2 x H=8 x N=4096, d=64, bf16, no decay",
           "workspace_bytes": need_tc}
    alg = causal_bytes(B, H, N, d, d)
    auto, cc = lib.LINATTN_KERNEL_AUTO, lib.LINATTN_KERNEL_CUDA_CORES
    legs = (("tensor_core", auto,
             lambda: lib.linattn_fwd_causal_ws(q, k, v, None, w.eps, None, None, out, S, z, ws,
                                               stream)),
            ("tensor_core_single_pass", auto,
             lambda: lib.linattn_fwd_causal(q, k, v, None, w.eps, out, S, z, stream)),
            ("cuda_core_single_pass", cc,
             lambda: lib.linattn_fwd_causal(q, k, v, None, w.eps, out, S, z, stream)),
            ("cuda_core_segmented", cc,
             lambda: lib.linattn_fwd_causal_ws(q, k, v, None, w.eps, None, None, out, S, z, ws,
                                               stream)))
    for name, kernel, fn in legs:
        with lib.kernel_choice(lib.LINATTN_OP_CAUSAL, kernel):
            with torch.cuda.stream(stream):
                ms = time_steps(fn, args.steps, args.warmup, world, stream)
        per = ms / 1e3 / args.steps
        res[name] = {"value": B * N * world / per, "unit": "tokens/s", "ms_per_step": per * 1e3,
                     "roofline": {"bound": "hbm", "achieved": alg / per / 1e9, "peak": hbm,
                                  "unit": "GB/s", "frac": alg / per / 1e9 / hbm,
                                  "algorithmic_bytes_per_launch": alg}}
    assert lib.linattn_device_status(clear=True, stream=stream) == 0
    del q, k, v, out, ws
    torch.cuda.empty_cache()
    return res


def bwd_mma_flops(B, H, N, d, with_dlam=True):
    """MMA flops of the tensor-core backward (bf16, d_k = d_v = d = 128, chunks
    of C = 128 tokens), each group a 128 x 128 x 128 product (2 * 128^3):
    pass F per chunk P, At V, W, B Kt (and Q St, w St^T after the first
    chunk, the state update before the last); pass L (dlambda) Ms (and the
    two state updates before the last); pass R P^T, W^T, A^T w, B^T Q (and
    Lk K R, Lk V R^T after the last chunk, the R update before the first)."""
    C = 128
    n = -(-N // C)
    g = 2 * C * C * d
    f = 4 * n + 2 * (n - 1) + (n - 1)
    lpass = (n + 2 * (n - 1)) if with_dlam else 0
    r = 4 * n + 2 * (n - 1) + (n - 1)
    return B * H * g * (f + lpass + r)


def bwd_bytes(B, H, N, d, es=2):
    """Algorithmic HBM bytes of one backward: q, k, v, dy read once and dq,
    dk, dv written once (the per-token den, dden stash and dlambda aside)."""
    return 7 * B * H * N * d * es


def bwd_leg(lib, args, world, rank, stream, tensor_peak, hbm_peak):
    """Backward (dq, dk, dv, dlambda) of the causal forward on the
    causal_decay_d128 workload, a few steps: the tensor-core passes (bf16,
    d = 128)."""
    B, H, N, d = args.batch or WL.B, WL.H, WL.N, WL.d
    dev = torch.device("cuda")
    q, k, v = inputs.qkv((B, H, N, d), (B, H, N, d), WL.seed * 1000 + rank, WL.scale,
                         WL.dtype, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(WL.seed * 1000 + 500 + rank)
    dy = torch.randn(B, H, N, d, generator=g, device=dev).to(WL.dtype)
    lam = inputs.decay(WL).to(dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dl = torch.empty(H, device=dev)
    # the product call with its workspace (the split point's states and the
    # per-token stash), allocated once like the forward leg's
    need = lib.linattn_bwd_causal_workspace(B, H, N, d, d, WL.dtype)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

    def step():
        lib.linattn_bwd_causal(q, k, v, lam, WL.eps, dy, dq, dk, dv, dl, stream, workspace=ws)

    def step_no_dlam():
        lib.linattn_bwd_causal(q, k, v, lam, WL.eps, dy, dq, dk, dv, None, stream, workspace=ws)

    steps = max(1, min(args.steps, 10))
    with torch.cuda.stream(stream):
        ms = time_steps(step, steps, args.warmup, world, stream)
        ms_nd = time_steps(step_no_dlam, steps, args.warmup, world, stream)
    assert lib.linattn_device_status(clear=True, stream=stream) == 0
    per = ms / 1e3 / steps
    fl = bwd_mma_flops(B, H, N, d)
    by = bwd_bytes(B, H, N, d)
    res = {"value": B * N * world / per, "unit": "tokens/s", "ms_per_step": per * 1e3,
           "steps": steps, "ctas": B * H, "workspace_bytes": need,
           "without_dlambda": {"ms_per_step": ms_nd / steps,
                               "flops_per_launch": bwd_mma_flops(B, H, N, d, with_dlam=False)},
           "roofline": {"bound": "tensor", "achieved": fl / per / 1e12, "peak": tensor_peak,
                        "unit": "TFLOP/s", "frac": fl / per / 1e12 / tensor_peak,
                        "flops_per_launch": fl,
                        "kernel": "bwd_tc_s_kernel + bwd_tc_f_kernel + bwd_tc_l_kernel + "
                                  "bwd_tc_r_kernel",
                        "traffic": None},
           "hbm": {"algorithmic_bytes": by, "achieved": by / per / 1e9, "peak": hbm_peak,
                   "unit": "GB/s", "frac": by / per / 1e9 / hbm_peak}}
    del q, k, v, dy, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return res


def features_bytes(rows, d, m, es=2):
    """Algorithmic HBM bytes of one feature launch: x read, 2m features written,
    omega read once."""
    return rows * (d + 2 * m) * es + m * d * es


def performer_leg(lib, args, world, rank, stream, hbm):
    """Causal attention on Performer random features (performer_d128: B=4 x
    H=16 x N=16384, d=128, m=64 orthogonal features, bf16, decay): the
    feature kernel on q and on k, then the causal forward in identity mode on
    the 128 features.  The feature kernel is also timed alone."""
    p = inputs.PERFORMER["performer_d128"]
    B = args.batch or p["B"]
    H, N, d, m = p["H"], p["N"], p["d"], p["m"]
    dev = torch.device("cuda")
    q, k, v, lam, w = inputs.performer_inputs("performer_d128", B=B, device=dev)
    lam = lam.to(dev)
    fq = torch.empty(B, H, N, 2 * m, dtype=q.dtype, device=dev)
    fk = torch.empty_like(fq)
    out = torch.empty_like(v)
    S = torch.empty(B, H, 2 * m, d, device=dev)
    z = torch.empty(B, H, 2 * m, device=dev)
    K = lib.LINATTN_PERFORMER_SOFTMAX

    # the attention through the product call (workspace: the segment plan)
    need = lib.linattn_fwd_causal_workspace(B, H, N, 2 * m, d, q.dtype)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

    def feat_q():
        lib.linattn_performer_features(q, w, K, fq, stream)

    def attn():
        lib.linattn_fwd_causal_ws(fq, fk, v, lam, 1e-6, None, None, out, S, z, ws, stream,
                                  phi=lib.LINATTN_PHI_IDENTITY)

    def step():
        lib.linattn_performer_features(q, w, K, fq, stream)
        lib.linattn_performer_features(k, w, K, fk, stream)
        attn()

    with torch.cuda.stream(stream):
        ms = time_steps(step, args.steps, args.warmup, world, stream)
        ms_f = time_steps(feat_q, args.steps, args.warmup, world, stream)
        ms_a = time_steps(attn, args.steps, args.warmup, world, stream)
    assert lib.linattn_device_status(clear=True, stream=stream) == 0
    per, per_f, per_a = (x / 1e3 / args.steps for x in (ms, ms_f, ms_a))
    fb = features_bytes(B * H * N, d, m)
    ab = causal_bytes(B, H, N, 2 * m, d)
    res = {"workload": f"performer_d128: B={B} x H={H} x N={N}, d={d}, m={m} orthogonal "
                       "features (softmax kernel), bf16, lambda_h=linspace(0.9,0.999,16)",
           "value": B * N * world / per, "unit": "tokens/s", "ms_per_step": per * 1e3,
           "gpu_launches_per_step": 4 if need > 0 else 3,
           "features": {"kernel": "performer_tc_kernel", "ms_per_launch": per_f * 1e3,
                        "roofline": {"bound": "hbm", "achieved": fb / per_f / 1e9, "peak": hbm,
                                     "unit": "GB/s", "frac": fb / per_f / 1e9 / hbm,
                                     "algorithmic_bytes_per_launch": fb,
                                     "traffic": traffic_record("performer_tc_kernel")}},
           "attention": {"kernel": ("causal_seg_state_tc_kernel + causal_seg_tc_kernel (identity "
                                    "features, overlapped)" if need > 0 else
                                    "causal_seg_tc_kernel (identity features)"),
                         "ms_per_launch": per_a * 1e3,
                         "roofline": {"bound": "hbm", "achieved": ab / per_a / 1e9, "peak": hbm,
                                      "unit": "GB/s", "frac": ab / per_a / 1e9 / hbm,
                                      "algorithmic_bytes_per_launch": ab}}}
    del q, k, v, fq, fk, out, ws
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- oracle
def oracle_sample(target_s=12.0, heads=None):
    """Times the fp64 oracle (as it stands) on a bounded sample of the causal
    workload: `heads` heads of a prefix of one sequence, the prefix sized to
    take about target_s seconds; once the prefix is the whole sequence, more
    of the workload's sequences, then repeated calls, until about target_s
    seconds of CPU work.  Returns (tokens/s, cores, description, seconds)."""
    import oracle
    cores = oracle.num_threads(0)
    h = heads or max(1, min(WL.H, cores))
    n = 256
    q, k, v = inputs.causal_inputs(WL, B=1, N=n)
    lam = inputs.decay(WL)
    t0 = time.perf_counter()
    oracle.causal(q[:, :h], k[:, :h], v[:, :h], lam[:h], WL.eps)
    dt = time.perf_counter() - t0
    n = int(min(WL.N, max(256, n * target_s / max(dt, 1e-3))))
    b = 1
    if n == WL.N:
        per_seq = dt * WL.N / 256
        b = int(min(WL.B, max(1, target_s / max(per_seq, 1e-3))))
    q, k, v = inputs.causal_inputs(WL, B=b, N=n)
    q, k, v = q[:, :h].contiguous(), k[:, :h].contiguous(), v[:, :h].contiguous()
    reps, spent = 0, 0.0
    while reps == 0 or spent < target_s * 0.8:
        t0 = time.perf_counter()
        oracle.causal(q, k, v, lam[:h], WL.eps)
        spent += time.perf_counter() - t0
        reps += 1
    # a token of the workload = one position of one sequence across all H heads
    tok_s = reps * b * n * (h / WL.H) / spent
    used = min(cores, b * h)
    desc = (f"oracle causal recurrence (fp64, {used} threads) on {b} sequence(s) x {h}/{WL.H} "
            f"heads x {n} tokens of causal_decay_d128, {reps} call(s), {spent:.1f} s; tokens/s "
            f"scaled by {h}/{WL.H} heads")
    return tok_s, used, desc, spent / reps


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps = []
    per_step_target = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        tok_s, cores, desc, dt = oracle_sample(target_s=per_step_target)
        if i >= args.warmup:
            steps.append((tok_s, dt))
    value = statistics.median(t for t, _ in steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.median(dt for _, dt in steps) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "causal_decay_d128 (B=4,H=16,N=16384,d=128,lambda_h in "
                               "[0.9,0.999]); each step a bounded sample on the host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--segments", type=int, default=0,
                    help="causal leg: ask for at most this many segments per sequence "
                         "(0: the library's plan)")
    ap.add_argument("--seq-parallel", action="store_true",
                    help="causal leg: split each sequence by token position across the "
                         "ranks (each rank N tokens; one all-gather of segment states)")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-legs", dest="legs", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu", action="store_false")
    ap.add_argument("--only", default="all",
                    choices=["all", "causal", "decode", "global", "backward", "segmented",
                             "performer", "tiny"])
    ap.add_argument("--batch", type=int, default=0, help="causal leg batch (profiling)")
    ap.add_argument("--dec-batch", type=int, default=0, help="decode sequences (profiling)")
    ap.add_argument("--dec-steps", type=int, default=0, help="decode steps (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return reference_arm(args)

    world, rank, local = dist_setup()
    from weight_state_recurrence_b200 import linattn as lib
    lib.load()
    hbm, tcp, peak_src = peaks()
    stream = torch.cuda.Stream()

    if args.only in ("decode", "global", "backward", "segmented", "performer", "tiny"):
        if args.only == "tiny":
            r = tiny_leg(lib, args, world, rank, stream, hbm)
        elif args.only == "performer":
            r = performer_leg(lib, args, world, rank, stream, hbm)
        elif args.only == "backward":
            r = bwd_leg(lib, args, world, rank, stream, tcp, hbm)
        elif args.only == "segmented":
            r = seg_leg(lib, args, world, rank, stream, hbm)
        else:
            leg = decode_leg if args.only == "decode" else global_leg
            r = leg(lib, args, world, rank, stream, hbm)
        line = {"metric": METRIC, "leg": args.only, "n_gpus": world, args.only: r}
        if rank == 0:
            print(json.dumps(line), flush=True)
        return 0
    res = causal_leg(lib, args, world, rank, stream, hbm, tcp)
    B = args.batch or WL.B
    line = {
        "metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded torch RNG on the device, N(0,1)/sqrt(d))",
        "config": {"workload": f"causal_decay_d128: B={B} x H=16 x N=16384, d_k=d_v=128, bf16 "
                               "q/k/v, lambda_h=linspace(0.9,0.999,16), fp32 S/z, eps=1e-6",
                   "global_batch": B if args.seq_parallel else B * world,
                   "seq_len": WL.N * (world if args.seq_parallel else 1), "heads": WL.H,
                   "d": WL.d,
                   "parallelism": (f"sp{world} (each sequence split by token position, "
                                   f"{WL.N} tokens per rank; one all-gather of segment "
                                   "states)") if args.seq_parallel else
                                  f"dp{world} (batch sharded, no data-path collective)",
                   "l2": f"inputs larger than L2 ({3 * B * WL.H * WL.N * WL.d * 2 / 1e6:.0f} MB "
                         "per step)"},
        "roofline": res["roofline"], "clocks": res["clocks"],
        "gpu_launches": res["gpu_launches"], "peaks": peak_src,
    }
    if "e2e" in res:
        line["e2e"] = res["e2e"]
    if args.legs and args.only == "all":
        line["decode"] = decode_leg(lib, args, world, rank, stream, hbm)
        line["global"] = global_leg(lib, args, world, rank, stream, hbm)
        line["backward"] = bwd_leg(lib, args, world, rank, stream, tcp, hbm)
        line["segmented"] = seg_leg(lib, args, world, rank, stream, hbm)
        line["performer"] = performer_leg(lib, args, world, rank, stream, hbm)
        line["tiny"] = tiny_leg(lib, args, world, rank, stream, hbm)
    if args.cpu and world == 1 and rank == 0:
        tok_s, cores, desc, _ = oracle_sample()
        line["cpu_baseline"] = {"value": tok_s, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    wdist.finalize()
    return 0


if __name__ == "__main__":
    sys.exit(main())
