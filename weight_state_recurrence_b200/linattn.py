"""Thin ctypes binding over liblinattn.so (include/linattn.h).

The functions named ``linattn_*`` mirror the C entry points one to one and do
argument marshalling only: shapes and dtypes of torch tensors are turned into
a ``linattn_dims`` struct, device pointers and the current CUDA stream.  Every
step of the computation runs in the library's kernels.  There is no CPU or
PyTorch fallback: if the library cannot be loaded, the call raises.

``fwd_causal`` / ``fwd_global`` / ``decode_step`` are conveniences that
allocate the outputs with torch and call the entry points.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblinattn.so")

LINATTN_BF16, LINATTN_F32 = 0, 1
LINATTN_OK = 0
LINATTN_ERR_INVALID = 1
LINATTN_ERR_UNSUPPORTED = 2
LINATTN_ERR_CUDA = 3
LINATTN_ERR_DEVICE = 4
LINATTN_PHI_ELU1, LINATTN_PHI_IDENTITY = 0, 1
LINATTN_PERFORMER_SOFTMAX, LINATTN_PERFORMER_GAUSSIAN = 0, 1
LINATTN_OP_CAUSAL, LINATTN_OP_GLOBAL, LINATTN_OP_PERFORMER, LINATTN_OP_BACKWARD = 0, 1, 2, 3
LINATTN_KERNEL_AUTO, LINATTN_KERNEL_CUDA_CORES, LINATTN_KERNEL_TC_PAIRED = 0, 1, 2

ENTRY_POINTS = ("linattn_fwd_causal", "linattn_fwd_causal_from", "linattn_fwd_causal_workspace",
                "linattn_fwd_causal_ws", "linattn_fwd_causal_noalloc", "linattn_bwd_causal",
                "linattn_fwd_global", "linattn_fwd_global_cross", "linattn_decode_step",
                "linattn_performer_features", "linattn_status_string", "linattn_device_status",
                "linattn_version", "linattn_set_kernel_choice", "linattn_causal_state",
                "linattn_combine_states", "linattn_fwd_global_masked",
                "linattn_bwd_causal_workspace", "linattn_bwd_causal_ws")


class linattn_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("dtype", ctypes.c_int),
                ("phi", ctypes.c_int)]


class LinattnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: status {code} ({status_string(code)})")


_lib = None


def load(build_if_missing: bool = True):
    """Load liblinattn.so (building it with nvcc first if it is missing or
    older than its sources)."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_missing:
        from . import build as _build
        try:
            _build.build()
        except Exception:
            if not os.path.exists(LIB_PATH):
                raise
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library missing: {LIB_PATH}")
    lib = ctypes.CDLL(LIB_PATH)
    vp, fp, i, f = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    dp = ctypes.POINTER(linattn_dims)
    lib.linattn_fwd_causal.argtypes = [dp, vp, vp, vp, fp, f, vp, fp, fp, vp]
    lib.linattn_fwd_causal.restype = i
    lib.linattn_fwd_causal_from.argtypes = [dp, vp, vp, vp, fp, f, fp, fp, vp, fp, fp, vp]
    lib.linattn_fwd_causal_from.restype = i
    lib.linattn_fwd_causal_workspace.argtypes = [dp]
    lib.linattn_fwd_causal_workspace.restype = ctypes.c_size_t
    lib.linattn_fwd_causal_ws.argtypes = [dp, vp, vp, vp, fp, f, fp, fp, vp, fp, fp, vp,
                                          ctypes.c_size_t, vp]
    lib.linattn_fwd_causal_ws.restype = i
    lib.linattn_fwd_causal_noalloc.argtypes = [dp, vp, vp, vp, fp, f, vp, fp, fp, vp]
    lib.linattn_fwd_causal_noalloc.restype = i
    lib.linattn_bwd_causal.argtypes = [dp, vp, vp, vp, fp, f, vp, vp, vp, vp, fp, vp]
    lib.linattn_bwd_causal.restype = i
    lib.linattn_bwd_causal_workspace.argtypes = [dp]
    lib.linattn_bwd_causal_workspace.restype = ctypes.c_size_t
    lib.linattn_bwd_causal_ws.argtypes = [dp, vp, vp, vp, fp, f, vp, vp, vp, vp, fp, vp,
                                          ctypes.c_size_t, vp]
    lib.linattn_bwd_causal_ws.restype = i
    lib.linattn_fwd_global.argtypes = [dp, vp, vp, vp, f, vp, fp, fp, vp]
    lib.linattn_fwd_global.restype = i
    lib.linattn_fwd_global_cross.argtypes = [dp, i, vp, vp, vp, f, vp, fp, fp, vp]
    lib.linattn_fwd_global_cross.restype = i
    lib.linattn_decode_step.argtypes = [dp, vp, vp, vp, fp, f, fp, fp, vp, vp]
    lib.linattn_decode_step.restype = i
    lib.linattn_performer_features.argtypes = [ctypes.c_longlong, i, i, i, i, vp, vp, vp, vp]
    lib.linattn_performer_features.restype = i
    lib.linattn_status_string.argtypes = [i]
    lib.linattn_status_string.restype = ctypes.c_char_p
    lib.linattn_device_status.argtypes = [i, vp]
    lib.linattn_device_status.restype = i
    lib.linattn_version.argtypes = []
    lib.linattn_version.restype = i
    lib.linattn_set_kernel_choice.argtypes = [i, i, i]
    lib.linattn_set_kernel_choice.restype = i
    lib.linattn_causal_state.argtypes = [dp, vp, vp, fp, fp, fp, vp]
    lib.linattn_causal_state.restype = i
    lib.linattn_combine_states.argtypes = [dp, i, fp, fp, fp, fp, fp, vp]
    lib.linattn_combine_states.restype = i
    lib.linattn_fwd_global_masked.argtypes = [dp, i, vp, vp, vp, vp, f, vp, fp, fp, vp]
    lib.linattn_fwd_global_masked.restype = i
    _lib = lib
    return lib


def linattn_set_kernel_choice(op: int, kernel: int, segments: int = 0) -> None:
    """Choose the kernel family of an operation (tests and benchmarks only;
    see include/linattn.h)."""
    _check(load().linattn_set_kernel_choice(int(op), int(kernel), int(segments)),
           "linattn_set_kernel_choice")


class kernel_choice:
    """Context manager: ``with kernel_choice(LINATTN_OP_CAUSAL,
    LINATTN_KERNEL_CUDA_CORES): ...`` runs the block with that kernel family
    and restores the automatic choice afterwards."""

    def __init__(self, op: int, kernel: int, segments: int = 0):
        self.op, self.kernel, self.segments = op, kernel, segments

    def __enter__(self):
        linattn_set_kernel_choice(self.op, self.kernel, self.segments)
        return self

    def __exit__(self, *exc):
        linattn_set_kernel_choice(self.op, LINATTN_KERNEL_AUTO, 0)
        return False


def status_string(code: int) -> str:
    return load().linattn_status_string(int(code)).decode()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return LINATTN_BF16
    if t == torch.float32:
        return LINATTN_F32
    raise TypeError(f"unsupported dtype {t}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(code, where):
    if code != LINATTN_OK:
        raise LinattnError(code, where)


def _f32(t, shape, name):
    if t is None:
        return
    if t.dtype != torch.float32 or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be float32 with shape {tuple(shape)}")


def linattn_fwd_causal(q, k, v, lam, eps, out, S_final=None, z_final=None, stream=None, *,
                       phi=LINATTN_PHI_ELU1):
    """Causal forward: q, k [B,H,N,dk], v/out [B,H,N,dv] (bf16 or fp32),
    lam [H] fp32 or None, S_final [B,H,dk,dv] / z_final [B,H,dk] fp32 or None."""
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or tuple(v.shape) != (B, H, N, dv) or out.shape != v.shape:
        raise ValueError("shape mismatch among q, k, v, out")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("q, k, v, out must share one dtype")
    _f32(lam, (H,), "lambda")
    _f32(S_final, (B, H, dk, dv), "S_final")
    _f32(z_final, (B, H, dk), "z_final")
    d = linattn_dims(B, H, N, dk, dv, _dtype_code(q.dtype), int(phi))
    _check(load().linattn_fwd_causal(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                     float(eps), _ptr(out), _ptr(S_final), _ptr(z_final),
                                     _stream(stream)), "linattn_fwd_causal")


def linattn_fwd_causal_from(q, k, v, lam, eps, S_init, z_init, out, S_final=None, z_final=None,
                            stream=None, *, phi=LINATTN_PHI_ELU1):
    """Causal forward continued from (S_init [B,H,dk,dv], z_init [B,H,dk]) fp32,
    both given or both None; the other arguments as linattn_fwd_causal."""
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or tuple(v.shape) != (B, H, N, dv) or out.shape != v.shape:
        raise ValueError("shape mismatch among q, k, v, out")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("q, k, v, out must share one dtype")
    _f32(lam, (H,), "lambda")
    _f32(S_init, (B, H, dk, dv), "S_init")
    _f32(z_init, (B, H, dk), "z_init")
    _f32(S_final, (B, H, dk, dv), "S_final")
    _f32(z_final, (B, H, dk), "z_final")
    d = linattn_dims(B, H, N, dk, dv, _dtype_code(q.dtype), int(phi))
    _check(load().linattn_fwd_causal_from(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                          float(eps), _ptr(S_init), _ptr(z_init), _ptr(out),
                                          _ptr(S_final), _ptr(z_final), _stream(stream)),
           "linattn_fwd_causal_from")


def _causal_dims(q, k, v, out, S_final, z_final, lam, phi=LINATTN_PHI_ELU1):
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or tuple(v.shape) != (B, H, N, dv) or out.shape != v.shape:
        raise ValueError("shape mismatch among q, k, v, out")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("q, k, v, out must share one dtype")
    _f32(lam, (H,), "lambda")
    _f32(S_final, (B, H, dk, dv), "S_final")
    _f32(z_final, (B, H, dk), "z_final")
    return linattn_dims(B, H, N, dk, dv, _dtype_code(q.dtype), int(phi))


def linattn_fwd_causal_workspace(B, H, N, dk, dv, dtype, phi=LINATTN_PHI_ELU1) -> int:
    """Workspace bytes the segment-parallel causal forward wants (0: none)."""
    d = linattn_dims(B, H, N, dk, dv, _dtype_code(dtype), int(phi))
    return int(load().linattn_fwd_causal_workspace(ctypes.byref(d)))


def linattn_fwd_causal_ws(q, k, v, lam, eps, S_init, z_init, out, S_final, z_final, workspace,
                          stream=None, *, phi=LINATTN_PHI_ELU1):
    """Causal forward (optionally from S_init, z_init) with a caller workspace:
    a CUDA tensor of at least linattn_fwd_causal_workspace bytes, or None."""
    d = _causal_dims(q, k, v, out, S_final, z_final, lam, phi)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().linattn_fwd_causal_ws(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                        float(eps), _ptr(S_init), _ptr(z_init), _ptr(out),
                                        _ptr(S_final), _ptr(z_final), _ptr(workspace),
                                        ctypes.c_size_t(nbytes), _stream(stream)),
           "linattn_fwd_causal_ws")


def linattn_fwd_causal_noalloc(q, k, v, lam, eps, out, S_final=None, z_final=None, stream=None,
                               *, phi=LINATTN_PHI_ELU1):
    """linattn_fwd_causal whose segment-parallel form uses the library's own scratch."""
    d = _causal_dims(q, k, v, out, S_final, z_final, lam, phi)
    _check(load().linattn_fwd_causal_noalloc(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v),
                                             _ptr(lam), float(eps), _ptr(out), _ptr(S_final),
                                             _ptr(z_final), _stream(stream)),
           "linattn_fwd_causal_noalloc")


def linattn_bwd_causal_workspace(B, H, N, dk, dv, dtype, phi=LINATTN_PHI_ELU1) -> int:
    d = linattn_dims(B, H, N, dk, dv, _dtype_code(dtype), int(phi))
    return int(load().linattn_bwd_causal_workspace(ctypes.byref(d)))


def linattn_bwd_causal(q, k, v, lam, eps, dy, dq, dk, dv, dlam=None, stream=None, *,
                       phi=LINATTN_PHI_ELU1, workspace=None):
    """Backward of the causal forward: dy like v; dq, dk like q; dv like v;
    dlam [H] fp32 or None; workspace: a uint8 device tensor for
    linattn_bwd_causal_ws (None: linattn_bwd_causal)."""
    B, H, N, dk_ = q.shape
    dv_ = v.shape[-1]
    if (k.shape != q.shape or tuple(v.shape) != (B, H, N, dv_) or dy.shape != v.shape or
            dq.shape != q.shape or dk.shape != q.shape or dv.shape != v.shape):
        raise ValueError("shape mismatch among q, k, v, dy, dq, dk, dv")
    if len({t.dtype for t in (q, k, v, dy, dq, dk, dv)}) != 1:
        raise ValueError("q, k, v, dy, dq, dk, dv must share one dtype")
    _f32(lam, (H,), "lambda")
    _f32(dlam, (H,), "dlambda")
    d = linattn_dims(B, H, N, dk_, dv_, _dtype_code(q.dtype), int(phi))
    if workspace is not None:
        _check(load().linattn_bwd_causal_ws(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                            float(eps), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv),
                                            _ptr(dlam), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(),
                                            _stream(stream)), "linattn_bwd_causal_ws")
        return
    _check(load().linattn_bwd_causal(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                     float(eps), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv),
                                     _ptr(dlam), _stream(stream)), "linattn_bwd_causal")


def linattn_fwd_global(q, k, v, eps, out, KV, ksum, stream=None, *, phi=LINATTN_PHI_ELU1):
    """Global forward: q, k [B,H,N,dk], v/out [B,H,N,dv]; KV [B,H,dk,dv] and
    ksum [B,H,dk] fp32 are written."""
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or tuple(v.shape) != (B, H, N, dv) or out.shape != v.shape:
        raise ValueError("shape mismatch among q, k, v, out")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("q, k, v, out must share one dtype")
    _f32(KV, (B, H, dk, dv), "KV")
    _f32(ksum, (B, H, dk), "ksum")
    d = linattn_dims(B, H, N, dk, dv, _dtype_code(q.dtype), int(phi))
    _check(load().linattn_fwd_global(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), float(eps),
                                     _ptr(out), _ptr(KV), _ptr(ksum), _stream(stream)),
           "linattn_fwd_global")


def linattn_fwd_global_cross(q, k, v, eps, out, KV, ksum, stream=None, *,
                             phi=LINATTN_PHI_ELU1):
    """Cross global forward: q/out [B,H,Nq,dk/dv], k/v [B,H,Nk,dk/dv];
    KV [B,H,dk,dv] and ksum [B,H,dk] fp32 (written)."""
    B, H, Nq, dk = q.shape
    Nk, dv = k.shape[2], v.shape[-1]
    if (tuple(k.shape) != (B, H, Nk, dk) or tuple(v.shape) != (B, H, Nk, dv) or
            tuple(out.shape) != (B, H, Nq, dv)):
        raise ValueError("shape mismatch among q, k, v, out")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("q, k, v, out must share one dtype")
    _f32(KV, (B, H, dk, dv), "KV")
    _f32(ksum, (B, H, dk), "ksum")
    d = linattn_dims(B, H, Nq, dk, dv, _dtype_code(q.dtype), int(phi))
    _check(load().linattn_fwd_global_cross(ctypes.byref(d), int(Nk), _ptr(q), _ptr(k), _ptr(v),
                                           float(eps), _ptr(out), _ptr(KV), _ptr(ksum),
                                           _stream(stream)), "linattn_fwd_global_cross")


def linattn_fwd_global_masked(q, k, v, key_padding_mask, eps, out, KV, ksum, stream=None, *,
                              phi=LINATTN_PHI_ELU1):
    """Cross global forward with a key padding mask [B, Nk] (bool or uint8,
    nonzero = padding, on the device; None = no padding); the other arguments
    as linattn_fwd_global_cross."""
    B, H, Nq, dk = q.shape
    Nk, dv = k.shape[2], v.shape[-1]
    if (tuple(k.shape) != (B, H, Nk, dk) or tuple(v.shape) != (B, H, Nk, dv) or
            tuple(out.shape) != (B, H, Nq, dv)):
        raise ValueError("shape mismatch among q, k, v, out")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("q, k, v, out must share one dtype")
    _f32(KV, (B, H, dk, dv), "KV")
    _f32(ksum, (B, H, dk), "ksum")
    m = key_padding_mask
    if m is not None:
        if tuple(m.shape) != (B, Nk) or m.dtype not in (torch.bool, torch.uint8):
            raise ValueError(f"key_padding_mask must be bool/uint8 with shape {(B, Nk)}")
        m = m.view(torch.uint8) if m.dtype == torch.bool else m
    d = linattn_dims(B, H, Nq, dk, dv, _dtype_code(q.dtype), int(phi))
    _check(load().linattn_fwd_global_masked(ctypes.byref(d), int(Nk), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(m), float(eps), _ptr(out), _ptr(KV), _ptr(ksum),
                                            _stream(stream)), "linattn_fwd_global_masked")


def linattn_decode_step(q, k, v, lam, eps, S, z, out, stream=None, *, phi=LINATTN_PHI_ELU1):
    """One decode step: q, k [B,H,dk], v/out [B,H,dv]; S [B,H,dk,dv] and z
    [B,H,dk] fp32 are updated in place."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or tuple(v.shape) != (B, H, dv) or out.shape != v.shape:
        raise ValueError("shape mismatch among q, k, v, out")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("q, k, v, out must share one dtype")
    _f32(lam, (H,), "lambda")
    _f32(S, (B, H, dk, dv), "S")
    _f32(z, (B, H, dk), "z")
    d = linattn_dims(B, H, 1, dk, dv, _dtype_code(q.dtype), int(phi))
    _check(load().linattn_decode_step(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                      float(eps), _ptr(S), _ptr(z), _ptr(out), _stream(stream)),
           "linattn_decode_step")


def linattn_performer_features(x, omega, kernel, out, stream=None):
    """Performer random features: x [..., d] (rows = the product of the
    leading dims), omega [m, d], out [..., 2m], one dtype; kernel
    LINATTN_PERFORMER_SOFTMAX or LINATTN_PERFORMER_GAUSSIAN."""
    d = x.shape[-1]
    if omega.dim() != 2 or omega.shape[1] != d:
        raise ValueError("omega must have shape [m, d]")
    m = omega.shape[0]
    if tuple(out.shape) != tuple(x.shape[:-1]) + (2 * m,):
        raise ValueError("out must have shape x.shape[:-1] + (2m,)")
    if not (x.dtype == omega.dtype == out.dtype):
        raise ValueError("x, omega, out must share one dtype")
    rows = x.numel() // d if d else 0
    _check(load().linattn_performer_features(ctypes.c_longlong(rows), int(d), int(m), int(kernel),
                                             _dtype_code(x.dtype), _ptr(x), _ptr(omega),
                                             _ptr(out), _stream(stream)),
           "linattn_performer_features")


def linattn_causal_state(k, v, lam, S, z, stream=None, *, phi=LINATTN_PHI_ELU1):
    """State-only pass: S [B,H,dk,dv], z [B,H,dk] fp32 (written) from
    k [B,H,N,dk], v [B,H,N,dv] and lam [H] fp32 or None."""
    B, H, N, dk = k.shape
    dv = v.shape[-1]
    if tuple(v.shape) != (B, H, N, dv) or k.dtype != v.dtype:
        raise ValueError("k and v must agree in B, H, N and dtype")
    _f32(lam, (H,), "lambda")
    _f32(S, (B, H, dk, dv), "S")
    _f32(z, (B, H, dk), "z")
    d = linattn_dims(B, H, N, dk, dv, _dtype_code(k.dtype), int(phi))
    _check(load().linattn_causal_state(ctypes.byref(d), _ptr(k), _ptr(v), _ptr(lam), _ptr(S),
                                       _ptr(z), _stream(stream)), "linattn_causal_state")


def linattn_combine_states(seg_len, lam, S_init, z_init, dS, dz, stream=None):
    """In place: slots dS [G,B,H,dk,dv], dz [G,B,H,dk] fp32 holding segment
    states become the states at the start of each segment of seg_len tokens."""
    G, B, H, dk, dv = dS.shape
    _f32(dz, (G, B, H, dk), "dz")
    _f32(lam, (H,), "lambda")
    _f32(S_init, (B, H, dk, dv), "S_init")
    _f32(z_init, (B, H, dk), "z_init")
    d = linattn_dims(B, H, int(seg_len), dk, dv, LINATTN_F32, LINATTN_PHI_ELU1)
    _check(load().linattn_combine_states(ctypes.byref(d), int(G), _ptr(lam), _ptr(S_init),
                                         _ptr(z_init), _ptr(dS), _ptr(dz), _stream(stream)),
           "linattn_combine_states")


def linattn_status_string(code: int) -> str:
    return status_string(code)


def linattn_device_status(clear: bool = True, stream=None) -> int:
    return load().linattn_device_status(int(bool(clear)), _stream(stream))


def linattn_version() -> int:
    return load().linattn_version()


# ---------------------------------------------------------------- helpers
def fwd_causal(q, k, v, lam=None, eps=1e-6, want_state=True, S_init=None, z_init=None,
               stream=None, phi=LINATTN_PHI_ELU1):
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    out = torch.empty_like(v)
    S = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if want_state else None
    z = torch.empty((B, H, dk), dtype=torch.float32, device=q.device) if want_state else None
    if S_init is None and z_init is None:
        linattn_fwd_causal(q, k, v, lam, eps, out, S, z, stream, phi=phi)
    else:
        linattn_fwd_causal_from(q, k, v, lam, eps, S_init, z_init, out, S, z, stream, phi=phi)
    return out, S, z


def bwd_causal(q, k, v, dy, lam=None, eps=1e-6, want_dlam=False, stream=None,
               phi=LINATTN_PHI_ELU1, workspace=None):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dlam = (torch.empty(q.shape[1], dtype=torch.float32, device=q.device) if want_dlam else None)
    linattn_bwd_causal(q, k, v, lam, eps, dy, dq, dk, dv, dlam, stream, phi=phi,
                       workspace=workspace)
    return dq, dk, dv, dlam


def fwd_global(q, k, v, eps=1e-6, stream=None, phi=LINATTN_PHI_ELU1):
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    out = torch.empty_like(v)
    KV = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ks = torch.empty((B, H, dk), dtype=torch.float32, device=q.device)
    linattn_fwd_global(q, k, v, eps, out, KV, ks, stream, phi=phi)
    return out, KV, ks


def fwd_global_cross(q, k, v, eps=1e-6, stream=None, phi=LINATTN_PHI_ELU1):
    B, H, Nq, dk = q.shape
    dv = v.shape[-1]
    out = torch.empty((B, H, Nq, dv), dtype=v.dtype, device=v.device)
    KV = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ks = torch.empty((B, H, dk), dtype=torch.float32, device=q.device)
    linattn_fwd_global_cross(q, k, v, eps, out, KV, ks, stream, phi=phi)
    return out, KV, ks


def fwd_global_masked(q, k, v, key_padding_mask, eps=1e-6, stream=None, phi=LINATTN_PHI_ELU1):
    B, H, Nq, dk = q.shape
    dv = v.shape[-1]
    out = torch.empty((B, H, Nq, dv), dtype=v.dtype, device=v.device)
    KV = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ks = torch.empty((B, H, dk), dtype=torch.float32, device=q.device)
    linattn_fwd_global_masked(q, k, v, key_padding_mask, eps, out, KV, ks, stream, phi=phi)
    return out, KV, ks


def decode_step(q, k, v, S, z, lam=None, eps=1e-6, stream=None, phi=LINATTN_PHI_ELU1):
    out = torch.empty_like(v)
    linattn_decode_step(q, k, v, lam, eps, S, z, out, stream, phi=phi)
    return out


def performer_features(x, omega, kernel=LINATTN_PERFORMER_SOFTMAX, stream=None):
    out = torch.empty(tuple(x.shape[:-1]) + (2 * omega.shape[0],), dtype=x.dtype, device=x.device)
    linattn_performer_features(x, omega, kernel, out, stream)
    return out


def performer_causal(q, k, v, omega, lam=None, eps=1e-6, kernel=LINATTN_PERFORMER_SOFTMAX,
                     want_state=True, stream=None):
    """Causal attention on Performer features: the features of q and k
    ([B,H,N,2m]) from linattn_performer_features, then the causal forward in
    identity mode.  Returns (out, S_final, z_final)."""
    fq = performer_features(q, omega, kernel, stream)
    fk = performer_features(k, omega, kernel, stream)
    return fwd_causal(fq, fk, v, lam, eps, want_state, stream=stream, phi=LINATTN_PHI_IDENTITY)


def fwd_causal_host(q, k, v, lam=None, eps=1e-6, out=None, S_final=None, z_final=None,
                    pieces=None, device=None):
    """Causal forward on host-resident tensors (pinned for the copies to be
    asynchronous).  Every (sequence, head) is independent, so the B*H heads are
    cut into ``pieces`` runs of heads of one sequence (default: runs of 4
    heads, or whole sequences when H is not a multiple of 4) whose
    host-to-device copies, kernels and device-to-host copies run on three
    streams: the copies of one piece overlap the kernels and copies of the
    others, and the two copy directions overlap each other.  The device holds
    two pieces at a time.  ``out`` [B,H,N,dv] (q's dtype), ``S_final``
    [B,H,dk,dv] and ``z_final`` [B,H,dk] fp32 are host tensors, allocated
    (pinned) when None.  Returns (out, S_final, z_final); on return every copy
    has landed."""
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    pin = lambda shape, dt: torch.empty(shape, dtype=dt, pin_memory=True)
    out = pin((B, H, N, dv), q.dtype) if out is None else out
    S_final = pin((B, H, dk, dv), torch.float32) if S_final is None else S_final
    z_final = pin((B, H, dk), torch.float32) if z_final is None else z_final
    per_seq = max(1, (pieces or 4 * B) // max(B, 1))
    hp = max(1, -(-H // per_seq))               # heads per piece
    runs = [(b, h0, min(H, h0 + hp)) for b in range(B) for h0 in range(0, H, hp)]
    lam_d = None if lam is None else lam.to(dev, non_blocking=True)
    # one 16-byte aligned copy of lambda per head offset (the C ABI wants aligned pointers)
    lam_runs = {} if lam_d is None else {h0: lam_d[h0:h1].clone() for _, h0, h1 in runs}
    slots = [dict(q=torch.empty((hp, N, dk), dtype=q.dtype, device=dev),
                  k=torch.empty((hp, N, dk), dtype=q.dtype, device=dev),
                  v=torch.empty((hp, N, dv), dtype=q.dtype, device=dev),
                  y=torch.empty((hp, N, dv), dtype=q.dtype, device=dev),
                  S=torch.empty((hp, dk, dv), dtype=torch.float32, device=dev),
                  z=torch.empty((hp, dk), dtype=torch.float32, device=dev),
                  inputs_free=None, outputs_free=None) for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    cur = torch.cuda.current_stream(dev)
    for s in (s_in, s_cmp, s_out):
        s.wait_stream(cur)          # lambda and the slots are ready
    for p, (b, h0, h1) in enumerate(runs):
        sl, nh = slots[p % 2], h1 - h0
        with torch.cuda.stream(s_in):
            if sl["inputs_free"] is not None:
                s_in.wait_event(sl["inputs_free"])
            sl["q"][:nh].copy_(q[b, h0:h1], non_blocking=True)
            sl["k"][:nh].copy_(k[b, h0:h1], non_blocking=True)
            sl["v"][:nh].copy_(v[b, h0:h1], non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(s_in)
        s_cmp.wait_event(ready)
        if sl["outputs_free"] is not None:
            s_cmp.wait_event(sl["outputs_free"])
        view = lambda t: t[:nh].unsqueeze(0)   # [1, nh, ...]: one sequence, nh heads
        linattn_fwd_causal(view(sl["q"]), view(sl["k"]), view(sl["v"]), lam_runs.get(h0), eps,
                           view(sl["y"]), view(sl["S"]), view(sl["z"]), s_cmp)
        done = torch.cuda.Event()
        done.record(s_cmp)
        sl["inputs_free"] = done
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            out[b, h0:h1].copy_(sl["y"][:nh], non_blocking=True)
            S_final[b, h0:h1].copy_(sl["S"][:nh], non_blocking=True)
            z_final[b, h0:h1].copy_(sl["z"][:nh], non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_out)
        sl["outputs_free"] = landed
    s_out.synchronize()
    return out, S_final, z_final
