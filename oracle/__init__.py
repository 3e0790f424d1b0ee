"""Reference oracle (fp64, CPU) for causal linear attention as a fast-weight
recurrence.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product library (``weight_state_recurrence_b200``) never imports
it, and this package imports nothing from the product.

The arithmetic lives in ``linattn_oracle.c`` (plain scalar double loops); this
module only builds it with gcc, loads it with ctypes and marshals arrays.
Inputs are widened exactly to float64 before the call, so bf16/fp32 tensors
reach the oracle with the bit patterns the GPU sees.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "linattn_oracle.c")
_LIB = os.path.join(_HERE, "liblinattn_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE double, no fast-math, no FMA
    contraction) into ``oracle/liblinattn_oracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
             "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i, d = ctypes.c_int, ctypes.c_double
        lib.oracle_causal.argtypes = [i, i, i, i, i, _dp, _dp, _dp, _dp, d, _dp, _dp,
                                      _dp, _dp, _dp, i]
        lib.oracle_causal.restype = i
        lib.oracle_decode_step.argtypes = [i, i, i, i, _dp, _dp, _dp, _dp, d, _dp, _dp,
                                           _dp, i]
        lib.oracle_decode_step.restype = i
        lib.oracle_global.argtypes = [i, i, i, i, i, _dp, _dp, _dp, d, _dp, _dp, _dp, i]
        lib.oracle_global.restype = i
        lib.oracle_global_cross.argtypes = [i, i, i, i, i, i, _dp, _dp, _dp, d, _dp, _dp, _dp, i]
        lib.oracle_global_cross.restype = i
        lib.oracle_global_masked.argtypes = [i, i, i, i, i, i, _dp, _dp, _dp,
                                             ctypes.POINTER(ctypes.c_ubyte), d, _dp, _dp, _dp, i]
        lib.oracle_global_masked.restype = i
        lib.oracle_feature_map.argtypes = [ctypes.c_long, _dp, _dp]
        lib.oracle_feature_map.restype = None
        lib.oracle_num_threads.argtypes = [i]
        lib.oracle_num_threads.restype = i
        _lib = lib
    return _lib


def _f64(x):
    """Exact widening to a C-contiguous float64 numpy array (torch tensors are
    moved to the CPU first; bf16 and fp32 both widen exactly)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def num_threads(nthreads: int = 0) -> int:
    return _load().oracle_num_threads(int(nthreads))


def feature_map(x):
    """phi(x) = elu(x) + 1, elementwise, in float64."""
    a = _f64(x)
    out = np.empty_like(a)
    _load().oracle_feature_map(a.size, _ptr(a), _ptr(out))
    return out


def causal(q, k, v, lam=None, eps=1e-6, S0=None, z0=None, nthreads=0):
    """Causal recurrence over [B, H, N, d] inputs.

    Returns ``(y [B,H,N,dv], S_N [B,H,dk,dv], z_N [B,H,dk])`` in float64.
    ``lam`` is a per-head decay ``[H]`` (None: no decay).  ``S0``/``z0`` give a
    starting state (None: zeros)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (B, H, N, dk) or v.shape != (B, H, N, dv):
        raise ValueError("q, k, v shapes disagree")
    lam = _f64(lam)
    if lam is not None and lam.shape != (H,):
        raise ValueError("lambda must have shape [H]")
    S0, z0 = _f64(S0), _f64(z0)
    y = np.empty((B, H, N, dv))
    S = np.empty((B, H, dk, dv))
    z = np.empty((B, H, dk))
    rc = _load().oracle_causal(B, H, N, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                               float(eps), _ptr(S0), _ptr(z0), _ptr(y), _ptr(S), _ptr(z),
                               int(nthreads))
    if rc != 0:
        raise ValueError("oracle_causal rejected its arguments")
    return y, S, z


def decode_step(q, k, v, S, z, lam=None, eps=1e-6, nthreads=0):
    """One decode step on [B, H, d] inputs from state (S, z).

    Returns ``(y [B,H,dv], S_new, z_new)``; the inputs S and z are not
    modified."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, dk = q.shape
    dv = v.shape[-1]
    S = _f64(S).copy()
    z = _f64(z).copy()
    lam = _f64(lam)
    y = np.empty((B, H, dv))
    rc = _load().oracle_decode_step(B, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                    float(eps), _ptr(S), _ptr(z), _ptr(y), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_decode_step rejected its arguments")
    return y, S, z


def global_cross(q, k, v, eps=1e-6, nthreads=0):
    """Cross form: q ``[B,H,Nq,dk]`` attends to k ``[B,H,Nk,dk]``, v ``[B,H,Nk,dv]``.
    Returns ``(y [B,H,Nq,dv], KV [B,H,dk,dv], ks [B,H,dk])``."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, dk = q.shape
    Nk, dv = k.shape[2], v.shape[-1]
    y = np.empty((B, H, Nq, dv))
    KV = np.empty((B, H, dk, dv))
    ks = np.empty((B, H, dk))
    rc = _load().oracle_global_cross(B, H, Nq, Nk, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                     float(eps), _ptr(y), _ptr(KV), _ptr(ks), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_global_cross rejected its arguments")
    return y, KV, ks


def global_masked(q, k, v, key_padding_mask, eps=1e-6, nthreads=0):
    """Cross form with a key padding mask ``[B, Nk]`` (nonzero: padding, left
    out of both sums; None: no padding).  Returns ``(y, KV, ks)`` as
    ``global_cross``."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, dk = q.shape
    Nk, dv = k.shape[2], v.shape[-1]
    pad = None
    if key_padding_mask is not None:
        m = key_padding_mask
        if hasattr(m, "detach"):
            m = m.detach().to("cpu").numpy()
        pad = np.ascontiguousarray(np.asarray(m) != 0, dtype=np.uint8)
        if pad.shape != (B, Nk):
            raise ValueError("key_padding_mask must have shape [B, Nk]")
    y = np.empty((B, H, Nq, dv))
    KV = np.empty((B, H, dk, dv))
    ks = np.empty((B, H, dk))
    rc = _load().oracle_global_masked(
        B, H, Nq, Nk, dk, dv, _ptr(q), _ptr(k), _ptr(v),
        None if pad is None else pad.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)), float(eps),
        _ptr(y), _ptr(KV), _ptr(ks), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_global_masked rejected its arguments")
    return y, KV, ks


def global_attn(q, k, v, eps=1e-6, nthreads=0):
    """Non-causal form.  Returns ``(y [B,H,N,dv], KV [B,H,dk,dv], ks [B,H,dk])``."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    y = np.empty((B, H, N, dv))
    KV = np.empty((B, H, dk, dv))
    ks = np.empty((B, H, dk))
    rc = _load().oracle_global(B, H, N, dk, dv, _ptr(q), _ptr(k), _ptr(v), float(eps),
                               _ptr(y), _ptr(KV), _ptr(ks), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_global rejected its arguments")
    return y, KV, ks
