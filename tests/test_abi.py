"""Host-side checks of the C ABI (no GPU needed).

The library must load on a machine without a GPU, export every entry point
that include/linattn.h declares, and reject bad arguments with the documented
status code before anything is queued.  Only argument combinations that are
rejected on the host are exercised here, so no kernel is ever launched.
"""
import ctypes
import os
import re
import subprocess

import pytest

from weight_state_recurrence_b200 import linattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "linattn.h")


def declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"\b(linattn_[a-z_]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    return linattn.load()


def test_header_declares_the_entry_points():
    assert set(declared()) == set(linattn.ENTRY_POINTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", linattn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for name in declared():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # nothing else leaks out of the library (hidden visibility)
    extra = {e for e in exported if e.startswith("linattn_")} - set(declared())
    assert not extra, extra


def test_status_strings_and_version(lib):
    for code in range(5):
        s = linattn.status_string(code)
        assert isinstance(s, str) and s
    assert linattn.status_string(99) == "unknown status"
    assert lib.linattn_version() >= 100


def D(B=1, H=1, N=8, dk=64, dv=64, dtype=0):
    return linattn.linattn_dims(B, H, N, dk, dv, dtype)


P = ctypes.c_void_p
FAKE = P(0x7F0000000000)   # never dereferenced: every call below fails validation
FAKE2 = P(0x7F0000100000)
FAKE3 = P(0x7F0000200000)
FAKE4 = P(0x7F0000300000)
MIS = P(0x7F0000400008)    # 8-byte aligned only


def causal(lib, d, q=FAKE, k=FAKE2, v=FAKE3, lam=None, eps=1e-6, out=FAKE4, S=None, z=None):
    return lib.linattn_fwd_causal(ctypes.byref(d) if d is not None else None, q, k, v, lam,
                                  eps, out, S, z, None)


def test_causal_rejects_bad_arguments(lib):
    assert causal(lib, None) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(B=-1)) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(N=-3)) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(dk=48)) == linattn.LINATTN_ERR_UNSUPPORTED
    assert causal(lib, D(dv=256)) == linattn.LINATTN_ERR_UNSUPPORTED
    assert causal(lib, D(dtype=7)) == linattn.LINATTN_ERR_UNSUPPORTED
    assert causal(lib, D(B=1 << 12, H=1 << 10, N=1 << 10)) == linattn.LINATTN_ERR_UNSUPPORTED
    assert causal(lib, D(), eps=-1.0) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(), eps=float("nan")) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(), eps=float("inf")) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(), q=None) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(), out=None) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(), q=MIS) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(), S=MIS) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(), lam=MIS) == linattn.LINATTN_ERR_INVALID
    # output aliasing an input
    assert causal(lib, D(), out=FAKE3) == linattn.LINATTN_ERR_INVALID
    assert causal(lib, D(), out=FAKE) == linattn.LINATTN_ERR_INVALID


def test_causal_from_rejects_bad_state_arguments(lib):
    S0, z0 = P(0x7F0000500000), P(0x7F0000600000)
    Sf, zf = P(0x7F0000700000), P(0x7F0000800000)
    cf = lambda **kw: lib.linattn_fwd_causal_from(
        ctypes.byref(kw.get("d", D())), FAKE, FAKE2, FAKE3, None, 1e-6, kw.get("S0", S0),
        kw.get("z0", z0), kw.get("out", FAKE4), kw.get("Sf", Sf), kw.get("zf", zf), None)
    assert cf(z0=None) == linattn.LINATTN_ERR_INVALID        # one of the pair missing
    assert cf(S0=None) == linattn.LINATTN_ERR_INVALID
    assert cf(S0=MIS) == linattn.LINATTN_ERR_INVALID
    assert cf(z0=MIS) == linattn.LINATTN_ERR_INVALID
    assert cf(Sf=S0) == linattn.LINATTN_ERR_INVALID          # state read and written in place
    assert cf(zf=z0) == linattn.LINATTN_ERR_INVALID
    assert cf(out=S0) == linattn.LINATTN_ERR_INVALID
    assert cf(d=D(dk=48)) == linattn.LINATTN_ERR_UNSUPPORTED


def test_bwd_rejects_bad_arguments(lib):
    DY, DQ, DK, DV = (P(0x7F0000500000), P(0x7F0000600000), P(0x7F0000700000),
                      P(0x7F0000800000))
    bw = lambda **kw: lib.linattn_bwd_causal(
        ctypes.byref(kw.get("d", D())), FAKE, FAKE2, FAKE3, kw.get("lam", None),
        kw.get("eps", 1e-6), kw.get("dy", DY), kw.get("dq", DQ), kw.get("dk", DK),
        kw.get("dv", DV), kw.get("dl", None), None)
    assert bw(dy=None) == linattn.LINATTN_ERR_INVALID
    assert bw(dq=None) == linattn.LINATTN_ERR_INVALID
    assert bw(dk=MIS) == linattn.LINATTN_ERR_INVALID
    assert bw(eps=-1.0) == linattn.LINATTN_ERR_INVALID
    assert bw(d=D(dv=24)) == linattn.LINATTN_ERR_UNSUPPORTED
    assert bw(dq=FAKE) == linattn.LINATTN_ERR_INVALID        # gradient over an input
    assert bw(dv=DY) == linattn.LINATTN_ERR_INVALID
    assert bw(dk=DQ) == linattn.LINATTN_ERR_INVALID          # two gradients overlap
    assert bw(dl=MIS) == linattn.LINATTN_ERR_INVALID


def test_bwd_workspace_entry_points_on_the_host(lib):
    DY, DQ, DK, DV = (P(0x7F0000500000), P(0x7F0000600000), P(0x7F0000700000),
                      P(0x7F0000800000))
    WS = P(0x7F0000900000)
    bw = lambda **kw: lib.linattn_bwd_causal_ws(
        ctypes.byref(kw.get("d", D())), FAKE, FAKE2, FAKE3, None, 1e-6, DY, DQ, DK, DV, None,
        kw.get("ws", WS), kw.get("nb", 1 << 20), None)
    assert bw(ws=None, nb=64) == linattn.LINATTN_ERR_INVALID     # NULL with bytes
    assert bw(ws=MIS) == linattn.LINATTN_ERR_INVALID             # unaligned
    assert bw(ws=DQ) == linattn.LINATTN_ERR_INVALID              # over an output
    assert bw(ws=FAKE) == linattn.LINATTN_ERR_INVALID            # over an input
    assert bw(d=D(dv=24)) == linattn.LINATTN_ERR_UNSUPPORTED
    # the CUDA-core kernel (fp32, or d != 128) needs no workspace
    wsq = lambda d: lib.linattn_bwd_causal_workspace(ctypes.byref(d))
    assert wsq(D()) == 0
    bf = linattn.linattn_dims(2, 3, 300, 128, 128, linattn.LINATTN_BF16, 0)
    # the tensor-core passes: at least the 8-byte stash of every token
    assert wsq(bf) >= 2 * 3 * 300 * 8
    assert wsq(linattn.linattn_dims(2, 3, 0, 128, 128, linattn.LINATTN_BF16, 0)) == 0


def test_global_cross_rejects_bad_arguments(lib):
    KV, ks = P(0x7F0000500000), P(0x7F0000600000)
    gc = lambda **kw: lib.linattn_fwd_global_cross(
        ctypes.byref(kw.get("d", D())), kw.get("nk", 8), FAKE, FAKE2, FAKE3, 1e-6,
        kw.get("out", FAKE4), kw.get("KV", KV), kw.get("ks", ks), None)
    assert gc(nk=-1) == linattn.LINATTN_ERR_INVALID
    assert gc(KV=None) == linattn.LINATTN_ERR_INVALID
    assert gc(out=FAKE2) == linattn.LINATTN_ERR_INVALID      # output over the keys
    assert gc(KV=FAKE) == linattn.LINATTN_ERR_INVALID        # KV over the queries
    assert gc(nk=1 << 30) == linattn.LINATTN_ERR_UNSUPPORTED
    assert gc(d=D(dk=20)) == linattn.LINATTN_ERR_UNSUPPORTED


def test_empty_batch_is_a_no_op(lib):
    # B*H == 0: nothing to do, nothing launched, even with NULL buffers
    assert causal(lib, D(B=0), q=None, k=None, v=None, out=None) == linattn.LINATTN_OK
    d = D(H=0)
    assert lib.linattn_fwd_global(ctypes.byref(d), None, None, None, 1e-6, None, None, None,
                                  None) == linattn.LINATTN_OK
    assert lib.linattn_decode_step(ctypes.byref(d), None, None, None, None, 1e-6, None, None,
                                   None, None) == linattn.LINATTN_OK


def test_global_rejects_bad_arguments(lib):
    d = D()
    g = lambda **kw: lib.linattn_fwd_global(ctypes.byref(kw.get("d", d)), kw.get("q", FAKE),
                                            FAKE2, FAKE3, kw.get("eps", 1e-6),
                                            kw.get("out", FAKE4), kw.get("KV", P(0x7F0000500000)),
                                            kw.get("ks", P(0x7F0000600000)), None)
    assert g(KV=None) == linattn.LINATTN_ERR_INVALID
    assert g(ks=None) == linattn.LINATTN_ERR_INVALID
    assert g(KV=MIS) == linattn.LINATTN_ERR_INVALID
    assert g(eps=-2.0) == linattn.LINATTN_ERR_INVALID
    assert g(d=D(dk=12)) == linattn.LINATTN_ERR_UNSUPPORTED
    assert g(out=FAKE2) == linattn.LINATTN_ERR_INVALID
    assert g(KV=FAKE4) == linattn.LINATTN_ERR_INVALID


def test_decode_rejects_bad_arguments(lib):
    d = D()
    S, z = P(0x7F0000500000), P(0x7F0000600000)
    dec = lambda **kw: lib.linattn_decode_step(
        ctypes.byref(kw.get("d", d)), kw.get("q", FAKE), FAKE2, FAKE3, kw.get("lam", None),
        kw.get("eps", 1e-6), kw.get("S", S), kw.get("z", z), kw.get("out", FAKE4), None)
    assert dec(S=None) == linattn.LINATTN_ERR_INVALID
    assert dec(z=None) == linattn.LINATTN_ERR_INVALID
    assert dec(q=None) == linattn.LINATTN_ERR_INVALID
    assert dec(out=None) == linattn.LINATTN_ERR_INVALID
    assert dec(S=MIS) == linattn.LINATTN_ERR_INVALID
    assert dec(eps=float("nan")) == linattn.LINATTN_ERR_INVALID
    assert dec(d=D(dv=100)) == linattn.LINATTN_ERR_UNSUPPORTED
    assert dec(d=D(dtype=3)) == linattn.LINATTN_ERR_UNSUPPORTED
    assert dec(z=S) == linattn.LINATTN_ERR_INVALID          # state buffers overlap
    assert dec(out=S) == linattn.LINATTN_ERR_INVALID


def test_python_binding_checks_shapes():
    import torch
    q = torch.zeros(1, 2, 4, 64)
    with pytest.raises(ValueError):
        linattn.linattn_fwd_causal(q, q, torch.zeros(1, 2, 5, 64), None, 1e-6, q)


def test_phi_field_is_checked(lib):
    d = D()
    d.phi = 2
    assert causal(lib, d) == linattn.LINATTN_ERR_UNSUPPORTED
    d.phi = -1
    assert causal(lib, d) == linattn.LINATTN_ERR_UNSUPPORTED
    # identity features still go through the other checks
    d = D(dk=48)
    d.phi = linattn.LINATTN_PHI_IDENTITY
    assert causal(lib, d) == linattn.LINATTN_ERR_UNSUPPORTED
    assert ctypes.sizeof(linattn.linattn_dims) == 7 * 4


def feats(lib, rows=16, d=64, m=32, kernel=0, dtype=0, x=FAKE, w=FAKE2, out=FAKE3):
    return lib.linattn_performer_features(rows, d, m, kernel, dtype, x, w, out, None)


def test_performer_features_rejects_bad_arguments(lib):
    E_INV, E_UNS = linattn.LINATTN_ERR_INVALID, linattn.LINATTN_ERR_UNSUPPORTED
    assert feats(lib, rows=-1) == E_INV
    assert feats(lib, d=48) == E_UNS
    assert feats(lib, d=256) == E_UNS
    assert feats(lib, m=128) == E_UNS          # 2m would exceed the attention's dk
    assert feats(lib, m=12) == E_UNS
    assert feats(lib, kernel=2) == E_UNS
    assert feats(lib, dtype=5) == E_UNS
    assert feats(lib, rows=1 << 25, d=128) == E_UNS
    assert feats(lib, x=None) == E_INV
    assert feats(lib, w=None) == E_INV
    assert feats(lib, out=None) == E_INV
    assert feats(lib, x=MIS) == E_INV
    assert feats(lib, out=MIS) == E_INV
    # out overlapping x or omega
    assert feats(lib, out=P(FAKE.value + 64)) == E_INV
    assert feats(lib, out=P(FAKE2.value - 64)) == E_INV


def test_performer_features_zero_rows_is_a_no_op(lib):
    assert feats(lib, rows=0, x=None, w=None, out=None) == linattn.LINATTN_OK


def test_python_binding_checks_performer_shapes():
    import torch
    x = torch.zeros(3, 64, dtype=torch.bfloat16)
    w = torch.zeros(32, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):      # omega's d differs from x's
        linattn.linattn_performer_features(x, torch.zeros(32, 16, dtype=torch.bfloat16), 0,
                                           torch.zeros(3, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):      # out must hold 2m features per row
        linattn.linattn_performer_features(x, w, 0, torch.zeros(3, 32, dtype=torch.bfloat16))
    with pytest.raises(ValueError):      # one dtype for x, omega and out
        linattn.linattn_performer_features(x, w.float(), 0, torch.zeros(3, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):      # omega must be [m, d]
        linattn.linattn_performer_features(x, torch.zeros(2, 32, 64, dtype=torch.bfloat16), 0,
                                           torch.zeros(3, 64, dtype=torch.bfloat16))


def test_python_binding_passes_phi_into_the_dims():
    import torch
    captured = {}

    class FakeLib:
        def linattn_fwd_causal(self, d, *args):
            captured["phi"] = d._obj.phi
            captured["dtype"] = d._obj.dtype
            return linattn.LINATTN_OK

    real = linattn._lib
    try:
        linattn._lib = FakeLib()
        # tensors on the CPU never reach a kernel: the fake library records the dims
        orig_ptr = linattn._ptr
        linattn._ptr = lambda t: None
        try:
            q = torch.zeros(1, 2, 4, 64, dtype=torch.bfloat16)
            linattn.linattn_fwd_causal(q, q, q, None, 1e-6, q, stream=0,
                                       phi=linattn.LINATTN_PHI_IDENTITY)
            assert captured == {"phi": 1, "dtype": linattn.LINATTN_BF16}
            linattn.linattn_fwd_causal(q, q, q, None, 1e-6, q, stream=0)
            assert captured["phi"] == linattn.LINATTN_PHI_ELU1
        finally:
            linattn._ptr = orig_ptr
    finally:
        linattn._lib = real
