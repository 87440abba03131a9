"""Host-only checks of the C ABI: the library loads, exports every entry point
include/ckda.h declares, and rejects bad arguments before any launch.

No GPU: every call below fails host-side validation, so nothing is launched
and no device pointer is ever dereferenced (the fake pointers are never
reached by a kernel).
"""
import ctypes
import os
import re

import pytest

from gated_delta_rule_114_b200 import build as ckda_build
from gated_delta_rule_114_b200 import ckda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ckda.h")


@pytest.fixture(scope="module")
def lib():
    ckda_build.build()
    return ckda.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ckda_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("ckda_fwd_chunked", "ckda_decode_step", "ckda_status_string",
                 "ckda_last_error", "ckda_version"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(5):
        assert lib.ckda_status_string(s).decode().startswith("CKDA_")
    assert b"UNKNOWN" in lib.ckda_status_string(99)
    assert lib.ckda_version() >= 100


# fake, 16-byte aligned, never dereferenced: every call fails validation first
P = ctypes.c_void_p(0x10000)
P2 = ctypes.c_void_p(0x20000)
P3 = ctypes.c_void_p(0x30000)
P4 = ctypes.c_void_p(0x40000)
P5 = ctypes.c_void_p(0x50000)
P6 = ctypes.c_void_p(0x60000)
ODD = ctypes.c_void_p(0x10004)
NULL = None


def fwd(lib, q=P, k=P2, v=P3, a=P4, b=P5, s0=NULL, sf=NULL, o=P6, cu=NULL,
        cuh=NULL, N=1, T=8, H=1, dk=16, dv=16, chunk=0, dt=ckda.CKDA_F32,
        ws=NULL, wsb=0):
    return lib.ckda_fwd_chunked(q, k, v, a, b, s0, sf, o, cu, cuh, N, T, H, dk,
                                dv, chunk, 1.0, dt, ws, wsb, None)


def dec(lib, q=P, k=P2, v=P3, a=P4, b=P5, s=P6, o=ctypes.c_void_p(0x70000),
        N=1, H=1, dk=16, dv=16, dt=ckda.CKDA_F32):
    return lib.ckda_decode_step(q, k, v, a, b, s, o, N, H, dk, dv, 1.0, dt, None)


@pytest.mark.parametrize("kw,want", [
    (dict(q=NULL), ckda.CKDA_ERR_ARG),
    (dict(o=NULL), ckda.CKDA_ERR_ARG),
    (dict(b=NULL), ckda.CKDA_ERR_ARG),
    (dict(q=ODD), ckda.CKDA_ERR_ARG),
    (dict(H=0), ckda.CKDA_ERR_ARG),
    (dict(N=-1), ckda.CKDA_ERR_ARG),
    (dict(T=-5), ckda.CKDA_ERR_ARG),
    (dict(dk=48), ckda.CKDA_ERR_UNSUPPORTED),
    (dict(dv=256), ckda.CKDA_ERR_UNSUPPORTED),
    (dict(chunk=24), ckda.CKDA_ERR_UNSUPPORTED),
    (dict(dt=7), ckda.CKDA_ERR_UNSUPPORTED),
    # sequences or heads beyond a grid dimension
    (dict(N=65536), ckda.CKDA_ERR_UNSUPPORTED),
    (dict(H=65536), ckda.CKDA_ERR_UNSUPPORTED),
    # output aliasing an input
    (dict(o=P), ckda.CKDA_ERR_ARG),
    # host cu_seqlens without a device copy
    (dict(cuh=ctypes.cast((ctypes.c_int32 * 2)(0, 8), ctypes.c_void_p)),
     ckda.CKDA_ERR_ARG),
])
def test_fwd_rejects(lib, kw, want):
    assert fwd(lib, **kw) == want


def test_workspace_query(lib):
    # tensor-core path (bf16, d_k=128, chunk 64): one block per (slot, head)
    # plus a table of 8 bytes per slot (rounded up to 1 KB);
    # 1 sequence of 64 tokens: floor(64/64) + 1 = 2 chunk slots
    def table(slots):
        return (slots * 8 + 1023) // 1024 * 1024
    block = (ckda.ckda_fwd_workspace_bytes(1, 64, 2, 128, 128)
             - ckda.ckda_fwd_workspace_bytes(1, 64, 1, 128, 128)) // 2
    assert block > 0 and block % 1024 == 0
    assert ckda.ckda_fwd_workspace_bytes(1, 64, 1, 128, 128) == 2 * block + table(2)
    slots = 2 * 8192 // 64 + 2
    assert ckda.ckda_fwd_workspace_bytes(2, 8192, 32, 128, 128) == slots * 32 * block + table(slots)
    assert ckda.ckda_fwd_workspace_bytes(1, 100, 1, 128, 128, varlen=True) == 2 * block + table(2)
    assert ckda.ckda_fwd_workspace_bytes(1, 64, 1, 128, 32) < 2 * block
    # CUDA-core path and unsupported arguments need none
    assert ckda.ckda_fwd_workspace_bytes(1, 64, 1, 64, 64) == 0
    assert ckda.ckda_fwd_workspace_bytes(1, 64, 1, 128, 128, dtype=__import__("torch").float32) == 0
    assert ckda.ckda_fwd_workspace_bytes(0, 64, 1, 128, 128) == 0


def test_fwd_rejects_missing_workspace(lib):
    # bf16, d=128, chunk 64 needs scratch: none given -> argument error
    st = fwd(lib, dk=128, dv=128, dt=ckda.CKDA_BF16, T=64)
    assert st == ckda.CKDA_ERR_ARG
    st = fwd(lib, dk=128, dv=128, dt=ckda.CKDA_BF16, T=64,
             ws=ctypes.c_void_p(0x1000000), wsb=16)
    assert st == ckda.CKDA_ERR_ARG


@pytest.mark.parametrize("cu_host", [(1, 8), (0, 9), (0, 5, 3, 8)])
def test_fwd_rejects_bad_host_seqlens(lib, cu_host):
    arr = (ctypes.c_int32 * len(cu_host))(*cu_host)
    st = fwd(lib, cu=P, cuh=ctypes.cast(arr, ctypes.c_void_p),
             N=len(cu_host) - 1, T=8, q=P2, k=P3, v=P4, a=P5, b=P6,
             o=ctypes.c_void_p(0x70000))
    assert st == ckda.CKDA_ERR_ARG


@pytest.mark.parametrize("kw,want", [
    (dict(s=NULL), ckda.CKDA_ERR_ARG),
    (dict(o=P6), ckda.CKDA_ERR_ARG),  # o aliases the state
    (dict(a=ODD), ckda.CKDA_ERR_ARG),
    (dict(H=0), ckda.CKDA_ERR_ARG),
    (dict(N=-2), ckda.CKDA_ERR_ARG),
    (dict(dk=8), ckda.CKDA_ERR_UNSUPPORTED),
    (dict(dt=3), ckda.CKDA_ERR_UNSUPPORTED),
])
def test_decode_rejects(lib, kw, want):
    assert dec(lib, **kw) == want


def test_python_binding_requires_cuda_tensors(lib):
    import torch
    x = torch.zeros(4, 1, 16)
    with pytest.raises(ValueError):
        ckda.ckda_fwd_chunked(x, x, x, x, torch.zeros(4, 1), None, None, x,
                              N=1, T=4)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(ckda, "_lib", None)
    with pytest.raises(RuntimeError):
        ckda.load(str(tmp_path / "nope.so"))


@pytest.mark.parametrize("gp,ok", [((-1.0, 1.0, 2.0, 0.0), True), ((0.0, 1.0, 1.0, 1e-6), True),
                                   ((-1.5, 1.0, 2.0, 0.0), False), ((0.0, 1.2, 1.0, 0.0), False),
                                   ((0.5, 0.2, 1.0, 0.0), False), ((0.0, 1.0, 2.5, 0.0), False),
                                   ((0.0, 1.0, -0.1, 0.0), False), ((0.0, 1.0, 1.0, -1.0), False),
                                   ((0.0, float("nan"), 1.0, 0.0), False),
                                   ((0.0, 1.0, float("inf"), 0.0), False)])
def test_gate_params_are_validated_first(lib, gp, ok):
    # d_k = 48 is unsupported: valid gate parameters reach that check
    # (CKDA_ERR_UNSUPPORTED), invalid ones are rejected before it (CKDA_ERR_ARG)
    g = ckda.GateParams(*gp)
    want = ckda.CKDA_ERR_UNSUPPORTED if ok else ckda.CKDA_ERR_ARG
    st = lib.ckda_fwd_chunked_gated(P, P2, P3, P4, P5, NULL, NULL, P6, NULL, NULL, 1, 8, 1,
                                    48, 16, 0, 1.0, ckda.CKDA_F32, g, NULL, 0, None)
    assert st == want
    st = lib.ckda_decode_step_gated(P, P2, P3, P4, P5, P6, ctypes.c_void_p(0x70000), 1, 1,
                                    48, 16, 1.0, ckda.CKDA_F32, g, None)
    assert st == want


def test_gated_forward_rejects_like_the_plain_one(lib):
    g = ckda.GateParams(-1.0, 1.0, 2.0, 1e-6)
    # missing logits, misaligned logits, output aliasing the raw keys
    assert lib.ckda_fwd_chunked_gated(P, P2, P3, NULL, P5, NULL, NULL, P6, NULL, NULL, 1, 8,
                                      1, 16, 16, 0, 1.0, ckda.CKDA_F32, g, NULL, 0,
                                      None) == ckda.CKDA_ERR_ARG
    assert lib.ckda_fwd_chunked_gated(P, P2, P3, ODD, P5, NULL, NULL, P6, NULL, NULL, 1, 8,
                                      1, 16, 16, 0, 1.0, ckda.CKDA_F32, g, NULL, 0,
                                      None) == ckda.CKDA_ERR_ARG
    assert lib.ckda_fwd_chunked_gated(P, P2, P3, P4, P5, NULL, NULL, P2, NULL, NULL, 1, 8,
                                      1, 16, 16, 0, 1.0, ckda.CKDA_F32, g, NULL, 0,
                                      None) == ckda.CKDA_ERR_ARG


def declared_arities():
    """Parameter count of every function include/ckda.h declares."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(ckda_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", src):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header(lib):
    """Every ctypes signature the binding declares has the header's arity."""
    ar = declared_arities()
    assert "ckda_bwd" in ar and "ckda_bwd_workspace_bytes" in ar and "ckda_bwd_chunked" in ar
    for name, n in ar.items():
        fn = getattr(lib, name)
        if fn.argtypes is not None:
            assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def bwd(lib, q=P, k=P2, v=P3, a=P4, b=P5, do=P6, dq=ctypes.c_void_p(0x70000),
        dk=ctypes.c_void_p(0x80000), dv=ctypes.c_void_p(0x90000),
        da=ctypes.c_void_p(0xA0000), db=ctypes.c_void_p(0xB0000), N=1, T=8, H=1, dkd=16,
        dvd=16, dt=ckda.CKDA_F32, ws=ctypes.c_void_p(0x100000), wsb=1 << 30, fn="ckda_bwd"):
    return getattr(lib, fn)(q, k, v, a, b, NULL, do, NULL, dq, dk, dv, da, db, NULL, NULL, NULL,
                            N, T, H, dkd, dvd, 1.0, dt, ws, wsb, None)


@pytest.mark.parametrize("kw,want", [
    (dict(q=NULL), ckda.CKDA_ERR_ARG),
    (dict(do=NULL), ckda.CKDA_ERR_ARG),
    (dict(db=NULL), ckda.CKDA_ERR_ARG),
    (dict(k=ODD), ckda.CKDA_ERR_ARG),
    (dict(H=0), ckda.CKDA_ERR_ARG),
    (dict(N=-1), ckda.CKDA_ERR_ARG),
    (dict(dkd=48), ckda.CKDA_ERR_UNSUPPORTED),
    (dict(dvd=256), ckda.CKDA_ERR_UNSUPPORTED),
    (dict(dt=7), ckda.CKDA_ERR_UNSUPPORTED),
    (dict(N=65536), ckda.CKDA_ERR_UNSUPPORTED),
    # a gradient aliasing an input, two gradients aliasing each other
    (dict(dq=P), ckda.CKDA_ERR_ARG),
    (dict(dk=ctypes.c_void_p(0x70000)), ckda.CKDA_ERR_ARG),
    # workspace missing or too small
    (dict(ws=NULL), ckda.CKDA_ERR_ARG),
    (dict(wsb=1024), ckda.CKDA_ERR_ARG),
])
@pytest.mark.parametrize("fn", ["ckda_bwd", "ckda_bwd_chunked"])
def test_bwd_rejects(lib, kw, want, fn):
    assert bwd(lib, fn=fn, **kw) == want


def test_bwd_workspace_query(lib):
    # checkpoints every 16 tokens: floor(T_total / 16) + N slots per head, plus
    # a 16-state buffer per (sequence, head); fp32 d_k x d_v states; plus the
    # fp32 partials of dq, dk, dalpha (d_k each) and dbeta per token-head for
    # each 32-column tile (d_v = 64: 2 tiles)
    st = 32 * 64 * 4
    part = lambda th: 2 * th * (3 * 32 + 1) * 4
    assert lib.ckda_bwd_workspace_bytes(2, 40, 3, 32, 64, 0) == \
        ((80 // 16 + 2) * 3 + 2 * 3 * 16) * st + part(80 * 3)
    assert lib.ckda_bwd_workspace_bytes(2, 40, 3, 32, 64, 1) == \
        ((40 // 16 + 2) * 3 + 2 * 3 * 16) * st + part(40 * 3)
    assert lib.ckda_bwd_workspace_bytes(1, 8, 1, 48, 16, 0) == 0
    assert lib.ckda_bwd_workspace_bytes(0, 8, 1, 16, 16, 0) == 0


def test_bwd_chunked_workspace_query(lib):
    # per 16-token chunk slot (floor(T_total / 16) + N of them) and head: an
    # entry state and an exit-state gradient (d_k x d_v), gamma over the chunk
    # (d_k) and Abar (16 x 16); per token-head: W, Kbar, Wb, Qs, BK (d_k each)
    # and Utilde, X, U, dR (d_v each)
    def want(N, T_total, H, dk, dv):
        sl, th = (T_total // 16 + N) * H, T_total * H
        return 4 * (sl * (2 * dk * dv + dk + 256) + th * (5 * dk + 4 * dv))
    assert lib.ckda_bwd_chunked_workspace_bytes(2, 40, 3, 32, 64, 0) == want(2, 80, 3, 32, 64)
    assert lib.ckda_bwd_chunked_workspace_bytes(2, 40, 3, 32, 64, 1) == want(2, 40, 3, 32, 64)
    assert lib.ckda_bwd_chunked_workspace_bytes(1, 8, 1, 16, 16, 0) == want(1, 8, 1, 16, 16)
    assert lib.ckda_bwd_chunked_workspace_bytes(1, 8, 1, 48, 16, 0) == 0
    assert lib.ckda_bwd_chunked_workspace_bytes(0, 8, 1, 16, 16, 0) == 0


def test_bwd_zero_sequences_is_a_noop(lib):
    """N = 0: validated, nothing launched, CKDA_OK (the fake pointers are
    never dereferenced)."""
    assert bwd(lib, N=0, T=0, ws=NULL, wsb=0) == ckda.CKDA_OK
    assert bwd(lib, N=0, T=0, ws=NULL, wsb=0, fn="ckda_bwd_chunked") == ckda.CKDA_OK


def cplx(lib, q=P, k=P2, v=P3, a=P4, th=P5, b=P6, s0=NULL, sf=NULL,
         o=ctypes.c_void_p(0x70000), cu=NULL, cuh=NULL, N=1, T=8, H=1, dk=16, dv=16,
         chunked=False, ws=ctypes.c_void_p(0x100000), wsb=1 << 30):
    if chunked:
        return lib.ckda_fwd_complex_chunked(q, k, v, a, th, b, s0, sf, o, cu, cuh, N, T, H, dk,
                                            dv, 1.0, ws, wsb, None)
    return lib.ckda_fwd_complex(q, k, v, a, th, b, s0, sf, o, cu, cuh, N, T, H, dk, dv, 1.0,
                                None)


@pytest.mark.parametrize("kw,want", [
    (dict(q=NULL), ckda.CKDA_ERR_ARG),
    (dict(th=NULL), ckda.CKDA_ERR_ARG),
    (dict(v=ODD), ckda.CKDA_ERR_ARG),
    (dict(H=0), ckda.CKDA_ERR_ARG),
    (dict(T=-1), ckda.CKDA_ERR_ARG),
    (dict(dk=24), ckda.CKDA_ERR_UNSUPPORTED),
    (dict(N=65536), ckda.CKDA_ERR_UNSUPPORTED),
    # output over an input; final state over the output
    (dict(o=P3), ckda.CKDA_ERR_ARG),
    (dict(sf=ctypes.c_void_p(0x70000)), ckda.CKDA_ERR_ARG),
    # host cu_seqlens without a device copy
    (dict(cuh=ctypes.cast((ctypes.c_int32 * 2)(0, 8), ctypes.c_void_p)), ckda.CKDA_ERR_ARG),
])
@pytest.mark.parametrize("chunked", [False, True])
def test_complex_rejects(lib, kw, want, chunked):
    assert cplx(lib, chunked=chunked, **kw) == want


@pytest.mark.parametrize("kw", [dict(ws=NULL), dict(wsb=64), dict(ws=P)])
def test_complex_chunked_rejects_bad_workspace(lib, kw):
    """missing, too small, or over an input"""
    assert cplx(lib, chunked=True, **kw) == ckda.CKDA_ERR_ARG


def test_complex_chunked_workspace_query(lib):
    # complex64 (8 bytes): W, Kbar, Qhat per token-head (d_k each), Utilde (d_v);
    # per 16-token chunk slot and head: M (16 x 16) and gamma (d_k)
    def want(N, T_total, H, dk, dv):
        sl, th = (T_total // 16 + N) * H, T_total * H
        return 8 * (th * (3 * dk + dv) + sl * (256 + dk))
    q = lib.ckda_fwd_complex_chunked_workspace_bytes
    assert q(2, 40, 3, 32, 64, 0) == want(2, 80, 3, 32, 64)
    assert q(2, 40, 3, 32, 64, 1) == want(2, 40, 3, 32, 64)
    assert q(1, 8, 1, 24, 16, 0) == 0 and q(0, 8, 1, 16, 16, 0) == 0


@pytest.mark.parametrize("chunked", [False, True])
def test_complex_zero_sequences_is_a_noop(lib, chunked):
    assert cplx(lib, N=0, T=0, chunked=chunked, ws=NULL, wsb=0) == ckda.CKDA_OK
