"""Python binding of the CKDA C ABI (include/ckda.h).

Argument marshalling only: every step of the forward and the decode step runs
in the CUDA kernels of ``libckda.so``. PyTorch supplies device memory and
streams. There is no fallback of any kind: if the library cannot be loaded,
every call raises.

The functions named like the C entry points take caller-allocated tensors
(like the C ABI); ``fwd_chunked`` and ``decode_step`` are conveniences that
allocate the outputs with torch and then call the same entry points.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libckda.so")

CKDA_OK, CKDA_ERR_ARG, CKDA_ERR_UNSUPPORTED, CKDA_ERR_CUDA, CKDA_ERR_DEVICE = range(5)
CKDA_BF16, CKDA_F32 = 0, 1
_DT = {torch.bfloat16: CKDA_BF16, torch.float32: CKDA_F32}

_lib = None


class GateParams(ctypes.Structure):
    """ckda_gate_params (include/ckda.h): the fused input prologue's
    alpha = alpha_min + (alpha_max - alpha_min) sigmoid(a),
    beta = beta_max sigmoid(c), k = k_raw / (||k_raw|| + k_eps)."""
    _fields_ = [("alpha_min", ctypes.c_float), ("alpha_max", ctypes.c_float),
                ("beta_max", ctypes.c_float), ("k_eps", ctypes.c_float)]


CKDA_GATES = dict(alpha_min=-1.0, alpha_max=1.0, beta_max=2.0)  # CKDA ranges
KDA_GATES = dict(alpha_min=0.0, alpha_max=1.0, beta_max=1.0)    # KDA ranges


class CkdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.ckda_status_string(status).decode() if _lib else str(status)
        super().__init__("%s: %s" % (where, msg))


def load(path: str | None = None):
    """Load libckda.so (built in-tree by build.py). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(
            "libckda.so not found at %s: build it with "
            "`python -m gated_delta_rule_114_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    lib.ckda_fwd_chunked.restype = ctypes.c_int
    lib.ckda_fwd_chunked.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                     i32, i32, i32, i32, i32, i32, f32,
                                     ctypes.c_int, vp, ctypes.c_size_t, vp]
    lib.ckda_fwd_workspace_bytes.restype = ctypes.c_size_t
    lib.ckda_fwd_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32,
                                             ctypes.c_int]
    lib.ckda_fwd_chunked_noalloc.restype = ctypes.c_int
    lib.ckda_fwd_chunked_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                             i32, i32, i32, i32, i32, i32, f32,
                                             ctypes.c_int, vp]
    lib.ckda_decode_step.restype = ctypes.c_int
    lib.ckda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                     i32, f32, ctypes.c_int, vp]
    lib.ckda_fwd_chunked_gated.restype = ctypes.c_int
    lib.ckda_fwd_chunked_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                           i32, i32, i32, i32, i32, i32, f32,
                                           ctypes.c_int, GateParams, vp,
                                           ctypes.c_size_t, vp]
    lib.ckda_decode_step_gated.restype = ctypes.c_int
    lib.ckda_decode_step_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                           i32, f32, ctypes.c_int, GateParams, vp]
    lib.ckda_status_string.restype = ctypes.c_char_p
    lib.ckda_status_string.argtypes = [ctypes.c_int]
    lib.ckda_bwd.restype = ctypes.c_int
    lib.ckda_bwd.argtypes = [vp] * 16 + [i32] * 5 + [f32, ctypes.c_int, vp, ctypes.c_size_t, vp]
    lib.ckda_bwd_chunked.restype = ctypes.c_int
    lib.ckda_bwd_chunked.argtypes = lib.ckda_bwd.argtypes
    lib.ckda_fwd_complex.restype = ctypes.c_int
    lib.ckda_fwd_complex.argtypes = [vp] * 11 + [i32] * 5 + [f32, vp]
    lib.ckda_fwd_complex_chunked.restype = ctypes.c_int
    lib.ckda_fwd_complex_chunked.argtypes = [vp] * 11 + [i32] * 5 + [f32, vp, ctypes.c_size_t,
                                                                     vp]
    lib.ckda_fwd_complex_chunked_workspace_bytes.restype = ctypes.c_size_t
    lib.ckda_fwd_complex_chunked_workspace_bytes.argtypes = [i32] * 6
    lib.ckda_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.ckda_bwd_workspace_bytes.argtypes = [i32] * 6
    lib.ckda_bwd_chunked_workspace_bytes.restype = ctypes.c_size_t
    lib.ckda_bwd_chunked_workspace_bytes.argtypes = [i32] * 6
    lib.ckda_last_error.restype = ctypes.c_int
    lib.ckda_last_error.argtypes = [vp]
    lib.ckda_version.restype = ctypes.c_int32
    lib.ckda_version.argtypes = []
    _lib = lib
    return lib


def _p(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, where: str):
    if status != CKDA_OK:
        raise CkdaError(status, where)


def _need(t, name, dtype=None, dims=None):
    if t is None:
        raise ValueError("%s is required" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s" % (name, dtype))
    if dims is not None and t.dim() != dims:
        raise ValueError("%s must have %d dims" % (name, dims))


def ckda_fwd_workspace_bytes(N, T, H, d_k, d_v, chunk=0, varlen=False,
                             dtype=torch.bfloat16) -> int:
    """Scratch bytes ckda_fwd_chunked needs (see include/ckda.h)."""
    return int(load().ckda_fwd_workspace_bytes(int(N), int(T), int(H), int(d_k),
                                               int(d_v), int(chunk), int(bool(varlen)),
                                               _DT[dtype]))


def ckda_fwd_chunked(q, k, v, alpha, beta, initial_state, final_state, o,
                     cu_seqlens=None, cu_seqlens_host=None, N=None, T=None,
                     chunk: int = 0, scale: float = 1.0, stream=None,
                     workspace=None):
    """Marshal tensors into ckda_fwd_chunked (see include/ckda.h).

    q, k [T_total, H, d_k]; v, o [T_total, H, d_v] (bf16 or fp32, one dtype);
    alpha [T_total, H, d_k] fp32; beta [T_total, H] fp32; states
    [N, H, d_k, d_v] fp32 or None. With cu_seqlens (int32 CUDA [N+1]) the
    sequences are packed; otherwise give N and T (N sequences of T tokens).
    cu_seqlens_host: optional CPU int32 copy, validated by the library.
    workspace: optional uint8 CUDA tensor of at least ckda_fwd_workspace_bytes
    bytes; allocated with torch here when it is needed and not given.
    """
    _fwd_call(q, k, v, alpha, beta, initial_state, final_state, o, cu_seqlens,
              cu_seqlens_host, N, T, chunk, scale, stream, workspace, None)


def ckda_fwd_chunked_gated(q, k_raw, v, a_logit, c_logit, initial_state, final_state,
                           o, gates: GateParams, cu_seqlens=None, cu_seqlens_host=None,
                           N=None, T=None, chunk: int = 0, scale: float = 1.0,
                           stream=None, workspace=None):
    """Marshal tensors into ckda_fwd_chunked_gated (fused input prologue).

    As ckda_fwd_chunked with k_raw (unnormalised keys), a_logit
    [T_total, H, d_k] in q's dtype and c_logit [T_total, H] fp32 in place of
    k, alpha and beta; `gates` is a GateParams."""
    _fwd_call(q, k_raw, v, a_logit, c_logit, initial_state, final_state, o, cu_seqlens,
              cu_seqlens_host, N, T, chunk, scale, stream, workspace, gates)


def _fwd_call(q, k, v, alpha, beta, initial_state, final_state, o, cu_seqlens,
              cu_seqlens_host, N, T, chunk, scale, stream, workspace, gates):
    lib = load()
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, nme, q.dtype, 3)
    _need(alpha, "a_logit" if gates is not None else "alpha",
          q.dtype if gates is not None else torch.float32, 3)
    _need(beta, "c_logit" if gates is not None else "beta", torch.float32, 2)
    if q.dtype not in _DT:
        raise ValueError("q, k, v, o must be bfloat16 or float32")
    T_total, H, d_k = q.shape
    d_v = v.shape[2]
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        N = cu_seqlens.numel() - 1
        T = T_total
    elif N is None or T is None:
        raise ValueError("give cu_seqlens, or N and T")
    for t, nme in ((initial_state, "initial_state"), (final_state, "final_state")):
        if t is not None:
            _need(t, nme, torch.float32, 4)
    host_ptr = None
    if cu_seqlens_host is not None:
        if cu_seqlens_host.is_cuda or cu_seqlens_host.dtype != torch.int32 \
                or not cu_seqlens_host.is_contiguous():
            raise ValueError("cu_seqlens_host must be a contiguous CPU int32 tensor")
        host_ptr = ctypes.c_void_p(cu_seqlens_host.data_ptr())
    need = ckda_fwd_workspace_bytes(N, T, H, d_k, d_v, chunk,
                                    cu_seqlens is not None, q.dtype)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(initial_state),
            _p(final_state), _p(o), _p(cu_seqlens), host_ptr, int(N), int(T), int(H),
            int(d_k), int(d_v), int(chunk), float(scale), _DT[q.dtype])
    if gates is None:
        st = lib.ckda_fwd_chunked(*args, _p(workspace), ws_bytes, _stream(stream))
        _check(st, "ckda_fwd_chunked")
    else:
        st = lib.ckda_fwd_chunked_gated(*args, gates, _p(workspace), ws_bytes,
                                        _stream(stream))
        _check(st, "ckda_fwd_chunked_gated")


def ckda_bwd_workspace_bytes(N, T, H, d_k, d_v, varlen=False, chunked=False) -> int:
    """Scratch bytes ckda_bwd (ckda_bwd_chunked when ``chunked``) needs
    (see include/ckda.h)."""
    fn = load().ckda_bwd_chunked_workspace_bytes if chunked else load().ckda_bwd_workspace_bytes
    return int(fn(int(N), int(T), int(H), int(d_k), int(d_v), int(bool(varlen))))


def ckda_bwd(q, k, v, alpha, beta, initial_state, d_o, d_final_state, dq, dk, dv,
             dalpha, dbeta, d_initial_state, cu_seqlens=None, cu_seqlens_host=None,
             N=None, T=None, scale: float = 1.0, stream=None, workspace=None,
             chunked: bool = False):
    """Marshal tensors into ckda_bwd, or ckda_bwd_chunked when ``chunked``
    (see include/ckda.h): gradients of ckda_fwd_chunked for dL/do = d_o and
    dL/d(final state) = d_final_state (None = zero). dq, dk [T_total, H, d_k]
    and dv [T_total, H, d_v] in q's dtype, dalpha [T_total, H, d_k] and dbeta
    [T_total, H] fp32 and d_initial_state [N, H, d_k, d_v] fp32 (or None) are
    written."""
    lib = load()
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (d_o, "d_o"), (dq, "dq"), (dk, "dk"),
                   (dv, "dv")):
        _need(t, nme, q.dtype, 3)
    _need(alpha, "alpha", torch.float32, 3)
    _need(dalpha, "dalpha", torch.float32, 3)
    _need(beta, "beta", torch.float32, 2)
    _need(dbeta, "dbeta", torch.float32, 2)
    if q.dtype not in _DT:
        raise ValueError("q, k, v must be bfloat16 or float32")
    T_total, H, d_k = q.shape
    d_v = v.shape[2]
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        N = cu_seqlens.numel() - 1
        T = T_total
    elif N is None or T is None:
        raise ValueError("give cu_seqlens, or N and T")
    for t, nme in ((initial_state, "initial_state"), (d_final_state, "d_final_state"),
                   (d_initial_state, "d_initial_state")):
        if t is not None:
            _need(t, nme, torch.float32, 4)
    host_ptr = None
    if cu_seqlens_host is not None:
        if cu_seqlens_host.is_cuda or cu_seqlens_host.dtype != torch.int32 \
                or not cu_seqlens_host.is_contiguous():
            raise ValueError("cu_seqlens_host must be a contiguous CPU int32 tensor")
        host_ptr = ctypes.c_void_p(cu_seqlens_host.data_ptr())
    need = ckda_bwd_workspace_bytes(N, T, H, d_k, d_v, cu_seqlens is not None, chunked)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = lib.ckda_bwd_chunked if chunked else lib.ckda_bwd
    st = fn(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(initial_state), _p(d_o),
            _p(d_final_state), _p(dq), _p(dk), _p(dv), _p(dalpha), _p(dbeta),
            _p(d_initial_state), _p(cu_seqlens), host_ptr, int(N), int(T), int(H), int(d_k),
            int(d_v), float(scale), _DT[q.dtype], _p(workspace), ws_bytes, _stream(stream))
    _check(st, "ckda_bwd_chunked" if chunked else "ckda_bwd")


NOALLOC_SCRATCH_BYTES = 64 << 20  # CKDA_NOALLOC_SCRATCH_BYTES in include/ckda.h


def ckda_fwd_chunked_noalloc(q, k, v, alpha, beta, initial_state, final_state,
                             o, cu_seqlens=None, cu_seqlens_host=None, N=None,
                             T=None, chunk: int = 0, scale: float = 1.0,
                             stream=None):
    """Marshal tensors into ckda_fwd_chunked_noalloc (see include/ckda.h).

    For callers that cannot provide device scratch: the library uses its own
    fixed array of NOALLOC_SCRATCH_BYTES per device, shared by all calls, so
    calls must not overlap on the GPU. Arguments as in ckda_fwd_chunked.
    Nothing is allocated here either.
    """
    lib = load()
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, nme, q.dtype, 3)
    _need(alpha, "alpha", torch.float32, 3)
    _need(beta, "beta", torch.float32, 2)
    if q.dtype not in _DT:
        raise ValueError("q, k, v, o must be bfloat16 or float32")
    T_total, H, d_k = q.shape
    d_v = v.shape[2]
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        N = cu_seqlens.numel() - 1
        T = T_total
    elif N is None or T is None:
        raise ValueError("give cu_seqlens, or N and T")
    for t, nme in ((initial_state, "initial_state"), (final_state, "final_state")):
        if t is not None:
            _need(t, nme, torch.float32, 4)
    host_ptr = None
    if cu_seqlens_host is not None:
        if cu_seqlens_host.is_cuda or cu_seqlens_host.dtype != torch.int32 \
                or not cu_seqlens_host.is_contiguous():
            raise ValueError("cu_seqlens_host must be a contiguous CPU int32 tensor")
        host_ptr = ctypes.c_void_p(cu_seqlens_host.data_ptr())
    st = lib.ckda_fwd_chunked_noalloc(_p(q), _p(k), _p(v), _p(alpha), _p(beta),
                                      _p(initial_state), _p(final_state), _p(o),
                                      _p(cu_seqlens), host_ptr, int(N), int(T),
                                      int(H), int(d_k), int(d_v), int(chunk),
                                      float(scale), _DT[q.dtype], _stream(stream))
    _check(st, "ckda_fwd_chunked_noalloc")


def ckda_decode_step(q, k, v, alpha, beta, state, o, scale: float = 1.0,
                     stream=None):
    """Marshal tensors into ckda_decode_step (state updated in place).

    q, k [N, H, d_k]; v, o [N, H, d_v] (bf16 or fp32); alpha [N, H, d_k] fp32;
    beta [N, H] fp32; state [N, H, d_k, d_v] fp32.
    """
    _decode_call(q, k, v, alpha, beta, state, o, scale, stream, None)


def ckda_decode_step_gated(q, k_raw, v, a_logit, c_logit, state, o, gates: GateParams,
                           scale: float = 1.0, stream=None):
    """Marshal tensors into ckda_decode_step_gated (fused input prologue):
    k_raw [N, H, d_k], a_logit [N, H, d_k] in q's dtype, c_logit [N, H] fp32."""
    _decode_call(q, k_raw, v, a_logit, c_logit, state, o, scale, stream, gates)


def _decode_call(q, k, v, alpha, beta, state, o, scale, stream, gates):
    lib = load()
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, nme, q.dtype, 3)
    _need(alpha, "a_logit" if gates is not None else "alpha",
          q.dtype if gates is not None else torch.float32, 3)
    _need(beta, "c_logit" if gates is not None else "beta", torch.float32, 2)
    _need(state, "state", torch.float32, 4)
    if q.dtype not in _DT:
        raise ValueError("q, k, v, o must be bfloat16 or float32")
    N, H, d_k = q.shape
    d_v = v.shape[2]
    args = (_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(state), _p(o), int(N), int(H),
            int(d_k), int(d_v), float(scale), _DT[q.dtype])
    if gates is None:
        _check(lib.ckda_decode_step(*args, _stream(stream)), "ckda_decode_step")
    else:
        _check(lib.ckda_decode_step_gated(*args, gates, _stream(stream)),
               "ckda_decode_step_gated")


def ckda_last_error(stream=None) -> int:
    """Synchronise the stream; return and clear the device error status."""
    return int(load().ckda_last_error(_stream(stream)))


def version() -> int:
    return int(load().ckda_version())


def fwd_chunked(q, k, v, alpha, beta, initial_state=None, cu_seqlens=None,
                cu_seqlens_host=None, N=None, T=None, chunk: int = 0,
                scale: float = 1.0, output_final_state: bool = True,
                stream=None, workspace=None):
    """Allocate o (and the final state) with torch, then call ckda_fwd_chunked."""
    T_total, H, d_k = q.shape
    d_v = v.shape[2]
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
    elif N is None:
        N, T = 1, T_total
    o = torch.empty((T_total, H, d_v), dtype=q.dtype, device=q.device)
    sf = None
    if output_final_state:
        sf = torch.empty((N, H, d_k, d_v), dtype=torch.float32, device=q.device)
    ckda_fwd_chunked(q, k, v, alpha, beta, initial_state, sf, o, cu_seqlens,
                     cu_seqlens_host, N, T, chunk, scale, stream, workspace)
    return o, sf


def fwd_chunked_gated(q, k_raw, v, a_logit, c_logit, gates: GateParams,
                      initial_state=None, cu_seqlens=None, cu_seqlens_host=None,
                      N=None, T=None, chunk: int = 0, scale: float = 1.0,
                      stream=None, workspace=None):
    """Allocate o and the final state with torch, then call
    ckda_fwd_chunked_gated."""
    T_total, H, d_k = q.shape
    d_v = v.shape[2]
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
    elif N is None:
        N, T = 1, T_total
    o = torch.empty((T_total, H, d_v), dtype=q.dtype, device=q.device)
    sf = torch.empty((N, H, d_k, d_v), dtype=torch.float32, device=q.device)
    ckda_fwd_chunked_gated(q, k_raw, v, a_logit, c_logit, initial_state, sf, o, gates,
                           cu_seqlens, cu_seqlens_host, N, T, chunk, scale, stream,
                           workspace)
    return o, sf


def ckda_fwd_complex_chunked_workspace_bytes(N, T, H, d_k, d_v, varlen=False) -> int:
    """Scratch bytes ckda_fwd_complex_chunked needs (see include/ckda.h)."""
    return int(load().ckda_fwd_complex_chunked_workspace_bytes(
        int(N), int(T), int(H), int(d_k), int(d_v), int(bool(varlen))))


def ckda_fwd_complex(q, k, v, alpha, theta, beta, initial_state, final_state, o,
                     cu_seqlens=None, cu_seqlens_host=None, N=None, T=None,
                     scale: float = 1.0, stream=None, chunked: bool = False, workspace=None):
    """Marshal tensors into ckda_fwd_complex, or ckda_fwd_complex_chunked when
    ``chunked`` (see include/ckda.h): q, k [T_total, H, d_k] and v, o
    [T_total, H, d_v] complex64; alpha, theta [T_total, H, d_k] and beta
    [T_total, H] fp32; states [N, H, d_k, d_v] complex64 or None. The chunked
    call allocates its workspace with torch unless one is given."""
    lib = load()
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, nme, torch.complex64, 3)
    for t, nme in ((alpha, "alpha"), (theta, "theta")):
        _need(t, nme, torch.float32, 3)
    _need(beta, "beta", torch.float32, 2)
    T_total, H, d_k = q.shape
    d_v = v.shape[2]
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        N = cu_seqlens.numel() - 1
        T = T_total
    elif N is None or T is None:
        raise ValueError("give cu_seqlens, or N and T")
    for t, nme in ((initial_state, "initial_state"), (final_state, "final_state")):
        if t is not None:
            _need(t, nme, torch.complex64, 4)
    host_ptr = None
    if cu_seqlens_host is not None:
        if cu_seqlens_host.is_cuda or cu_seqlens_host.dtype != torch.int32 \
                or not cu_seqlens_host.is_contiguous():
            raise ValueError("cu_seqlens_host must be a contiguous CPU int32 tensor")
        host_ptr = ctypes.c_void_p(cu_seqlens_host.data_ptr())
    args = (_p(q), _p(k), _p(v), _p(alpha), _p(theta), _p(beta), _p(initial_state),
            _p(final_state), _p(o), _p(cu_seqlens), host_ptr, int(N), int(T), int(H), int(d_k),
            int(d_v), float(scale))
    if not chunked:
        _check(lib.ckda_fwd_complex(*args, _stream(stream)), "ckda_fwd_complex")
        return
    need = ckda_fwd_complex_chunked_workspace_bytes(N, T, H, d_k, d_v, cu_seqlens is not None)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ckda_fwd_complex_chunked(*args, _p(workspace), ws_bytes, _stream(stream)),
           "ckda_fwd_complex_chunked")


def fwd_complex(q, k, v, alpha, theta, beta, initial_state=None, cu_seqlens=None,
                cu_seqlens_host=None, N=None, T=None, scale: float = 1.0, stream=None,
                chunked: bool = False):
    """The complex-phase gate: allocate o and the final state (complex64) with
    torch, then call ckda_fwd_complex (ckda_fwd_complex_chunked when
    ``chunked``). Returns (o, final_state)."""
    T_total, H, d_k = q.shape
    d_v = v.shape[2]
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
    elif N is None:
        N, T = 1, T_total
    o = torch.empty((T_total, H, d_v), dtype=torch.complex64, device=q.device)
    sf = torch.empty((N, H, d_k, d_v), dtype=torch.complex64, device=q.device)
    ckda_fwd_complex(q, k, v, alpha, theta, beta, initial_state, sf, o, cu_seqlens,
                     cu_seqlens_host, N, T, scale, stream, chunked)
    return o, sf


def bwd(q, k, v, alpha, beta, d_o, initial_state=None, d_final_state=None,
        cu_seqlens=None, cu_seqlens_host=None, N=None, T=None, scale: float = 1.0,
        stream=None, workspace=None, chunked: bool = False):
    """Allocate the gradients with torch, then call ckda_bwd (ckda_bwd_chunked
    when ``chunked``). Returns (dq, dk, dv, dalpha, dbeta, d_initial_state)."""
    T_total, H, d_k = q.shape
    d_v = v.shape[2]
    if cu_seqlens is not None:
        N = cu_seqlens.numel() - 1
    elif N is None:
        N, T = 1, T_total
    dq, dk = torch.empty_like(q), torch.empty_like(k)
    dv = torch.empty_like(v)
    dalpha, dbeta = torch.empty_like(alpha), torch.empty_like(beta)
    ds0 = torch.empty((N, H, d_k, d_v), dtype=torch.float32, device=q.device)
    ckda_bwd(q, k, v, alpha, beta, initial_state, d_o, d_final_state, dq, dk, dv, dalpha,
             dbeta, ds0, cu_seqlens, cu_seqlens_host, N, T, scale, stream, workspace, chunked)
    return dq, dk, dv, dalpha, dbeta, ds0


def decode_step(q, k, v, alpha, beta, state, scale: float = 1.0, stream=None):
    """Allocate o with torch, then call ckda_decode_step (state in place)."""
    N, H, _ = q.shape
    o = torch.empty((N, H, v.shape[2]), dtype=q.dtype, device=q.device)
    ckda_decode_step(q, k, v, alpha, beta, state, o, scale, stream)
    return o
