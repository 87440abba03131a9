"""CKDA oracle: a plain fp64 CPU implementation of the recurrence.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package. The CUDA library never
imports, links or calls it, and this package imports nothing from the CUDA
library: the two share only the seeded input generators, which hold none of
the method's arithmetic.

The arithmetic lives in ``ckda_oracle.c`` (one token at a time, fp64, the
recurrence of "Semidirect Fourier Delta Attention" §1 eq. (1) / §2.2 eq. (9)
with the readout of §3 eq. (14); ranges from "Complex KDA", abstract). This
module only compiles it with gcc (no fast-math) and marshals numpy arrays.

Every function here is pinned by ``tests/test_oracle_pins.py``,
``tests/test_oracle_prologue.py``, ``tests/test_oracle_bwd.py`` and
``tests/test_oracle_complex.py`` against
the lesson's worked traces, closed forms, the dense affine composition
(§2.2 eq. (10)) and, for the backward pass, central finite differences of
the forward; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ckda_oracle.c")
_LIB = os.path.join(_HERE, "libckda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ckda_oracle.c into libckda_oracle.so (gcc -O2 -fopenmp, IEEE fp64)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    """Load a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int32)
    lp = ctypes.POINTER(ctypes.c_int64)
    i32 = ctypes.c_int32
    lib.ckda_oracle_fwd.restype = ctypes.c_int
    lib.ckda_oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, ip,
                                    i32, i32, i32, i32, ctypes.c_double, i32]
    lib.ckda_oracle_decode.restype = ctypes.c_int
    lib.ckda_oracle_decode.argtypes = [dp, dp, dp, dp, dp, dp, dp,
                                       i32, i32, i32, i32, ctypes.c_double,
                                       lp, ctypes.c_int64, i32]
    lib.ckda_oracle_max_threads.restype = ctypes.c_int
    return lib


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (CPU); upcast exactly
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a, ty=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ty))


def max_threads() -> int:
    return int(_load().ckda_oracle_max_threads())


def fwd(q, k, v, alpha, beta, initial_state=None, cu_seqlens=None,
        scale: float = 1.0, nthreads: int = 0, lib=None):
    """Token-by-token fp64 forward.

    q, k: [total_T, H, d_k]; v: [total_T, H, d_v]; alpha: [total_T, H, d_k];
    beta: [total_T, H]; initial_state: [N, H, d_k, d_v] or None (zero);
    cu_seqlens: [N+1] int (None = one sequence of total_T tokens).
    Returns (o [total_T, H, d_v], final_state [N, H, d_k, d_v]) in fp64.
    ``lib`` selects another compiled copy of the oracle (the mutation tests
    load deliberately broken copies to show the pins catch them).
    """
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    s0 = _f64(initial_state)
    T, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int32)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    N = cu.shape[0] - 1
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal total_T")
    if s0 is not None and s0.shape != (N, H, dk, dv):
        raise ValueError("initial_state shape mismatch")
    o = np.zeros((T, H, dv), dtype=np.float64)
    sf = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load(lib).ckda_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                 _ptr(beta), _ptr(s0), _ptr(sf), _ptr(o),
                                 _ptr(cu, ctypes.c_int32), N, H, dk, dv,
                                 float(scale), int(nthreads))
    if rc != 0:
        raise RuntimeError("ckda_oracle_fwd failed (%d)" % rc)
    return o, sf


def decode(q, k, v, alpha, beta, state, scale: float = 1.0, pairs=None,
           nthreads: int = 0, lib=None):
    """One fp64 decode step, in place on ``state`` (an fp64 numpy array).

    q, k: [N, H, d_k]; v: [N, H, d_v]; alpha: [N, H, d_k]; beta: [N, H];
    state: [N, H, d_k, d_v] float64, C-contiguous, updated in place.
    pairs: optional int64 array of flattened (n*H + h) indices to step; the
    other pairs' state and output are left untouched (output rows zero).
    Returns o [N, H, d_v] (fp64).
    """
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64
            and state.flags.c_contiguous):
        raise TypeError("state must be a C-contiguous float64 numpy array")
    N, H, dk = q.shape
    dv = v.shape[2]
    if state.shape != (N, H, dk, dv):
        raise ValueError("state shape mismatch")
    o = np.zeros((N, H, dv), dtype=np.float64)
    pp = None
    npairs = 0
    if pairs is not None:
        pp = np.ascontiguousarray(pairs, dtype=np.int64)
        npairs = pp.shape[0]
    rc = _load(lib).ckda_oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                    _ptr(beta), _ptr(state), _ptr(o), N, H, dk,
                                    dv, float(scale),
                                    _ptr(pp, ctypes.c_int64), npairs,
                                    int(nthreads))
    if rc != 0:
        raise RuntimeError("ckda_oracle_decode failed (%d)" % rc)
    return o


def sigmoid(x):
    """1 / (1 + exp(-x)) in fp64, without overflow for large |x|."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def gate_prologue(a_logit, c_logit, k_raw, alpha_min: float, alpha_max: float,
                  beta_max: float, k_eps: float):
    """The fused input prologue in fp64, the stable parameterisation of
    "Semidirect Fourier Delta Attention" §3, eqs. (15), (17), (18):

        alpha = alpha_min + (alpha_max - alpha_min) * sigmoid(a)   per channel
        beta  = beta_max * sigmoid(c)                              per token
        k     = k_raw / (||k_raw||_2 + k_eps)                      per token

    with k = 0 where ||k_raw|| + k_eps is 0. Returns (alpha, beta, k)."""
    a, c, kr = _f64(a_logit), _f64(c_logit), _f64(k_raw)
    alpha = alpha_min + (alpha_max - alpha_min) * sigmoid(a)
    beta = beta_max * sigmoid(c)
    den = np.sqrt((kr * kr).sum(axis=-1, keepdims=True)) + k_eps
    k = np.where(den > 0, kr / np.where(den > 0, den, 1.0), 0.0)
    return alpha, beta, k


def fwd_gated(q, k_raw, v, a_logit, c_logit, gates: dict, initial_state=None,
              cu_seqlens=None, scale: float = 1.0):
    """The forward with the fused input prologue: gate_prologue, then fwd."""
    alpha, beta, k = gate_prologue(a_logit, c_logit, k_raw, **gates)
    return fwd(q, k, v, alpha, beta, initial_state, cu_seqlens, scale)


def decode_gated(q, k_raw, v, a_logit, c_logit, state, gates: dict,
                 scale: float = 1.0, pairs=None):
    """One decode step with the fused input prologue: gate_prologue, then
    decode (state updated in place)."""
    alpha, beta, k = gate_prologue(a_logit, c_logit, k_raw, **gates)
    return decode(q, k, v, alpha, beta, state, scale, pairs)


def _bwd_head(q, k, v, alpha, beta, do, s0, g_final, scale):
    """Reverse-mode gradients of one (sequence, head) token recurrence, fp64.

    Forward step (state S_prev before token t):
        S' = diag(alpha_t) S_prev,  w = v_t - S'^T k_t,  S_t = S' + beta_t k_t w^T,
        o_t = scale S_t^T q_t.
    Backward step, G = dL/dS_t coming from the later tokens:
        G += scale q_t do_t^T;  dq_t = scale S_t do_t;  g = G^T k_t;
        dv_t = beta_t g;  dbeta_t = g . w;  dk_t = beta_t (G w - S' g);
        dS' = G - beta_t k_t g^T;  dalpha_t = rowsum(dS' * S_prev);
        G <- diag(alpha_t) dS'  (= dL/dS_prev).
    """
    L = q.shape[0]
    S = s0.copy()
    prev, ws = [], []
    for t in range(L):
        prev.append(S)
        Sp = alpha[t][:, None] * S
        w = v[t] - Sp.T @ k[t]
        S = Sp + beta[t] * np.outer(k[t], w)
        ws.append(w)
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    dal = np.zeros_like(alpha); dbe = np.zeros_like(beta)
    G = g_final.copy()
    for t in range(L - 1, -1, -1):
        S_prev, w = prev[t], ws[t]
        Sp = alpha[t][:, None] * S_prev
        St = Sp + beta[t] * np.outer(k[t], w)
        G = G + scale * np.outer(q[t], do[t])
        dq[t] = scale * (St @ do[t])
        g = G.T @ k[t]
        dv[t] = beta[t] * g
        dbe[t] = g @ w
        dk[t] = beta[t] * (G @ w - Sp @ g)
        dSp = G - beta[t] * np.outer(k[t], g)
        dal[t] = (dSp * S_prev).sum(axis=1)
        G = alpha[t][:, None] * dSp
    return dq, dk, dv, dal, dbe, G


def bwd(q, k, v, alpha, beta, d_o, initial_state=None, d_final_state=None,
        cu_seqlens=None, scale: float = 1.0, _head=None):
    """Gradients of the forward (``fwd``) for a loss L with dL/do = d_o and
    dL/d(final state) = d_final_state (None = 0), in fp64.

    The pages state the forward recurrence only ("Semidirect Fourier Delta
    Attention" §1 eq. (1), §3 eq. (14)); the backward here is its adjoint,
    one token at a time in reverse (``_bwd_head``). Shapes as ``fwd``; d_o
    is [total_T, H, d_v]. Returns (dq, dk, dv, dalpha, dbeta,
    d_initial_state), the last [N, H, d_k, d_v]. ``_head`` replaces the
    per-head routine (the mutation tests pass deliberately broken copies).
    """
    q, k, v, alpha, beta, d_o = map(_f64, (q, k, v, alpha, beta, d_o))
    s0 = _f64(initial_state)
    gf = _f64(d_final_state)
    T, H, dk_ = q.shape
    dv_ = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.asarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal total_T")
    head = _head or _bwd_head
    out = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v),
           np.zeros_like(alpha), np.zeros_like(beta),
           np.zeros((N, H, dk_, dv_), dtype=np.float64)]
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            st0 = s0[n, h] if s0 is not None else np.zeros((dk_, dv_))
            g0 = gf[n, h] if gf is not None else np.zeros((dk_, dv_))
            r = head(q[a:b, h], k[a:b, h], v[a:b, h], alpha[a:b, h], beta[a:b, h],
                     d_o[a:b, h], st0, g0, float(scale))
            for i in range(5):
                out[i][a:b, h] = r[i]
            out[5][n, h] = r[5]
    return tuple(out)


def fwd_complex(q, k, v, alpha, theta, beta, initial_state=None, cu_seqlens=None,
                scale: float = 1.0):
    """The complex-phase gate of "Semidirect Fourier Delta Attention" §3,
    eqs. (13)-(14), token by token in complex128:

        S_t = (I - beta_t k_t k_t^*) Lambda_t S_{t-1} + beta_t k_t v_t^*,
        Lambda_t = diag(alpha_t * exp(i theta_t)),   o_t = scale S_t^* q_t

    (^* the conjugate transpose). q, k: [total_T, H, d_k] complex; v:
    [total_T, H, d_v] complex; alpha, theta: [total_T, H, d_k] real; beta:
    [total_T, H] real; states [N, H, d_k, d_v] complex. With theta = 0 and
    real inputs this is ``fwd``. Returns (o, final_state) in complex128.
    """
    def c128(x):
        if x is None:
            return None
        if hasattr(x, "detach"):
            x = x.detach().to("cpu").numpy()
        return np.ascontiguousarray(x, dtype=np.complex128)

    q, k, v = c128(q), c128(k), c128(v)
    alpha, theta, beta = _f64(alpha), _f64(theta), _f64(beta)
    s0 = c128(initial_state)
    T, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.asarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    o = np.zeros((T, H, dv), dtype=np.complex128)
    sf = np.zeros((N, H, dk, dv), dtype=np.complex128)
    for n in range(N):
        for h in range(H):
            S = s0[n, h].copy() if s0 is not None else np.zeros((dk, dv), dtype=np.complex128)
            for t in range(int(cu[n]), int(cu[n + 1])):
                lam = alpha[t, h] * np.exp(1j * theta[t, h])
                S = lam[:, None] * S                                  # Lambda_t S_{t-1}
                kt = k[t, h]
                S = S - beta[t, h] * np.outer(kt, kt.conj() @ S)       # (I - beta k k^*) .
                S = S + beta[t, h] * np.outer(kt, v[t, h].conj())      # + beta k v^*
                o[t, h] = scale * (S.conj().T @ q[t, h])               # S^* q
            sf[n, h] = S
    return o, sf
