"""Test-only fp64 restatement of the chunkwise (WY / UT-transform) form.

Used by the oracle self-tests to show, in exact-ish fp64 arithmetic, that the
chunked form the CUDA kernels use produces the same numbers as the token
recurrence ("chunkwise execution changes cost, never the numbers": Kimi Delta
Attention: a bounded case study, Exercise 2; affine chunk transfer and write
summary: Semidirect Fourier Delta Attention §1 contribution 4, §2.2
eq. (9)-(10)). It is not the oracle and not the CUDA path; it imports neither.

Derivation (positions i, j in 1..L inside one chunk; S = chunk-entry state;
G_{i<-j} = prod_{s=j+1..i} diag(alpha_s); gamma_i = G_{i<-0};
sigma_j = G_{L<-j}): with u_i = beta_i (v_i - (D_i S_{i-1})^T k_i) the token
step is S_i = D_i S_{i-1} + k_i u_i^T, and unrolling gives
    (I + A) U = diag(beta) (V - Khat S),  A_ij = beta_i k_i^T G_{i<-j} k_j (j<i)
    O   = Qhat S + M U,                   M_ij = q_i^T G_{i<-j} k_j (j<=i)
    S_L = diag(gamma_L) S + Kbar^T U,
with Khat_i = gamma_i * k_i, Qhat_i = gamma_i * q_i, Kbar_j = sigma_j * k_j.
Gate factors are plain products (no division), so zero and negative gates
need nothing special.
"""
from __future__ import annotations

import numpy as np


def pair_gates(alpha: np.ndarray) -> np.ndarray:
    """G[i, j, :] = prod_{s=j+1..i} alpha[s] for j <= i (0 above the diagonal)."""
    L, d = alpha.shape
    dt = np.result_type(alpha, 1.0)            # real gates, or complex ones
    G = np.zeros((L, L, d), dtype=dt)
    for j in range(L):
        g = np.ones(d, dtype=dt)
        G[j, j] = g
        for i in range(j + 1, L):
            g = g * alpha[i]
            G[i, j] = g
    return G


def chunk_step(S, q, k, v, alpha, beta, scale=1.0, return_T=False):
    """One chunk of L tokens from entry state S [d_k, d_v]; returns (O, S_L)."""
    L = q.shape[0]
    G = pair_gates(alpha)
    A = np.zeros((L, L))
    M = np.zeros((L, L))
    for i in range(L):
        for j in range(i + 1):
            gk = G[i, j] * k[j]
            M[i, j] = q[i] @ gk
            if j < i:
                A[i, j] = beta[i] * (k[i] @ gk)
    gamma = np.cumprod(alpha, axis=0)                 # gamma_i = G_{i<-0}
    sigma = np.stack([G[L - 1, j] for j in range(L)])  # sigma_j = G_{L<-j}
    T = np.linalg.inv(np.eye(L) + A)
    Khat = gamma * k
    Qhat = gamma * q
    Kbar = sigma * k
    W = T @ (beta[:, None] * Khat)
    Ut = T @ (beta[:, None] * v)
    U = Ut - W @ S
    O = scale * (Qhat @ S + M @ U)
    S_new = gamma[L - 1][:, None] * S + Kbar.T @ U
    if return_T:
        return O, S_new, T
    return O, S_new


def chunked_fwd(q, k, v, alpha, beta, S0, C, scale=1.0):
    """Whole sequence [T, d] for one head, in chunks of C tokens."""
    T = q.shape[0]
    S = np.array(S0, dtype=np.float64, copy=True)
    o = np.zeros((T, v.shape[1]))
    for s in range(0, T, C):
        e = min(T, s + C)
        o[s:e], S = chunk_step(S, q[s:e], k[s:e], v[s:e], alpha[s:e],
                               beta[s:e], scale)
    return o, S


def chunk_step_complex(S, q, k, v, lam, beta, scale=1.0):
    """One chunk of the complex-phase gate ("Semidirect Fourier Delta
    Attention" §3, eqs. (13)-(14)): S' = Lambda S with complex diagonal
    gates lam = alpha exp(i theta), S_i = S'_i + k_i u_i^T with
    u_i^T = beta_i (v_i^* - k_i^* S'_i), and o_i = scale S_i^* q_i. The same
    unrolling as the real case, with conjugates where k^* and q^* stand:
        (I + A) U = diag(beta) (conj(V) - Khat S),  A_ij = beta_i k_i^* G_ij k_j (j < i)
        conj(O)   = scale (Qhat S + M U),           M_ij = q_i^* G_ij k_j (j <= i)
        S_L       = diag(gamma_L) S + Kbar^T U,
    with Khat_i = gamma_i conj(k_i), Qhat_i = gamma_i conj(q_i),
    Kbar_j = sigma_j k_j. Returns (O, S_L)."""
    L = q.shape[0]
    G = pair_gates(lam)
    A = np.zeros((L, L), dtype=complex)
    M = np.zeros((L, L), dtype=complex)
    for i in range(L):
        for j in range(i + 1):
            gk = G[i, j] * k[j]
            M[i, j] = q[i].conj() @ gk
            if j < i:
                A[i, j] = beta[i] * (k[i].conj() @ gk)
    gamma = np.cumprod(lam, axis=0)
    sigma = np.stack([G[L - 1, j] for j in range(L)])
    T = np.linalg.inv(np.eye(L) + A)
    U = T @ (beta[:, None] * (v.conj() - (gamma * k.conj()) @ S))
    O = scale * ((gamma * q.conj()) @ S + M @ U).conj()
    S_new = gamma[L - 1][:, None] * S + (sigma * k).T @ U
    return O, S_new
