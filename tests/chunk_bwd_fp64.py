"""Test-only fp64 restatement of a chunkwise backward pass.

The token-serial adjoint (the oracle's backward) visits every token three
times with a column sum over the state per step. This module states the same
gradients in the chunk form of the forward (``chunk_wy_fp64``), so that all
contractions over d_k or d_v are matrix products per chunk, and checks of it
against the oracle show that the chunk form loses nothing. It is not the
oracle and not the CUDA path; it imports neither.

Forward of one chunk (positions 1..L, entry state S; A = diag(beta) Abar):
    R = diag(beta) (V - Khat S),  U = T R,  T = (I + A)^-1
    O = scale (Qhat S + M U),     S_L = diag(gamma_L) S + Kbar^T U
("Semidirect Fourier Delta Attention" §2.2 eqs. (9)-(10); "Kimi Delta
Attention: a bounded case study", Exercise 2.)

Reverse of one chunk, given dO and dS_L (the gradient of the exit state):
    dU  = scale M^T dO + Kbar dS_L
    dR  = T^T dU                                  (= g_t, the adjoint of u_t)
    dS  = scale Qhat^T dO + diag(gamma_L) dS_L - Khat^T diag(beta) dR
    dV  = diag(beta) dR
    dbeta_i = dR_i . (V - Khat S - Abar U)_i      (= g_t . w_t of the token form)
    dM  = scale dO U^T (j <= i),  dAbar_ij = -beta_i dR_i . u_j (j < i)
    dQhat = scale dO S^T,  dKhat = -diag(beta) dR S^T,  dKbar = U dS_L^T
and dq, dk gather the gated Gram terms (every M_ij, Abar_ij is
sum_c x_ic G_{i<-j,c} k_jc). Only dS crosses chunks, so the reverse scan over
chunks carries one d_k x d_v matrix, as the forward does.

The gate gradient without division. Every alpha_{s,c} enters through a
product G_{i<-j,c} with j < s <= i, where j = 0 stands for the chunk entry
(gamma, the diag(gamma_L) S term) and i = L for the chunk exit (sigma). With
E_{ij,c} the coefficient of G_{i<-j,c} in the loss,
    dalpha_{s,c} = sum_{j < s <= i} E_{ij,c} G_{s-1<-j,c} G_{i<-s,c},
i.e. the product with the one factor alpha_s left out. Per channel it is
two running products (no division), so zero and negative gates need nothing
special, where the usual log-space form (alpha dalpha from cumulative sums,
then divide by alpha) fails at alpha = 0 and loses accuracy near it.
"""
from __future__ import annotations

import numpy as np

from chunk_wy_fp64 import pair_gates


def chunk_parts(q, k, v, alpha, beta):
    """The per-chunk quantities of the forward that do not depend on S."""
    L = q.shape[0]
    G = pair_gates(alpha)                      # G[i, j, c] = G_{i<-j,c}, j <= i
    Abar = np.einsum("ic,ijc,jc->ij", k, G, k) * np.tril(np.ones((L, L)), -1)
    M = np.einsum("ic,ijc,jc->ij", q, G, k) * np.tril(np.ones((L, L)))
    gamma = np.cumprod(alpha, axis=0)
    sigma = G[L - 1]                           # sigma_j = G_{L<-j}
    T = np.linalg.inv(np.eye(L) + beta[:, None] * Abar)
    return dict(G=G, Abar=Abar, M=M, gamma=gamma, sigma=sigma, T=T,
                Qhat=gamma * q, Khat=gamma * k, Kbar=sigma * k)


def chunk_fwd(S, q, k, v, alpha, beta, scale, parts=None):
    """(O, S_L, U) of one chunk from entry state S."""
    p = parts or chunk_parts(q, k, v, alpha, beta)
    U = p["T"] @ (beta[:, None] * (v - p["Khat"] @ S))
    O = scale * (p["Qhat"] @ S + p["M"] @ U)
    S_L = p["gamma"][-1][:, None] * S + p["Kbar"].T @ U
    return O, S_L, U


def gate_grad(E, alpha):
    """dalpha[s-1, c] = sum_{0 <= j < s <= i <= L} E[i, j, c] G_{s-1<-j,c} G_{i<-s,c}.

    E is [L+1, L+1, d] over positions 0..L (row i, column j, j < i); position
    0 is the chunk entry. Two running products per channel, no division:
    F_s(i) = sum_{j<s} G_{s-1<-j} E_ij grows by F_{s+1} = alpha_s F_s + E_{., s},
    and the sum over i >= s is a Horner pass backwards from i = L.
    """
    L = alpha.shape[0]
    d = alpha.shape[1]
    out = np.zeros((L, d))
    F = E[:, 0, :].copy()                      # F_1(i) = E_{i0}
    for s in range(1, L + 1):
        if s > 1:
            F = alpha[s - 2] * F + E[:, s - 1, :]
        h = F[L].copy()
        for i in range(L - 1, s - 1, -1):
            h = alpha[i] * h + F[i]            # alpha[i] is alpha_{i+1}
        out[s - 1] = h
    return out


def chunk_bwd(S, dS_L, q, k, v, alpha, beta, do, scale):
    """Gradients of one chunk: (dq, dk, dv, dalpha, dbeta, dS)."""
    L = q.shape[0]
    p = chunk_parts(q, k, v, alpha, beta)
    G, M, Abar, T = p["G"], p["M"], p["Abar"], p["T"]
    gamma, sigma = p["gamma"], p["sigma"]
    U = T @ (beta[:, None] * (v - p["Khat"] @ S))

    dU = scale * M.T @ do + p["Kbar"] @ dS_L
    dR = T.T @ dU
    dS = (scale * p["Qhat"].T @ do + gamma[-1][:, None] * dS_L
          - p["Khat"].T @ (beta[:, None] * dR))
    dv = beta[:, None] * dR
    w = v - p["Khat"] @ S - Abar @ U
    dbeta = np.einsum("iv,iv->i", dR, w)
    dM = scale * (do @ U.T) * np.tril(np.ones((L, L)))
    dAbar = -(beta[:, None] * (dR @ U.T)) * np.tril(np.ones((L, L)), -1)
    dQhat = scale * do @ S.T
    dKhat = -(beta[:, None] * dR) @ S.T
    dKbar = U @ dS_L.T

    # Gram terms: M_ij = sum_c q_ic G_ijc k_jc, Abar_ij = sum_c k_ic G_ijc k_jc
    dq = gamma * dQhat + np.einsum("ij,ijc,jc->ic", dM, G, k)
    dk = (gamma * dKhat + sigma * dKbar
          + np.einsum("ij,ijc,ic->jc", dM, G, q)
          + np.einsum("ij,ijc,ic->jc", dAbar, G, k)
          + np.einsum("ij,ijc,jc->ic", dAbar, G, k))

    # coefficients of G_{i<-j} over positions 0..L (0 = entry, L = exit)
    d = q.shape[1]
    E = np.zeros((L + 1, L + 1, d))
    E[1:, 1:] = (np.einsum("ij,ic,jc->ijc", dM, q, k)
                 + np.einsum("ij,ic,jc->ijc", dAbar, k, k))
    for i in range(L + 1):
        E[i, i] = 0.0                          # G_{i<-i} = I holds no gate
    E[1:, 0] = q * dQhat + k * dKhat           # gamma_i = G_{i<-0}
    E[L, 1:L] += (k * dKbar)[:L - 1]           # sigma_j = G_{L<-j}, j < L
    E[L, 0] += np.einsum("cv,cv->c", S, dS_L)  # diag(gamma_L) S
    dalpha = gate_grad(E, alpha)
    return dq, dk, dv, dalpha, dbeta, dS


def chunked_bwd(q, k, v, alpha, beta, do, S0, dS_final, C, scale=1.0):
    """One head of one sequence [T, d]: the forward over chunks keeps each
    chunk's entry state, then the reverse scan carries dS chunk by chunk."""
    Tn = q.shape[0]
    starts = list(range(0, Tn, C))
    S = np.array(S0, dtype=np.float64, copy=True)
    entry = []
    for s in starts:
        e = min(Tn, s + C)
        entry.append(S)
        _, S, _ = chunk_fwd(S, q[s:e], k[s:e], v[s:e], alpha[s:e], beta[s:e], scale)
    grads = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v),
             np.zeros_like(alpha), np.zeros_like(beta)]
    dS = np.array(dS_final, dtype=np.float64, copy=True)
    for n in range(len(starts) - 1, -1, -1):
        s = starts[n]
        e = min(Tn, s + C)
        r = chunk_bwd(entry[n], dS, q[s:e], k[s:e], v[s:e], alpha[s:e],
                      beta[s:e], do[s:e], scale)
        for g, x in zip(grads, r[:5]):
            g[s:e] = x
        dS = r[5]
    return (*grads, dS)


# ---------------------------------------------------------------------------
# The same gradients split into the phases a GPU implementation runs: the
# forward scan keeps each chunk's entry state; a per-chunk prep (parallel over
# chunks) folds T into two products; the reverse scan then carries only dS,
# with two dependent matrix products per chunk (as the forward scan does);
# last, every chunk's gradients follow from its (S, dS_L) in parallel.

def scan_prep(q, k, v, alpha, beta, do, scale):
    """Chunk-local terms of the reverse scan: dR = X + Wb dS_L and
    dS = P + diag(gamma_L) dS_L - BK^T dR."""
    p = chunk_parts(q, k, v, alpha, beta)
    T = p["T"]
    return dict(X=T.T @ (scale * p["M"].T @ do), Wb=T.T @ p["Kbar"],
                P=scale * p["Qhat"].T @ do, BK=beta[:, None] * p["Khat"],
                gL=p["gamma"][-1])


def scan_step(pr, dS_L):
    """One chunk of the reverse scan: dS_L -> (dR, dS)."""
    dR = pr["X"] + pr["Wb"] @ dS_L
    return dR, pr["P"] + pr["gL"][:, None] * dS_L - pr["BK"].T @ dR


def chunked_bwd_phased(q, k, v, alpha, beta, do, S0, dS_final, C, scale=1.0):
    Tn = q.shape[0]
    spans = [(s, min(Tn, s + C)) for s in range(0, Tn, C)]
    S = np.array(S0, dtype=np.float64, copy=True)
    entry = []
    for s, e in spans:                         # forward scan: entry states
        entry.append(S)
        _, S, _ = chunk_fwd(S, q[s:e], k[s:e], v[s:e], alpha[s:e], beta[s:e], scale)
    preps = [scan_prep(q[s:e], k[s:e], v[s:e], alpha[s:e], beta[s:e], do[s:e], scale)
             for s, e in spans]                # parallel over chunks
    exit_grad = [None] * len(spans)
    dS = np.array(dS_final, dtype=np.float64, copy=True)
    for n in range(len(spans) - 1, -1, -1):    # reverse scan: dS only
        exit_grad[n] = dS
        _, dS = scan_step(preps[n], dS)
    grads = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v),
             np.zeros_like(alpha), np.zeros_like(beta)]
    for n, (s, e) in enumerate(spans):         # parallel over chunks
        r = chunk_bwd(entry[n], exit_grad[n], q[s:e], k[s:e], v[s:e],
                      alpha[s:e], beta[s:e], do[s:e], scale)
        for g, x in zip(grads, r[:5]):
            g[s:e] = x
    return (*grads, dS)


# ---------------------------------------------------------------------------
# The gated Gram adjoints through the bounded factorisation of the forward:
# for sub-blocks I > J (c tokens each) and r the last position of block I-1,
# G_{i<-j} = G_{i<-r} G_{r<-j} with both factors of magnitude <= 1, so each
# off-diagonal block is a plain matrix product of gate-scaled operands; the
# diagonal blocks take the per-pair gates directly.

def gram_adjoints(dM, dAbar, q, k, alpha, c=16):
    """(dq, dk) contributions of M (j <= i) and Abar (j < i):
    dq_i = sum_j dM_ij G_ij k_j; dk_j = sum_i (dM_ij G_ij q_i + dAbar_ij G_ij k_i);
    dk_i += sum_j dAbar_ij G_ij k_j."""
    L, d = q.shape
    dq = np.zeros((L, d))
    dk = np.zeros((L, d))
    nb = (L + c - 1) // c
    for I in range(nb):
        i0, i1 = I * c, min(L, I * c + c)
        # diagonal block: per-pair gates
        G = pair_gates(alpha[i0:i1])
        dMb, dAb = dM[i0:i1, i0:i1], dAbar[i0:i1, i0:i1]
        qI, kI = q[i0:i1], k[i0:i1]
        dq[i0:i1] += np.einsum("ij,ijc,jc->ic", dMb, G, kI)
        dk[i0:i1] += (np.einsum("ij,ijc,ic->jc", dMb, G, qI)
                      + np.einsum("ij,ijc,ic->jc", dAb, G, kI)
                      + np.einsum("ij,ijc,jc->ic", dAb, G, kI))
        if I == 0:
            continue
        r = i0 - 1                                     # last position of block I-1
        F = np.cumprod(alpha[i0:i1], axis=0)           # F_i = G_{i<-r}
        for J in range(I):
            j0, j1 = J * c, (J + 1) * c
            # B_j = G_{r<-j} = prod alpha[j+1..r]: suffix products within [j0, r]
            B = np.ones((j1 - j0, d))
            acc = np.ones(d)
            for t in range(r, j0 - 1, -1):
                if t < j1:
                    B[t - j0] = acc
                acc = acc * alpha[t]
            dMb, dAb = dM[i0:i1, j0:j1], dAbar[i0:i1, j0:j1]
            kJB = k[j0:j1] * B
            dq[i0:i1] += F * (dMb @ kJB)
            dk[i0:i1] += F * (dAb @ kJB)
            dk[j0:j1] += B * (dMb.T @ (F * qI) + dAb.T @ (F * kI))
    return dq, dk
