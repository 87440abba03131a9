"""The chunkwise backward (``chunk_bwd_fp64``) reproduces the oracle's
token-serial adjoint in fp64, for every chunk length and on the gates where a
log-space gate gradient breaks down (alpha = 0 exactly, alpha = -1, tiny
|alpha|). The oracle is itself pinned to central finite differences of the
forward (``test_oracle_bwd.py``), so this ties the chunk formulas, including
the division-free gate gradient, to the recurrence of "Semidirect Fourier
Delta Attention" §1 eq. (1)."""
import numpy as np
import pytest

import oracle
from chunk_bwd_fp64 import chunked_bwd, chunked_bwd_phased, gate_grad, gram_adjoints
from chunk_wy_fp64 import pair_gates


def case(seed, T, dk=5, dv=4, gates="mixed"):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(T, dk))
    k = rng.normal(size=(T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.normal(size=(T, dv))
    alpha = np.tanh(2 * rng.normal(size=(T, dk)))
    if gates == "mixed":                       # exact 0 and +-1 entries, some tiny
        u = rng.uniform(size=(T, dk))
        alpha = np.where(u < 0.08, np.sign(rng.normal(size=(T, dk))), alpha)
        alpha = np.where((u >= 0.08) & (u < 0.16), 0.0, alpha)
        alpha = np.where((u >= 0.16) & (u < 0.2), 1e-9 * rng.normal(size=(T, dk)), alpha)
    elif gates == "zero":
        alpha = np.zeros((T, dk))
    elif gates == "sign":
        alpha = np.sign(rng.normal(size=(T, dk)))
    beta = rng.uniform(0, 2, size=T)
    do = rng.normal(size=(T, dv))
    s0 = rng.normal(size=(dk, dv))
    gf = rng.normal(size=(dk, dv))
    return q, k, v, alpha, beta, do, s0, gf


def oracle_head(q, k, v, alpha, beta, do, s0, gf, scale):
    r = oracle.bwd(q[:, None], k[:, None], v[:, None], alpha[:, None], beta[:, None],
                   do[:, None], s0[None, None], gf[None, None], scale=scale)
    return tuple(x[:, 0] for x in r[:5]) + (r[5][0, 0],)


NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dS0")


def check(got, want, tol=1e-10):
    for name, a, b in zip(NAMES, got, want):
        err = np.abs(a - b).max() / max(1.0, np.abs(b).max())
        assert err < tol, (name, err)


@pytest.mark.parametrize("C", [1, 3, 4, 16, 64])
def test_chunked_backward_equals_the_token_adjoint(C):
    args = case(C, T=37)
    want = oracle_head(*args, scale=0.8)
    got = chunked_bwd(*args, C, scale=0.8)
    check(got, want)


@pytest.mark.parametrize("gates", ["zero", "sign", "plain"])
def test_degenerate_gates(gates):
    args = case(11, T=20, gates=gates)
    want = oracle_head(*args, scale=1.0)
    check(chunked_bwd(*args, 8, scale=1.0), want)


def test_zero_gate_gradient_is_finite_and_exact():
    """A zero gate still has a gradient: the loss moves when alpha leaves 0.
    The log-space form (alpha dalpha, then divide) has nothing to divide here."""
    args = list(case(5, T=16, gates="plain"))
    args[3][7, 2] = 0.0
    want = oracle_head(*args, scale=1.0)
    got = chunked_bwd(*args, 16, scale=1.0)
    assert abs(want[3][7, 2]) > 1e-3
    check(got, want)


def test_no_write_gradient_is_the_gla_form():
    """beta = 0: nothing is written, so S_t = diag(gamma_t) S_0, the diagonal
    (GLA-type) closed form; then dq_t = scale gamma_t * (S_0 do_t) and dv = 0."""
    q, k, v, alpha, beta, do, s0, gf = case(8, T=12, gates="plain")
    beta = np.zeros_like(beta)
    got = chunked_bwd(q, k, v, alpha, beta, do, s0, gf, 5, scale=0.5)
    gamma = np.cumprod(alpha, axis=0)
    np.testing.assert_allclose(got[0], 0.5 * gamma * (do @ s0.T), atol=1e-12)
    np.testing.assert_allclose(got[2], 0.0, atol=0)


def test_gate_grad_is_the_leave_one_out_product():
    """gate_grad against the triple sum written out, on a tiny case."""
    rng = np.random.default_rng(2)
    L, d = 5, 3
    alpha = rng.uniform(-1, 1, size=(L, d))
    alpha[2, 1] = 0.0
    E = np.tril(rng.normal(size=(L + 1, L + 1, d)).transpose(2, 0, 1), -1).transpose(1, 2, 0)
    want = np.zeros((L, d))
    for s in range(1, L + 1):
        for j in range(s):
            for i in range(s, L + 1):
                p = np.ones(d)
                for t in range(j + 1, i + 1):
                    if t != s:
                        p = p * alpha[t - 1]
                want[s - 1] += E[i, j] * p
    np.testing.assert_allclose(gate_grad(E, alpha), want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("C", [4, 16, 64])
def test_phased_form_equals_the_plain_chunk_form(C):
    args = case(21 + C, T=70)
    want = chunked_bwd(*args, C, scale=0.6)
    got = chunked_bwd_phased(*args, C, scale=0.6)
    check(got, want, tol=1e-12)


@pytest.mark.parametrize("L", [64, 40, 16, 7])
@pytest.mark.parametrize("gates", ["mixed", "zero", "sign"])
def test_blocked_gram_adjoints_equal_the_per_pair_form(L, gates):
    q, k, _, alpha, _, _, _, _ = case(L, T=L, dk=6, gates=gates)
    rng = np.random.default_rng(L + 1)
    dM = np.tril(rng.normal(size=(L, L)))
    dA = np.tril(rng.normal(size=(L, L)), -1)
    G = pair_gates(alpha)
    want_q = np.einsum("ij,ijc,jc->ic", dM, G, k)
    want_k = (np.einsum("ij,ijc,ic->jc", dM, G, q) + np.einsum("ij,ijc,ic->jc", dA, G, k)
              + np.einsum("ij,ijc,jc->ic", dA, G, k))
    got_q, got_k = gram_adjoints(dM, dA, q, k, alpha, c=16)
    np.testing.assert_allclose(got_q, want_q, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got_k, want_k, rtol=0, atol=1e-12)
