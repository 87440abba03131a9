"""Pins of the complex-phase-gate oracle (``oracle.fwd_complex``,
"Semidirect Fourier Delta Attention" §3 eqs. (13)-(14)) against things other
than itself:
  * theta = 0 with real inputs reduces to the real recurrence, computed by the
    independent C oracle (``oracle.fwd``);
  * a pure phase gate (alpha = 1, beta = 0) rotates every state entry by
    exp(i sum theta): S_T = diag(exp(i sum_t theta_t)) S_0 and o_t = scale S_t^* q_t
    in closed form;
  * the gate acts on each (real, imaginary) pair as the 2x2 rotation-decay
    block alpha R(theta) (the page's real implementation);
  * with |alpha| = 1, beta in {0, 2} and unit complex keys every transition is
    unitary, so ||S||_F is preserved exactly (this needs the conjugate in
    k k^*: with k k^T the beta = 2 step is not unitary);
  * with v = 0, alpha, beta in [0, 1] and ||k|| <= 1 the state norm never grows;
  * the dense affine composition of the per-token maps S -> A_t S + B_t;
  * the chunkwise (WY / UT) form in complex arithmetic (``chunk_wy_fp64``),
    for several chunk lengths.
Two planted mistakes (the projector without the conjugate, the readout without
it) are each caught.
"""
import inspect

import numpy as np
import pytest

import oracle
from chunk_wy_fp64 import chunk_step_complex


def cplx(rng, *shape):
    return rng.normal(size=shape) + 1j * rng.normal(size=shape)


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def case(seed, T=9, H=2, dk=4, dv=3, real=False):
    rng = np.random.default_rng(seed)
    if real:
        q, k, v = rng.normal(size=(T, H, dk)), rng.normal(size=(T, H, dk)), rng.normal(size=(T, H, dv))
        s0 = rng.normal(size=(1, H, dk, dv))
    else:
        q, k, v = cplx(rng, T, H, dk), cplx(rng, T, H, dk), cplx(rng, T, H, dv)
        s0 = cplx(rng, 1, H, dk, dv)
    k = unit_rows(k)
    alpha = rng.uniform(0, 1, size=(T, H, dk))
    theta = rng.uniform(-np.pi, np.pi, size=(T, H, dk))
    beta = rng.uniform(0, 1, size=(T, H))
    return q, k, v, alpha, theta, beta, s0


def test_theta_zero_real_inputs_is_the_real_recurrence():
    q, k, v, alpha, theta, beta, s0 = case(1, real=True)
    alpha = np.tanh(np.random.default_rng(2).normal(size=alpha.shape) * 2)  # CKDA gates
    beta = 2 * beta
    o, sf = oracle.fwd_complex(q, k, v, alpha, np.zeros_like(theta), beta, s0, scale=0.7)
    o_r, sf_r = oracle.fwd(q, k, v, alpha, beta, s0, None, 0.7)
    np.testing.assert_allclose(o, o_r, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sf, sf_r, rtol=0, atol=1e-12)
    assert np.abs(o.imag).max() == 0 and np.abs(sf.imag).max() == 0


def test_pure_phase_rotates_the_state():
    q, k, v, alpha, theta, beta, s0 = case(3)
    alpha = np.ones_like(alpha)
    beta = np.zeros_like(beta)
    o, sf = oracle.fwd_complex(q, k, v, alpha, theta, beta, s0, scale=1.3)
    phase = np.zeros_like(theta[0])
    for t in range(q.shape[0]):
        phase = phase + theta[t]
        st = np.exp(1j * phase)[:, :, None] * s0[0]              # [H, dk, dv]
        ref = 1.3 * np.einsum("hkv,hk->hv", st.conj(), q[t])     # S^* q
        np.testing.assert_allclose(o[t], ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sf[0], np.exp(1j * phase)[:, :, None] * s0[0], rtol=0, atol=1e-12)


def test_gate_is_a_rotation_decay_block_on_real_pairs():
    """One token with beta = 0 and q = e_r: the (real, imaginary) parts of the
    new state row r are alpha R(theta) applied to those of the old row."""
    rng = np.random.default_rng(5)
    dk, dv = 3, 2
    s0 = cplx(rng, 1, 1, dk, dv)
    alpha = rng.uniform(0, 1, size=(1, 1, dk))
    theta = rng.uniform(-3, 3, size=(1, 1, dk))
    _, sf = oracle.fwd_complex(np.zeros((1, 1, dk)), np.zeros((1, 1, dk)), np.zeros((1, 1, dv)),
                               alpha, theta, np.zeros((1, 1)), s0)
    for r in range(dk):
        c, s, a = np.cos(theta[0, 0, r]), np.sin(theta[0, 0, r]), alpha[0, 0, r]
        x, y = s0[0, 0, r].real, s0[0, 0, r].imag
        np.testing.assert_allclose(sf[0, 0, r].real, a * (c * x - s * y), atol=1e-14)
        np.testing.assert_allclose(sf[0, 0, r].imag, a * (s * x + c * y), atol=1e-14)


def norm_steps(fn, q, k, v, alpha, theta, beta, s0):
    """||S_t||_F after each prefix, from independent calls on growing prefixes."""
    out = []
    for t in range(1, q.shape[0] + 1):
        _, sf = fn(q[:t], k[:t], v[:t], alpha[:t], theta[:t], beta[:t], s0)
        out.append(np.linalg.norm(sf))
    return np.array(out)


@pytest.mark.parametrize("b", [0.0, 2.0])
def test_unitary_transitions_preserve_the_norm(b):
    q, k, v, alpha, theta, beta, s0 = case(7, T=12)
    v = np.zeros_like(v)
    alpha = np.ones_like(alpha)
    beta = np.full_like(beta, b)
    n = norm_steps(oracle.fwd_complex, q, k, v, alpha, theta, beta, s0)
    np.testing.assert_allclose(n, np.linalg.norm(s0), rtol=1e-12)


def test_state_norm_never_grows_without_writes():
    q, k, v, alpha, theta, beta, s0 = case(9, T=12)
    v = np.zeros_like(v)
    n = norm_steps(oracle.fwd_complex, q, k, v, alpha, theta, beta, s0)
    assert np.all(np.diff(np.concatenate([[np.linalg.norm(s0)], n])) <= 1e-12)


def test_dense_affine_composition():
    q, k, v, alpha, theta, beta, s0 = case(11, T=7, H=1)
    o, sf = oracle.fwd_complex(q, k, v, alpha, theta, beta, s0, scale=0.9)
    dk = q.shape[2]
    Acc = np.eye(dk, dtype=complex)
    Bcc = np.zeros_like(s0[0, 0])
    for t in range(q.shape[0]):
        lam = np.diag(alpha[t, 0] * np.exp(1j * theta[t, 0]))
        kt = k[t, 0][:, None]
        A = (np.eye(dk) - beta[t, 0] * kt @ kt.conj().T) @ lam
        B = beta[t, 0] * kt @ v[t, 0][None, :].conj()
        Acc, Bcc = A @ Acc, A @ Bcc + B
        st = Acc @ s0[0, 0] + Bcc
        np.testing.assert_allclose(o[t, 0], 0.9 * st.conj().T @ q[t, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sf[0, 0], Acc @ s0[0, 0] + Bcc, rtol=0, atol=1e-12)


@pytest.mark.parametrize("C", [1, 4, 16])
def test_chunk_form_matches(C):
    q, k, v, alpha, theta, beta, s0 = case(13, T=37, H=1, dk=5, dv=3)
    alpha = np.where(np.random.default_rng(4).uniform(size=alpha.shape) < 0.1, 0.0, alpha)
    beta = 2 * beta
    o, sf = oracle.fwd_complex(q, k, v, alpha, theta, beta, s0, scale=0.7)
    lam = alpha[:, 0] * np.exp(1j * theta[:, 0])
    S = s0[0, 0]
    for s in range(0, 37, C):
        e = min(37, s + C)
        oc, S = chunk_step_complex(S, q[s:e, 0], k[s:e, 0], v[s:e, 0], lam[s:e], beta[s:e, 0], 0.7)
        np.testing.assert_allclose(oc, o[s:e, 0], rtol=0, atol=1e-11)
    np.testing.assert_allclose(S, sf[0, 0], rtol=0, atol=1e-11)


MUTATIONS = [
    ("projector without the conjugate", "np.outer(kt, kt.conj() @ S)", "np.outer(kt, kt @ S)"),
    ("readout without the conjugate", "(S.conj().T @ q[t, h])", "(S.T @ q[t, h])"),
]


@pytest.mark.parametrize("what,old,new", MUTATIONS)
def test_planted_mistakes_are_caught(what, old, new):
    src = inspect.getsource(oracle.fwd_complex)
    assert src.count(old) == 1, what
    ns = {"np": np, "_f64": oracle._f64}
    exec(src.replace(old, new), ns)
    bad = ns["fwd_complex"]
    caught = False
    # the unitary-norm pin (beta = 2) and the pure-phase readout pin
    q, k, v, alpha, theta, beta, s0 = case(7, T=12)
    n = norm_steps(bad, q, k, np.zeros_like(v), np.ones_like(alpha), theta,
                   np.full_like(beta, 2.0), s0)
    caught |= not np.allclose(n, np.linalg.norm(s0), rtol=1e-9)
    q, k, v, alpha, theta, beta, s0 = case(3)
    o, _ = bad(q, k, v, np.ones_like(alpha), theta, np.zeros_like(beta), s0, scale=1.3)
    st = np.exp(1j * theta[0])[:, :, None] * s0[0]
    caught |= not np.allclose(o[0], 1.3 * np.einsum("hkv,hk->hv", st.conj(), q[0]), atol=1e-9)
    assert caught, what
