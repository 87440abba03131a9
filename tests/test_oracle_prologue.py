"""Pins of the oracle's fused input prologue (gate_prologue): the stable
parameterisation of "Semidirect Fourier Delta Attention" §3 eqs. (15), (17),
(18), checked against closed forms, limits and a worked trace carried
through the whole gated forward."""
import numpy as np
import pytest

import oracle

CKDA = dict(alpha_min=-1.0, alpha_max=1.0, beta_max=2.0)
KDA = dict(alpha_min=0.0, alpha_max=1.0, beta_max=1.0)
RNG = np.random.default_rng(11)


def prologue(a, c, k, gates, eps=0.0):
    return oracle.gate_prologue(a, c, k, k_eps=eps, **gates)


def test_zero_logits_give_the_middle_of_the_ranges_exactly():
    a = np.zeros((3, 2, 4))
    c = np.zeros((3, 2))
    k = RNG.standard_normal((3, 2, 4))
    al, be, _ = prologue(a, c, k, CKDA)
    assert np.all(al == 0.0) and np.all(be == 1.0)  # CKDA: alpha = 0, beta = 1
    al, be, _ = prologue(a, c, k, KDA)
    assert np.all(al == 0.5) and np.all(be == 0.5)


def test_ckda_gate_is_tanh_of_half_the_logit():
    a = RNG.standard_normal((50, 3, 8)) * 4
    al, _, _ = prologue(a, np.zeros((50, 3)), np.ones((50, 3, 8)), CKDA)
    np.testing.assert_allclose(al, np.tanh(a / 2), rtol=0, atol=1e-15)


def test_kda_gate_is_exp_of_minus_softplus():
    # the KDA range of the workloads, exp(-softplus(x)), is sigmoid(-x)
    x = RNG.standard_normal((40, 2, 8)) * 3
    al, _, _ = prologue(-x, np.zeros((40, 2)), np.ones((40, 2, 8)), KDA)
    np.testing.assert_allclose(al, np.exp(-np.logaddexp(0.0, x)), rtol=1e-15, atol=0)


def test_limits_and_ranges():
    a = np.array([[[-800.0, -40.0, 0.0, 40.0, 800.0]]])
    c = np.array([[-800.0]]), np.array([[800.0]])
    for gates in (CKDA, KDA, dict(alpha_min=-0.5, alpha_max=0.25, beta_max=1.5)):
        al, b0, _ = prologue(a, c[0], np.ones_like(a), gates)
        _, b1, _ = prologue(a, c[1], np.ones_like(a), gates)
        assert al[0, 0, 0] == gates["alpha_min"] and al[0, 0, 4] == gates["alpha_max"]
        assert abs(al[0, 0, 1] - gates["alpha_min"]) < 1e-16
        assert abs(al[0, 0, 3] - gates["alpha_max"]) < 1e-16
        assert b0[0, 0] == 0.0 and b1[0, 0] == gates["beta_max"]
        x = RNG.standard_normal((200, 1, 8)) * 10
        al, be, _ = prologue(x, x[..., 0], np.ones_like(x), gates)
        assert al.min() >= gates["alpha_min"] and al.max() <= gates["alpha_max"]
        assert be.min() >= 0.0 and be.max() <= gates["beta_max"]


@pytest.mark.parametrize("eps", [0.0, 1e-6, 0.5])
def test_key_normalisation(eps):
    kr = RNG.standard_normal((30, 4, 16)) * RNG.uniform(0.01, 5.0, (30, 4, 1))
    kr[3, 1] = 0.0  # a zero key row
    _, _, k = prologue(np.zeros_like(kr), np.zeros((30, 4)), kr, CKDA, eps)
    n_raw = np.linalg.norm(kr, axis=-1)
    n = np.linalg.norm(k, axis=-1)
    keep = n_raw > 0
    np.testing.assert_allclose(n[keep], n_raw[keep] / (n_raw[keep] + eps), rtol=1e-14)
    if eps == 0.0:
        np.testing.assert_allclose(n[keep], 1.0, rtol=1e-15)
    assert np.all(k[3, 1] == 0.0)
    # direction unchanged
    cos = (k * kr).sum(-1)[keep] / (n[keep] * n_raw[keep])
    np.testing.assert_allclose(cos, 1.0, rtol=1e-14)


def test_worked_overwrite_trace_through_the_gated_forward():
    """The lesson's beta = 1 correction (Kimi Delta Attention: a bounded case
    study, the worked trace of Exercise 2): with unit key e2 and beta = 1 the
    written row of the state becomes exactly v = [4, 4]; two steps with gates
    [1, 0.2] then leave 4 * 0.2^2 = 0.16 there. Reached through the prologue:
    c = 0 with beta_max = 2 gives beta = 1, the raw key 3 e2 normalises to e2
    (eps = 0), logit 800 gives alpha = 1 and tanh(a/2) = 0.2 gives 0.2."""
    a02 = 2 * np.arctanh(0.2)
    q = np.zeros((3, 1, 2)); q[:, 0, 1] = 1.0
    k = np.zeros((3, 1, 2)); k[:, 0, 1] = 3.0
    v = np.zeros((3, 1, 2)); v[0, 0] = [4.0, 4.0]
    a = np.full((3, 1, 2), 800.0); a[1:, 0, 1] = a02
    c = np.array([[0.0], [-800.0], [-800.0]])
    s0 = np.zeros((1, 1, 2, 2)); s0[0, 0, 0] = [1.0, -2.0]
    o, sf = oracle.fwd_gated(q, k, v, a, c, dict(CKDA, k_eps=0.0), s0,
                             np.array([0, 3], dtype=np.int32))
    assert o[0, 0, 0] == 4.0 and o[0, 0, 1] == 4.0  # row 2 of S_1 read by q = e2
    np.testing.assert_allclose(o[2, 0], [0.16, 0.16], rtol=1e-14)
    np.testing.assert_allclose(sf[0, 0, 1], [0.16, 0.16], rtol=1e-14)
    np.testing.assert_allclose(sf[0, 0, 0], [1.0, -2.0], rtol=0, atol=0)
