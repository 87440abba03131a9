"""Pins of the oracle's backward pass (``oracle.bwd``).

The pages give the forward recurrence only, so the backward is pinned
against things other than itself:
  * central finite differences of the forward oracle (``oracle.fwd``, the C
    token recurrence pinned in test_oracle_pins.py) for every input: q, k,
    v, alpha, beta and the initial state, on small cases with negative,
    zero and unit gates and beta up to 2, varlen, with and without a
    final-state gradient;
  * the beta = 0 closed form (the diagonal SSM of Prop. 2.1 of "Semidirect
    Fourier Delta Attention": S_t = Lambda_t S_0 with Lambda_t the running
    product of diag(alpha)), where dk = dv = 0 exactly and dq, dS_0 are
    explicit sums;
  * planted mistakes in a copy of the per-head routine, each of which the
    finite differences must reject.
"""
import inspect

import numpy as np
import pytest

import oracle


def make_case(seed, lens, H, dk, dv, zero_gates=True):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    q = rng.normal(size=(T, H, dk))
    k = rng.normal(size=(T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(T, H, dv))
    alpha = np.tanh(rng.normal(size=(T, H, dk)) * 1.5)
    if zero_gates:
        alpha[0, 0, 0] = 0.0
        alpha[min(1, T - 1), 0, dk - 1] = -1.0
        alpha[T - 1, H - 1, 0] = 1.0
    beta = 2.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    beta[0, 0] = 2.0
    s0 = rng.normal(size=(len(lens), H, dk, dv)) * 0.3
    do = rng.normal(size=(T, H, dv))
    dsf = rng.normal(size=(len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, s0=s0, do=do, dsf=dsf, cu=cu)


def loss(c, scale, with_final, **over):
    x = dict(c, **over)
    o, sf = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["s0"],
                       x["cu"], scale)
    L = float((o * c["do"]).sum())
    if with_final:
        L += float((sf * c["dsf"]).sum())
    return L


def fd_grad(c, name, scale, with_final, h=1e-6):
    x = c[name]
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        xp = x.copy(); xp[idx] += h
        xm = x.copy(); xm[idx] -= h
        g[idx] = (loss(c, scale, with_final, **{name: xp}) -
                  loss(c, scale, with_final, **{name: xm})) / (2 * h)
    return g


def analytic(c, scale, with_final, head=None):
    return oracle.bwd(c["q"], c["k"], c["v"], c["alpha"], c["beta"], c["do"], c["s0"],
                      c["dsf"] if with_final else None, c["cu"], scale, _head=head)


NAMES = ["q", "k", "v", "alpha", "beta", "s0"]


@pytest.mark.parametrize("seed,lens,H,dk,dv,scale,with_final", [
    (1, [5], 1, 3, 2, 1.0, False),
    (2, [3, 4], 2, 3, 2, 0.7, True),
    (3, [1, 6, 2], 1, 4, 3, 1.3, True),
])
def test_bwd_matches_finite_differences(seed, lens, H, dk, dv, scale, with_final):
    c = make_case(seed, lens, H, dk, dv)
    got = analytic(c, scale, with_final)
    for name, g in zip(NAMES, got):
        ref = fd_grad(c, name, scale, with_final)
        err = np.abs(g - ref).max()
        assert err <= 1e-7 * max(1.0, np.abs(ref).max()), (name, err)


def test_bwd_beta_zero_closed_form():
    """beta = 0: S_t = Lambda_t S_0 (Lambda_t = prod_{s<=t} diag(alpha_s)), so
    dk = dv = 0, dq_t = scale Lambda_t S_0 do_t and
    dS_0 = scale sum_t Lambda_t q_t do_t^T + Lambda_T dS_T."""
    c = make_case(7, [6], 1, 4, 3)
    c["beta"] = np.zeros_like(c["beta"])
    scale = 0.9
    dq, dk, dv, dal, dbe, ds0 = analytic(c, scale, True)
    assert np.all(dk == 0.0) and np.all(dv == 0.0)
    lam = np.ones(4)
    dq_ref = np.zeros_like(dq)
    ds0_ref = np.zeros((4, 3))
    for t in range(6):
        lam = lam * c["alpha"][t, 0]
        dq_ref[t, 0] = scale * (lam[:, None] * c["s0"][0, 0]) @ c["do"][t, 0]
        ds0_ref += scale * lam[:, None] * np.outer(c["q"][t, 0], c["do"][t, 0])
    ds0_ref += lam[:, None] * c["dsf"][0, 0]
    np.testing.assert_allclose(dq, dq_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ds0[0, 0], ds0_ref, rtol=1e-12, atol=1e-12)


MUTATIONS = [
    ("dk_t = beta_t (G w - S' g)", "dk[t] = beta[t] * (G @ w - Sp @ g)", "dk[t] = beta[t] * (G @ w)"),
    ("dalpha against the new state", "dal[t] = (dSp * S_prev).sum(axis=1)", "dal[t] = (dSp * St).sum(axis=1)"),
    ("no gate on the carried gradient", "G = alpha[t][:, None] * dSp", "G = dSp"),
    ("readout gradient unscaled", "G = G + scale * np.outer(q[t], do[t])", "G = G + np.outer(q[t], do[t])"),
    ("dbeta against v", "dbe[t] = g @ w", "dbe[t] = g @ v[t]"),
    ("rank-one term dropped from dS'", "dSp = G - beta[t] * np.outer(k[t], g)", "dSp = G"),
]


@pytest.mark.parametrize("what,old,new", MUTATIONS)
def test_planted_mistakes_are_caught(what, old, new):
    src = inspect.getsource(oracle._bwd_head)
    assert src.count(old) == 1, what
    ns = {"np": np}
    exec(src.replace(old, new), ns)
    c = make_case(11, [2, 4], 1, 3, 2)
    got = analytic(c, 0.8, True, head=ns["_bwd_head"])
    worst = 0.0
    for name, g in zip(NAMES, got):
        ref = fd_grad(c, name, 0.8, True)
        worst = max(worst, np.abs(g - ref).max() / max(1.0, np.abs(ref).max()))
    assert worst > 1e-4, what
