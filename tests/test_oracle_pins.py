"""Pins of the fp64 oracle against what the pages and the mathematics fix.

No GPU. Each test names the passage it follows. Together they are chosen so a
plausible slip in the oracle (gate after the delta step, readout before the
update, a sign flip in the correction, a dropped beta, a transposed state)
fails at least one of them; ``test_oracle_mutations.py`` plants such slips in
copies of the oracle and checks that.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from chunk_wy_fp64 import chunk_step, chunked_fwd

GOLD = os.path.join(os.path.dirname(__file__), "golden", "lesson_traces.json")


def _cases():
    with open(GOLD) as f:
        return {c["id"]: c for c in json.load(f)["cases"]}


def one_head(q, k, v, alpha, beta, s0=None, scale=1.0, lib=None):
    """Run the oracle on a single (sequence, head): q,k,alpha [T,dk]; v [T,dv]."""
    T, dk = q.shape
    dv = v.shape[1]
    s0 = None if s0 is None else np.asarray(s0, float).reshape(1, 1, dk, dv)
    o, sf = oracle.fwd(q[:, None], k[:, None], v[:, None], alpha[:, None],
                       np.asarray(beta, float)[:, None], s0, None, scale,
                       lib=lib)
    return o[:, 0], sf[0, 0]


def rand_head(rng, T, dk, dv, alpha="ckda", beta_max=2.0):
    q = rng.standard_normal((T, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    if alpha == "ckda":
        a = np.tanh(2 * rng.standard_normal((T, dk)))
        u = rng.random((T, dk))
        a[u < 0.05] = 1.0
        a[(u >= 0.05) & (u < 0.10)] = -1.0
        a[(u >= 0.10) & (u < 0.14)] = 0.0
    else:
        a = np.exp(-np.log1p(np.exp(rng.standard_normal((T, dk)))))
    b = beta_max * rng.random(T)
    return q, k, v, a, b


# ---------------------------------------------------------------- worked traces

@pytest.mark.parametrize("cid", ["vector_gate_one_step", "vector_gate_variant_0p24",
                                 "per_channel_decay_row_10_10"])
def test_lesson_gate_traces(cid):
    """Exercise 1 worked solution / variant, and appendix §12.1 ([10,10] -> [9,2])."""
    c = _cases()[cid]
    dk, dv = c["d_k"], c["d_v"]
    q = np.eye(dk)[:1]
    k = np.zeros((1, dk))
    k[0, 0] = 1.0
    v = np.zeros((1, dv))
    _, S = one_head(q, k, v, np.array([c["alpha"]]), [c["beta"]],
                    s0=c["initial_state"])
    np.testing.assert_allclose(S, np.array(c["expected_state"]), atol=c["tol"])
    if "expected_ratio_channel2_vs_0p20" in c:
        _, S20 = one_head(q, k, v, np.array([[0.9, 0.2]]), [0.0],
                          s0=c["initial_state"])
        assert S[1, 0] / S20[1, 0] == pytest.approx(
            c["expected_ratio_channel2_vs_0p20"], abs=1e-12)
    # readout of each channel with q = e_r returns that channel's trace
    for r in range(dk):
        o, _ = one_head(np.eye(dk)[r:r + 1], k, v, np.array([c["alpha"]]),
                        [c["beta"]], s0=c["initial_state"])
        np.testing.assert_allclose(o[0], np.array(c["expected_state"])[r],
                                   atol=c["tol"])


def test_lesson_half_life():
    """Exercise 1: half-lives about 6.6 and 0.43 tokens, a 15x ratio.

    The oracle's trace after n steps of a constant gate is read off its state;
    the half-life is the n where the trace crosses 1/2, interpolated in log.
    """
    c = _cases()["half_life_ratio"]
    steps = 12
    dk = 2
    alpha = np.tile(np.array(c["alpha"]), (steps, 1))
    q = np.tile(np.eye(dk)[:1], (steps, 1))
    k = np.tile(np.eye(dk)[:1], (steps, 1))
    v = np.zeros((steps, 1))
    traces = []
    for n in range(1, steps + 1):
        _, S = one_head(q[:n], k[:n], v[:n], alpha[:n], np.zeros(n),
                        s0=[[1.0], [1.0]])
        traces.append(S[:, 0])
    traces = np.array(traces)  # [n, channel]
    # channel 1 (gate 0.9): the crossing lies between 6 and 7 steps
    assert traces[5, 0] > 0.5 > traces[6, 0]
    # channel 2 (gate 0.2): below 1/2 already after one step
    assert traces[0, 1] < 0.5
    hl = [math.log(0.5) / (math.log(traces[n - 1, ch]) / n)
          for ch, n in ((0, 7), (1, 1))]
    for got, want, tol in zip(hl, c["expected_half_life"], c["half_life_tol"]):
        assert abs(got - want) <= tol
    assert abs(hl[0] / hl[1] - c["expected_ratio"]) <= c["ratio_tol"]


def test_lesson_correction_then_decay():
    """Exercise 2: beta=1 correction -> exactly [4,4]; two 0.2 gates -> 0.160."""
    c = _cases()["correction_then_two_decays"]
    rng = np.random.default_rng(5)
    # any starting state; integer-valued so "exactly [4,4]" is exact in fp64
    s0 = rng.integers(-9, 10, (2, 2)).astype(float)
    steps = c["steps"]
    q = np.tile(np.array(c["readout_q"]), (len(steps), 1))
    k = np.array([s["k"] for s in steps])
    v = np.array([s["v"] for s in steps])
    a = np.array([s["alpha"] for s in steps])
    b = np.array([s["beta"] for s in steps])
    _, S1 = one_head(q[:1], k[:1], v[:1], a[:1], b[:1], s0=s0)
    assert np.array_equal(S1[1], np.array(c["expected_row2_after_step1"]))
    o, S3 = one_head(q, k, v, a, b, s0=s0)
    np.testing.assert_allclose(o[2], c["expected_readout_after_step3"],
                               atol=c["tol"])
    np.testing.assert_allclose(S3[1], c["expected_readout_after_step3"],
                               atol=c["tol"])
    # channel 1 keeps whatever the correction left there (gate 1 on it)
    np.testing.assert_allclose(S3[0], S1[0], atol=1e-15)


# ------------------------------------------------ dense affine composition

def dense_affine_prefix(q, k, v, alpha, beta, s0, scale=1.0):
    """Compose the per-token affine maps of §2.2 eq. (9) with eq. (10).

    A_t = (I - beta_t k_t k_t^T) diag(alpha_t), B_t = beta_t k_t v_t^T;
    (A2,B2) o (A1,B1) = (A2 A1, A2 B1 + B2). The running composite applied to
    S_0 gives S_t, read out as o_t = scale * S_t^T q_t (§3 eq. (14)).
    """
    T, dk = q.shape
    Acc = np.eye(dk)
    Bcc = np.zeros((dk, v.shape[1]))
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        A = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(alpha[t])
        B = beta[t] * np.outer(k[t], v[t])
        Acc, Bcc = A @ Acc, A @ Bcc + B
        o[t] = scale * (Acc @ s0 + Bcc).T @ q[t]
    return o, Acc @ s0 + Bcc


@pytest.mark.parametrize("seed,dk,dv,alpha", [(0, 4, 3, "ckda"), (1, 3, 5, "ckda"),
                                              (2, 4, 4, "kda"), (3, 2, 2, "ckda")])
def test_oracle_equals_dense_affine_composition(seed, dk, dv, alpha):
    rng = np.random.default_rng(seed)
    T = 8
    q, k, v, a, b = rand_head(rng, T, dk, dv, alpha)
    s0 = rng.standard_normal((dk, dv))
    o, S = one_head(q, k, v, a, b, s0=s0, scale=0.7)
    o_ref, S_ref = dense_affine_prefix(q, k, v, a, b, s0, scale=0.7)
    np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(S, S_ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("C", [1, 2, 4, 16, 64])
def test_chunked_equals_recurrent(C):
    """Exercise 2: chunking changes cost, never the numbers (fp64, to 1e-12)."""
    rng = np.random.default_rng(100 + C)
    T, dk, dv = 80, 8, 6
    q, k, v, a, b = rand_head(rng, T, dk, dv, "ckda")
    s0 = 0.3 * rng.standard_normal((dk, dv))
    o, S = one_head(q, k, v, a, b, s0=s0, scale=1.3)
    o_c, S_c = chunked_fwd(q, k, v, a, b, s0, C, scale=1.3)
    np.testing.assert_allclose(o, o_c, atol=1e-12, rtol=0)
    np.testing.assert_allclose(S, S_c, atol=1e-12, rtol=0)


def test_T_matrix_bound():
    """Columns of T=(I+A)^-1 are impulse responses of a non-expansive
    recurrence (Complex KDA, abstract): |T_ij| <= beta_i ||k_i|| <= 2."""
    rng = np.random.default_rng(11)
    worst = 0.0
    for _ in range(20):
        q, k, v, a, b = rand_head(rng, 64, 16, 4, "ckda")
        _, _, T = chunk_step(np.zeros((16, 4)), q, k, v, a, b, return_T=True)
        off = np.abs(np.tril(T, -1))
        assert np.all(off <= b[:, None] + 1e-12)
        worst = max(worst, off.max())
    assert worst <= 2.0


# ------------------------------------------------ invariants (Complex KDA)

def test_transition_non_expansive():
    """Complex KDA, abstract: DPLR transitions stay non-expansive for
    |alpha| <= 1, beta in [0,2], unit k: sigma_max(A_t) <= 1."""
    rng = np.random.default_rng(3)
    for _ in range(500):
        d = int(rng.integers(2, 9))
        k = rng.standard_normal(d)
        k /= np.linalg.norm(k)
        a = rng.uniform(-1, 1, d)
        b = rng.uniform(0, 2)
        A = (np.eye(d) - b * np.outer(k, k)) @ np.diag(a)
        assert np.linalg.norm(A, 2) <= 1 + 1e-12


def test_oracle_state_norm_non_increasing():
    rng = np.random.default_rng(4)
    T, dk, dv = 200, 8, 5
    q, k, v, a, b = rand_head(rng, T, dk, dv, "ckda")
    v[:] = 0.0
    S = rng.standard_normal((dk, dv))
    prev = np.linalg.norm(S)
    for t in range(T):
        _, S = one_head(q[t:t + 1], k[t:t + 1], v[t:t + 1], a[t:t + 1],
                        b[t:t + 1], s0=S)
        cur = np.linalg.norm(S)
        assert cur <= prev * (1 + 1e-13)
        prev = cur


def test_oracle_norm_preserved_orthogonal_transitions():
    """|alpha| = 1 with random signs and beta in {0, 2}: every transition is
    orthogonal (Complex KDA: orthogonal DPLR matrices are CKDA transitions),
    so ||S_t||_F stays ||S_0||_F over 1000 steps."""
    rng = np.random.default_rng(6)
    T, dk, dv = 1000, 6, 3
    q, k, v, _, _ = rand_head(rng, T, dk, dv, "ckda")
    a = rng.choice([-1.0, 1.0], size=(T, dk))
    b = rng.choice([0.0, 2.0], size=T)
    v[:] = 0.0
    s0 = rng.standard_normal((dk, dv))
    _, S = one_head(q, k, v, a, b, s0=s0)
    assert abs(np.linalg.norm(S) - np.linalg.norm(s0)) <= 1e-12 * np.linalg.norm(s0) * 10
    for t in range(5):
        A = (np.eye(dk) - b[t] * np.outer(k[t], k[t])) @ np.diag(a[t])
        np.testing.assert_allclose(A.T @ A, np.eye(dk), atol=1e-12)


@pytest.mark.parametrize("m", [3, 5, 8])
def test_oracle_rotation_from_gate_reflection(m):
    """Complex KDA, abstract: one delta step (beta=2) plus a reflection in the
    gate (alpha_1 = -1) is a 2D rotation. With k = (cos phi, sin phi, 0..),
    A = R(2 phi) + I on the rest; phi = pi/m returns to S_0 after m steps
    (a mod-m counter) and is R(2 n phi) after n steps."""
    phi = math.pi / m
    dk = dv = 3
    k = np.array([math.cos(phi), math.sin(phi), 0.0])
    steps = 2 * m + 1
    K = np.tile(k, (steps, 1))
    a = np.tile(np.array([-1.0, 1.0, 1.0]), (steps, 1))
    b = np.full(steps, 2.0)
    v = np.zeros((steps, dv))
    q = np.tile(np.eye(dk)[:1], (steps, 1))
    s0 = np.eye(dk)
    for n in range(1, steps + 1):
        _, S = one_head(q[:n], K[:n], v[:n], a[:n], b[:n], s0=s0)
        th = 2 * n * phi
        R = np.array([[math.cos(th), -math.sin(th), 0],
                      [math.sin(th), math.cos(th), 0], [0, 0, 1]])
        np.testing.assert_allclose(S, R, atol=1e-12)
    _, Sm = one_head(q[:m], K[:m], v[:m], a[:m], b[:m], s0=s0)
    np.testing.assert_allclose(Sm, np.eye(dk), atol=1e-12)


# ------------------------------------------------ reductions (Prop. 2.1)

def test_reduction_beta_zero_is_diagonal_ssm():
    """SFDA Prop. 2.1: beta = 0 leaves S_t = diag(alpha_t) S_{t-1}, so
    o_t = S_0^T (gamma_t * q_t) with gamma_t the running product of gates."""
    rng = np.random.default_rng(7)
    T, dk, dv = 30, 5, 4
    q, k, v, a, _ = rand_head(rng, T, dk, dv, "ckda")
    s0 = rng.standard_normal((dk, dv))
    o, S = one_head(q, k, v, a, np.zeros(T), s0=s0, scale=2.0)
    gamma = np.cumprod(a, axis=0)
    np.testing.assert_allclose(o, 2.0 * (gamma * q) @ s0, atol=1e-12)
    np.testing.assert_allclose(S, gamma[-1][:, None] * s0, atol=1e-12)


def test_reduction_alpha_zero_overwrites():
    """alpha = 0 wipes the state each step, so S_t = beta_t k_t v_t^T and
    o_t = beta_t (k_t . q_t) v_t (the readout sees the updated state)."""
    rng = np.random.default_rng(8)
    T, dk, dv = 12, 4, 3
    q, k, v, _, b = rand_head(rng, T, dk, dv, "ckda")
    o, S = one_head(q, k, v, np.zeros((T, dk)), b, s0=rng.standard_normal((dk, dv)))
    want = (b * np.sum(k * q, axis=1))[:, None] * v
    np.testing.assert_allclose(o, want, atol=1e-12)
    np.testing.assert_allclose(S, b[-1] * np.outer(k[-1], v[-1]), atol=1e-12)


def test_reduction_sign_flip_gate():
    """alpha = -1, beta = 0: S_t = (-1)^t S_0."""
    rng = np.random.default_rng(9)
    T, dk, dv = 7, 3, 2
    q, k, v, _, _ = rand_head(rng, T, dk, dv, "ckda")
    s0 = rng.standard_normal((dk, dv))
    o, S = one_head(q, k, v, -np.ones((T, dk)), np.zeros(T), s0=s0)
    for t in range(T):
        np.testing.assert_allclose(o[t], (-1) ** (t + 1) * s0.T @ q[t], atol=1e-13)
    np.testing.assert_allclose(S, -s0, atol=1e-13)


def test_orthonormal_keys_exact_retrieval():
    """Delta rule with beta = 1, alpha = 1 and orthonormal keys stores each
    v_s exactly (read-compare-correct, Exercise 2): reading with q = k_s
    returns v_s, whatever S_0 held there."""
    rng = np.random.default_rng(10)
    dk, dv = 6, 3
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[:4]
    v = rng.standard_normal((4, dv))
    a = np.ones((4, dk))
    b = np.ones(4)
    s0 = rng.standard_normal((dk, dv))
    _, S = one_head(k, k, v, a, b, s0=s0)
    for s in range(4):
        np.testing.assert_allclose(S.T @ k[s], v[s], atol=1e-12)


def test_scalar_closed_form():
    """d_k = d_v = 1: S_1 = (1 - beta k^2) alpha S_0 + beta k v."""
    for a, b, kk, vv, s0 in [(0.5, 1.5, 0.8, 2.0, 3.0), (-0.7, 0.3, -1.0, 1.0, -2.0),
                             (1.0, 2.0, 1.0, 0.0, 1.0)]:
        o, S = one_head(np.array([[1.0]]), np.array([[kk]]), np.array([[vv]]),
                        np.array([[a]]), [b], s0=[[s0]])
        want = (1 - b * kk * kk) * a * s0 + b * kk * vv
        assert S[0, 0] == pytest.approx(want, abs=1e-15)
        assert o[0, 0] == pytest.approx(want, abs=1e-15)


# ------------------------------------------------ split/resume, packing, decode

def test_split_resume_and_packing():
    """State carried from one call into the next equals one call (chunk to
    chunk carry, Exercise 2; affine chunk transfer §1 contribution 4), and
    packed sequences with cu_seqlens equal separate calls."""
    rng = np.random.default_rng(12)
    dk, dv, H = 5, 4, 2
    lens = [7, 0, 13, 1]
    T = sum(lens)
    cols = [rand_head(rng, T, dk, dv, "ckda") for _ in range(H)]
    q, k, v, a, b = (np.stack([c[i] for c in cols], 1) for i in range(5))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    s0 = rng.standard_normal((len(lens), H, dk, dv))
    o, sf = oracle.fwd(q, k, v, a, b, s0, cu)
    for n, L in enumerate(lens):
        s, e = cu[n], cu[n + 1]
        for h in range(H):
            o1, S1 = one_head(q[s:e, h], k[s:e, h], v[s:e, h], a[s:e, h],
                              b[s:e, h], s0=s0[n, h])
            np.testing.assert_allclose(o[s:e, h], o1, atol=0)
            np.testing.assert_allclose(sf[n, h], S1, atol=0)
            if L >= 2:
                m = L // 2
                oa, Sa = one_head(q[s:s + m, h], k[s:s + m, h], v[s:s + m, h],
                                  a[s:s + m, h], b[s:s + m, h], s0=s0[n, h])
                ob, Sb = one_head(q[s + m:e, h], k[s + m:e, h], v[s + m:e, h],
                                  a[s + m:e, h], b[s + m:e, h], s0=Sa)
                np.testing.assert_allclose(np.concatenate([oa, ob]), o1, atol=1e-14)
                np.testing.assert_allclose(Sb, S1, atol=1e-14)
    # a zero-length sequence passes its initial state through unchanged
    np.testing.assert_array_equal(sf[1], s0[1])


def test_decode_equals_forward_tokens():
    """The decode step is the recurrence applied once per call; a run of
    decode calls equals a forward over the same tokens (and only the listed
    pairs move when a subset is stepped)."""
    rng = np.random.default_rng(13)
    N, H, dk, dv, steps = 3, 2, 4, 3, 6
    state = rng.standard_normal((N, H, dk, dv))
    s0 = state.copy()
    toks = []
    outs = []
    for _ in range(steps):
        cols = [rand_head(rng, N * H, dk, dv, "ckda")]
        q, k, v, a, b = (c.reshape(N, H, -1) if c.ndim == 2 else c.reshape(N, H)
                         for c in cols[0])
        toks.append((q, k, v, a, b))
        outs.append(oracle.decode(q, k, v, a, b, state, scale=0.5))
    for n in range(N):
        for h in range(H):
            seq = [np.stack([t[i][n, h] for t in toks]) for i in range(4)]
            bb = np.array([t[4][n, h] for t in toks])
            o1, S1 = one_head(*seq, bb, s0=s0[n, h], scale=0.5)
            np.testing.assert_allclose(np.stack([o[n, h] for o in outs]), o1,
                                       atol=1e-13)
            np.testing.assert_allclose(state[n, h], S1, atol=1e-13)
    # subset stepping leaves the other pairs alone
    st2 = s0.copy()
    q, k, v, a, b = toks[0]
    o = oracle.decode(q, k, v, a, b, st2, pairs=np.array([1, 4]))
    moved = [i for i in range(N * H)
             if not np.array_equal(st2.reshape(N * H, dk, dv)[i],
                                   s0.reshape(N * H, dk, dv)[i])]
    assert moved == [1, 4]
    assert np.all(o.reshape(N * H, dv)[[0, 2, 3, 5]] == 0)


def test_oracle_rejects_bad_cu_seqlens():
    q = np.zeros((4, 1, 2))
    v = np.zeros((4, 1, 2))
    b = np.zeros((4, 1))
    with pytest.raises(ValueError):
        oracle.fwd(q, q, v, q, b, None, np.array([0, 3], np.int32))
    with pytest.raises(RuntimeError):
        oracle.fwd(q, q, v, q, b, None, np.array([0, 3, 2, 4], np.int32))
