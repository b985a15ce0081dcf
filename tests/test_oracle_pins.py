"""Pins for the fp64 oracle: each check ties it to something other than itself.

- a worked example computed by hand (tests/golden/kda_hand_example.json);
- the linear-attention and GLA closed forms when the delta write is replaced by an additive
  write ("From GPT-2 to Kimi K3, Explained", section "Linear Attention -- 2차 비용을 선형으로");
- scalar alpha reducing to Gated DeltaNet, both through a separately written textbook GDN
  recurrence and through the rescaling identity GDN(v) = gamma * DeltaNet(v / gamma)
  ("Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "선형 어텐션에서 Gated
  DeltaNet까지");
- the delta rule's write/read property S_t^T k_t = v_t for unit keys and beta = 1
  ("From GPT-2 to Kimi K3, Explained", section "DeltaNet -- 유한한 캐시의 덮어쓰기");
- brute force in exact rational arithmetic over the unrolled product of transition matrices
  (I - beta k k^T) Diag(alpha) ("generalized Householder" transitions, same sections);
- special cases: alpha -> 0 resets the state, beta = 0 is pure channel-wise decay, and
  splitting a sequence and continuing from its state changes nothing.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_inputs(rng, T, H, dk, dv, N_state=1):
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    la = -np.exp(rng.uniform(-7.0, -0.7, (T, H, dk)))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    s0 = 0.3 * rng.standard_normal((N_state, H, dk, dv))
    return q, k, v, la, beta, s0


def test_hand_worked_example(fwd=oracle.forward):
    with open(os.path.join(GOLDEN, "kda_hand_example.json")) as f:
        ex = json.load(f)
    q = np.array(ex["q"])[:, None, :]
    k = np.array(ex["k"])[:, None, :]
    v = np.array(ex["v"])[:, None, :]
    la = np.log(np.array(ex["alpha"]))[:, None, :]
    beta = np.array(ex["beta"])[:, None]
    s0 = np.array(ex["S0"], dtype=np.float64)[None, None]
    o, sf = fwd(q, k, v, la, beta, s0)
    np.testing.assert_allclose(o[:, 0, :], np.array(ex["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(sf[0, 0], np.array(ex["S_final"]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("lengths", [[37], [11, 0, 26, 1]])
def test_linear_attention_closed_form(lengths):
    """alpha = 1 and an additive write: o_t = S0^T q_t + sum_{i<=t} v_i (k_i . q_t)."""
    rng = np.random.default_rng(1)
    T, H, dk, dv = sum(lengths), 3, 5, 4
    q, k, v, _, beta, s0 = _rand_inputs(rng, T, H, dk, dv, len(lengths))
    la = np.zeros((T, H, dk))
    cu = np.cumsum([0] + lengths)
    o, sf = oracle.forward(q, k, v, la, beta, s0, cu, rule=oracle.RULE_ADDITIVE)
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        for h in range(H):
            Q, K, V = q[a:b, h], k[a:b, h], v[a:b, h]
            L = b - a
            mask = np.tril(np.ones((L, L)))
            expect = (Q @ K.T * mask) @ V + Q @ s0[n, h]
            np.testing.assert_allclose(o[a:b, h], expect, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(sf[n, h], s0[n, h] + K.T @ V, rtol=1e-12, atol=1e-12)


def test_gla_closed_form():
    """Channel-wise decay with an additive write:
    o_t = S0^T (e^{g_t} * q_t) + sum_{i<=t} v_i ((k_i * e^{g_t - g_i}) . q_t), g_t = sum_{j<=t} a_j."""
    rng = np.random.default_rng(2)
    T, H, dk, dv = 29, 2, 6, 3
    q, k, v, la, beta, s0 = _rand_inputs(rng, T, H, dk, dv)
    o, sf = oracle.forward(q, k, v, la, beta, s0, rule=oracle.RULE_ADDITIVE)
    for h in range(H):
        g = np.cumsum(la[:, h], axis=0)  # [T, dk]
        for t in range(T):
            expect = s0[0, h].T @ (np.exp(g[t]) * q[t, h])
            for i in range(t + 1):
                expect = expect + v[i, h] * np.dot(k[i, h] * np.exp(g[t] - g[i]), q[t, h])
            np.testing.assert_allclose(o[t, h], expect, rtol=1e-11, atol=1e-12)
        S_expect = np.exp(g[-1])[:, None] * s0[0, h]
        for i in range(T):
            S_expect = S_expect + np.outer(k[i, h] * np.exp(g[-1] - g[i]), v[i, h])
        np.testing.assert_allclose(sf[0, h], S_expect, rtol=1e-11, atol=1e-12)


def _gdn_textbook(q, k, v, alpha, beta, s0):
    """Gated DeltaNet with a scalar gate, written as S_t = alpha_t (S_{t-1} - beta_t k_t (k_t^T S_{t-1}))
    + beta_t k_t v_t^T (the gate scales the whole transition), o_t = S_t^T q_t."""
    S = s0.copy()
    out = []
    for t in range(q.shape[0]):
        kt = k[t]
        S = alpha[t] * (S - beta[t] * np.outer(kt, kt @ S)) + beta[t] * np.outer(kt, v[t])
        out.append(S.T @ q[t])
    return np.array(out), S


def test_scalar_alpha_reduces_to_gated_deltanet(fwd=oracle.forward):
    rng = np.random.default_rng(3)
    T, H, dk, dv = 24, 2, 5, 4
    q, k, v, _, beta, s0 = _rand_inputs(rng, T, H, dk, dv)
    a_scalar = -np.exp(rng.uniform(-3.0, -0.7, (T, H)))  # short T keeps 1/gamma moderate
    la = np.repeat(a_scalar[:, :, None], dk, axis=2)
    o, sf = fwd(q, k, v, la, beta, s0)
    for h in range(H):
        o_ref, s_ref = _gdn_textbook(q[:, h], k[:, h], v[:, h], np.exp(a_scalar[:, h]), beta[:, h], s0[0, h])
        np.testing.assert_allclose(o[:, h], o_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sf[0, h], s_ref, rtol=1e-12, atol=1e-12)
    # rescaling identity: GDN(v) = gamma_t * DeltaNet(v / gamma_t), gamma_t = prod_{j<=t} alpha_j
    gamma = np.exp(np.cumsum(a_scalar, axis=0))  # [T, H]
    o_dn, sf_dn = fwd(q, k, v / gamma[:, :, None], np.zeros_like(la), beta, s0)
    np.testing.assert_allclose(o, gamma[:, :, None] * o_dn, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(sf[0], gamma[-1][:, None, None] * sf_dn[0], rtol=1e-9, atol=1e-12)


def test_gdn_entry_points_follow_the_textbook_recurrence():
    """oracle.gdn_forward / gdn_decode_step (scalar log_alpha [T, H]) against the separately written
    Gated DeltaNet recurrence, over two packed sequences; and the decode step against one
    textbook step."""
    rng = np.random.default_rng(13)
    T, H, dk, dv = 30, 2, 6, 3
    q, k, v, _, beta, _ = _rand_inputs(rng, T, H, dk, dv)
    a_scalar = -np.exp(rng.uniform(-4.0, -0.5, (T, H)))
    s0 = 0.3 * rng.standard_normal((2, H, dk, dv))
    cu = np.array([0, 11, T])
    o, sf = oracle.gdn_forward(q, k, v, a_scalar, beta, s0, cu)
    for n in range(2):
        a, b = cu[n], cu[n + 1]
        for h in range(H):
            o_ref, s_ref = _gdn_textbook(q[a:b, h], k[a:b, h], v[a:b, h], np.exp(a_scalar[a:b, h]), beta[a:b, h],
                                         s0[n, h])
            np.testing.assert_allclose(o[a:b, h], o_ref, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(sf[n, h], s_ref, rtol=1e-12, atol=1e-12)
    od, Sd = oracle.gdn_decode_step(q[:1].reshape(1, H, dk), k[:1].reshape(1, H, dk), v[:1].reshape(1, H, dv),
                                    a_scalar[:1], beta[:1], s0[:1])
    for h in range(H):
        o_ref, s_ref = _gdn_textbook(q[:1, h], k[:1, h], v[:1, h], np.exp(a_scalar[:1, h]), beta[:1, h], s0[0, h])
        np.testing.assert_allclose(od[0, h], o_ref[0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(Sd[0, h], s_ref, rtol=1e-12, atol=1e-12)


def test_write_read_invariant(fwd=oracle.forward):
    """With ||k_t|| = 1 and beta_t = 1 the state returns v_t for key k_t right after the write."""
    rng = np.random.default_rng(4)
    T, H, dk, dv = 40, 2, 8, 5
    q, k, v, la, _, s0 = _rand_inputs(rng, T, H, dk, dv)
    beta = np.ones((T, H))
    S = s0
    for t in range(T):
        _, S = fwd(q[t:t + 1], k[t:t + 1], v[t:t + 1], la[t:t + 1], beta[t:t + 1], S)
        for h in range(H):
            read = S[0, h].T @ k[t, h]
            assert np.linalg.norm(read - v[t, h]) <= 1e-12 * np.linalg.norm(v[t, h])


def _frac_vec(xs):
    return [Fraction(x) for x in xs]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_transition_product(seed, fwd=oracle.forward):
    """S_T = (prod_{j=T..1} M_j) S0 + sum_i (prod_{j=T..i+1} M_j) beta_i k_i v_i^T with
    M_j = (I - beta_j k_j k_j^T) Diag(alpha_j), in exact rationals over dyadic inputs."""
    rng = np.random.default_rng(100 + seed)
    T, dk, dv = 6, 4, 3

    def dy(shape, lo=-8, hi=8, den=8):
        return rng.integers(lo, hi + 1, size=shape) / den

    q, k, v = dy((T, dk)), dy((T, dk)), dy((T, dv))
    alpha = rng.integers(1, 8, size=(T, dk)) / 8.0        # exact dyadics in (0, 1)
    beta = rng.integers(1, 8, size=T) / 8.0
    s0 = dy((dk, dv), -4, 4, 16)

    I = [[Fraction(int(i == j)) for j in range(dk)] for i in range(dk)]

    def matmul(A, B):
        return [[sum((A[i][m] * B[m][j] for m in range(len(B))), Fraction(0)) for j in range(len(B[0]))]
                for i in range(len(A))]

    def M(j):
        kj = _frac_vec(k[j]); aj = _frac_vec(alpha[j]); bj = Fraction(beta[j])
        return [[(I[r][c] - bj * kj[r] * kj[c]) * aj[c] for c in range(dk)] for r in range(dk)]

    Ms = [M(j) for j in range(T)]
    S0 = [_frac_vec(row) for row in s0]
    o_exact = []
    for t in range(T):  # state after token t: unrolled products, nothing shared across t
        P = I
        for j in range(t, -1, -1):
            P = matmul(P, Ms[j])
        S = matmul(P, S0)
        for i in range(t + 1):
            Pi = I
            for j in range(t, i, -1):
                Pi = matmul(Pi, Ms[j])
            ki = _frac_vec(k[i]); vi = _frac_vec(v[i]); bi = Fraction(beta[i])
            outer = [[bi * ki[r] * vi[c] for c in range(dv)] for r in range(dk)]
            add = matmul(Pi, outer)
            S = [[S[r][c] + add[r][c] for c in range(dv)] for r in range(dk)]
        qt = _frac_vec(q[t])
        o_exact.append([float(sum((S[r][c] * qt[r] for r in range(dk)), Fraction(0))) for c in range(dv)])
    S_exact = np.array([[float(x) for x in row] for row in S])

    o, sf = fwd(q[:, None], k[:, None], v[:, None], np.log(alpha)[:, None], beta[:, None], s0[None, None])
    # log(alpha) then exp() in the oracle costs a few ulp per factor
    np.testing.assert_allclose(o[:, 0], np.array(o_exact), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sf[0, 0], S_exact, rtol=1e-12, atol=1e-13)


def test_alpha_to_zero_resets_state():
    rng = np.random.default_rng(5)
    T, H, dk, dv = 9, 2, 4, 3
    q, k, v, _, beta, s0 = _rand_inputs(rng, T, H, dk, dv)
    la = np.full((T, H, dk), -1e4)  # exp underflows to exactly 0
    o, sf = oracle.forward(q, k, v, la, beta, s0)
    for t in range(T):
        for h in range(H):
            S_t = beta[t, h] * np.outer(k[t, h], v[t, h])
            np.testing.assert_allclose(o[t, h], S_t.T @ q[t, h], rtol=1e-13, atol=1e-14)
    for h in range(H):
        np.testing.assert_allclose(sf[0, h], beta[-1, h] * np.outer(k[-1, h], v[-1, h]), rtol=1e-13, atol=1e-14)


def test_beta_zero_is_pure_channel_decay():
    rng = np.random.default_rng(6)
    T, H, dk, dv = 17, 2, 6, 5
    q, k, v, la, _, s0 = _rand_inputs(rng, T, H, dk, dv)
    beta = np.zeros((T, H))
    o, sf = oracle.forward(q, k, v, la, beta, s0)
    for h in range(H):
        g = np.cumsum(la[:, h], axis=0)
        for t in range(T):
            S_t = np.exp(g[t])[:, None] * s0[0, h]
            np.testing.assert_allclose(o[t, h], S_t.T @ q[t, h], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(sf[0, h], np.exp(g[-1])[:, None] * s0[0, h], rtol=1e-12, atol=1e-14)


def test_split_continuation_is_bit_identical():
    rng = np.random.default_rng(7)
    T, H, dk, dv = 50, 2, 8, 6
    q, k, v, la, beta, s0 = _rand_inputs(rng, T, H, dk, dv)
    o, sf = oracle.forward(q, k, v, la, beta, s0)
    cut = 19
    o1, s1 = oracle.forward(q[:cut], k[:cut], v[:cut], la[:cut], beta[:cut], s0)
    o2, s2 = oracle.forward(q[cut:], k[cut:], v[cut:], la[cut:], beta[cut:], s1)
    assert np.array_equal(np.concatenate([o1, o2]), o)
    assert np.array_equal(s2, sf)


def test_varlen_packing_equals_separate_calls():
    rng = np.random.default_rng(8)
    lengths = [5, 0, 12, 1, 7]
    T, H, dk, dv = sum(lengths), 2, 4, 3
    q, k, v, la, beta, s0 = _rand_inputs(rng, T, H, dk, dv, len(lengths))
    cu = np.cumsum([0] + lengths)
    o, sf = oracle.forward(q, k, v, la, beta, s0, cu)
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        on, sn = oracle.forward(q[a:b], k[a:b], v[a:b], la[a:b], beta[a:b], s0[n:n + 1])
        assert np.array_equal(on, o[a:b])
        assert np.array_equal(sn[0], sf[n])
    # a length-0 sequence passes its state through
    assert np.array_equal(sf[1], s0[1])


def test_decode_step_equals_length_one_forward():
    rng = np.random.default_rng(9)
    B, H, dk, dv = 3, 2, 5, 4
    q, k, v, la, beta, _ = _rand_inputs(rng, B, H, dk, dv)
    S = 0.1 * rng.standard_normal((B, H, dk, dv))
    o_d, S_d = oracle.decode_step(q, k, v, la, beta, S)
    o_f, S_f = oracle.forward(q, k, v, la, beta, S, np.arange(B + 1))
    assert np.array_equal(o_d, o_f)
    assert np.array_equal(S_d, S_f)


def test_invalid_arguments_are_rejected():
    rng = np.random.default_rng(10)
    q, k, v, la, beta, s0 = _rand_inputs(rng, 4, 1, 2, 2)
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, la, beta, None, np.array([0, 3, 2, 4]))
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, la, beta, None, np.array([0, 5]))


# ---------------------------------------------------------------- the fused prologue's definitions

def test_l2norm_option_is_invariant_to_positive_row_scales_and_fixes_unit_rows():
    """l2norm_qk=True: rescaling each (token, head) vector of q and k by a positive factor changes
    nothing (a normalisation over any other axis would change), and rows that already have unit length
    (Pythagorean-triple rows such as (3/5, 4/5)) give what they give with the option off; an all-zero
    query row gives a zero output row."""
    rng = np.random.default_rng(21)
    T, H, dk, dv = 17, 2, 6, 3
    q, k, v, la, beta, s0 = _rand_inputs(rng, T, H, dk, dv)
    k = rng.standard_normal((T, H, dk))
    a = np.exp(rng.uniform(-2, 2, (T, H, 1)))
    b = np.exp(rng.uniform(-2, 2, (T, H, 1)))
    o1, s1 = oracle.forward(q, k, v, la, beta, s0, l2norm_qk=True)
    o2, s2 = oracle.forward(q * a, k * b, v, la, beta, s0, l2norm_qk=True)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s2, s1, rtol=1e-12, atol=1e-13)
    # unit rows: (3/5, 4/5) and (5/13, 12/13) placed in random channel pairs
    qu, ku = np.zeros((T, H, dk)), np.zeros((T, H, dk))
    for t in range(T):
        for h in range(H):
            i, j = rng.choice(dk, 2, replace=False)
            qu[t, h, i], qu[t, h, j] = 0.6, 0.8
            i, j = rng.choice(dk, 2, replace=False)
            ku[t, h, i], ku[t, h, j] = 5 / 13, 12 / 13
    o3, s3 = oracle.forward(qu, ku, v, la, beta, s0, l2norm_qk=True)
    o4, s4 = oracle.forward(qu, ku, v, la, beta, s0)
    np.testing.assert_allclose(o3, o4, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(s3, s4, rtol=1e-14, atol=1e-15)
    q0 = q.copy()
    q0[5, 1] = 0.0
    o5, _ = oracle.forward(q0, k, v, la, beta, s0, l2norm_qk=True)
    assert np.all(o5[5, 1] == 0.0)


def test_beta_logits_option_is_the_logistic_function():
    """beta_logits=True: logit 0 is beta = 1/2 exactly, and logits log(b / (1 - b)) reproduce the run
    with beta = b (the inverse of the logistic function)."""
    rng = np.random.default_rng(22)
    T, H, dk, dv = 15, 2, 5, 4
    q, k, v, la, beta, s0 = _rand_inputs(rng, T, H, dk, dv)
    o1, s1 = oracle.forward(q, k, v, la, np.zeros((T, H)), s0, beta_logits=True)
    o2, s2 = oracle.forward(q, k, v, la, np.full((T, H), 0.5), s0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)
    o3, s3 = oracle.forward(q, k, v, la, np.log(beta / (1 - beta)), s0, beta_logits=True)
    o4, s4 = oracle.forward(q, k, v, la, beta, s0)
    np.testing.assert_allclose(o3, o4, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s3, s4, rtol=1e-12, atol=1e-13)
    # decode: the same options on one step
    od1, Sd1 = oracle.decode_step(q[:1], k[:1], v[:1], la[:1], np.zeros((1, H)), s0, beta_logits=True,
                                  l2norm_qk=True)
    od2, Sd2 = oracle.decode_step(oracle.l2_normalise(q[:1]), oracle.l2_normalise(k[:1]), v[:1], la[:1],
                                  np.full((1, H), 0.5), s0)
    np.testing.assert_array_equal(od1, od2)
    np.testing.assert_array_equal(Sd1, Sd2)


def test_output_epilogue_is_a_per_head_rms_norm_and_gate():
    """epilogue=(gate, w, eps): with eps = 0 scaling v and S0 by c > 0 (which scales o by c) changes
    nothing; gate 0 halves, so 2 o' / w has unit root-mean-square over the dv values of every (token,
    head) row -- a norm over any other axis, a sum for the mean or a different activation fails."""
    rng = np.random.default_rng(23)
    T, H, dk, dv = 13, 3, 5, 6
    q, k, v, la, beta, s0 = _rand_inputs(rng, T, H, dk, dv)
    gate = rng.standard_normal((T, H, dv))
    w = np.exp(rng.uniform(-1, 1, dv))
    o1, _ = oracle.forward(q, k, v, la, beta, s0, epilogue=(gate, w, 0.0))
    o2, _ = oracle.forward(q, k, 7.5 * v, la, beta, 7.5 * s0, epilogue=(gate, w, 0.0))
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    o3, _ = oracle.forward(q, k, v, la, beta, s0, epilogue=(np.zeros((T, H, dv)), w, 0.0))
    np.testing.assert_allclose(np.sqrt(np.mean((2 * o3 / w) ** 2, axis=-1)), 1.0, rtol=1e-13)
    # eps: rows scaled so that mean(o^2) = m get exactly sqrt(m / (m + eps)) of the eps = 0 result
    o_raw, _ = oracle.forward(q, k, v, la, beta, s0)
    m = np.mean(o_raw ** 2, axis=-1, keepdims=True)
    o4, _ = oracle.forward(q, k, v, la, beta, s0, epilogue=(gate, w, 0.25))
    np.testing.assert_allclose(o4, o1 * np.sqrt(m / (m + 0.25)), rtol=1e-12, atol=1e-14)
    od, _ = oracle.decode_step(q[:1], k[:1], v[:1], la[:1], beta[:1], s0, epilogue=(gate[:1], w, 0.0))
    od_raw, _ = oracle.decode_step(q[:1], k[:1], v[:1], la[:1], beta[:1], s0)
    np.testing.assert_allclose(np.sqrt(np.mean((od / (w * oracle.sigmoid(gate[:1]))) ** 2, axis=-1)), 1.0,
                               rtol=1e-13)
    assert np.all(np.sign(od) == np.sign(od_raw))
