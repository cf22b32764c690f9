"""Pins of the fp64 oracle to facts the pages and the mathematics fix (no GPU needed).

Each test names the passage of "Kimi Linear: An Expressive, Efficient Attention Architecture"
it relies on. A plausible slip in the oracle — a dropped term, a wrong sign, a transposed operand,
decay on the wrong axis, reading S_{t-1} instead of S_t, an off-by-one in the chunk decay — fails
at least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle
from gated_delta_rule_120_b200 import roofline

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_inputs(rng, T, H, Dk, Dv, decay_scale=0.5, unit_keys=True):
    q = rng.standard_normal((T, H, Dk))
    k = rng.standard_normal((T, H, Dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, Dv))
    la = -np.log1p(np.exp(rng.standard_normal((T, H, Dk)))) * decay_scale
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    return q, k, v, la, beta


# --- P1: alpha = 1, beta = 0 leaves S constant and o_t = S_0^T q_t (Eq. 1, output read) -------
def test_identity_transition_reads_initial_state():
    rng = np.random.default_rng(1)
    T, H, Dk, Dv = 9, 2, 5, 3  # Dk != Dv and a non-symmetric S_0 catch transposes
    q, k, v, _, _ = _rand_inputs(rng, T, H, Dk, Dv)
    la = np.zeros((T, H, Dk))
    beta = np.zeros((T, H))
    S0 = rng.standard_normal((1, H, Dk, Dv))
    o, S = oracle.recurrent(q, k, v, la, beta, S0)
    assert np.array_equal(S, S0)
    expect = np.einsum("hkv,thk->thv", S0[0], q)
    np.testing.assert_allclose(o, expect, rtol=0, atol=1e-14)


# --- P2: beta = 0 is pure per-channel decay: S_t = Diag(prod alpha) S_0 (Eq. 1 with no write) --
def test_pure_decay_closed_form():
    rng = np.random.default_rng(2)
    T, H, Dk, Dv = 11, 3, 6, 4
    q, k, v, la, _ = _rand_inputs(rng, T, H, Dk, Dv)
    beta = np.zeros((T, H))
    S0 = rng.standard_normal((1, H, Dk, Dv))
    o, S = oracle.recurrent(q, k, v, la, beta, S0)
    g = np.cumsum(la, axis=0)  # [T,H,Dk] cumulative log decay
    expect_S = np.exp(g[-1])[:, :, None] * S0[0]
    np.testing.assert_allclose(S[0], expect_S, rtol=1e-13, atol=0)
    # o_t = S_t^T q_t with S_t = Diag(exp(g_t)) S_0: decay acts on key channels (rows)
    expect_o = np.einsum("hkv,thk->thv", S0[0], np.exp(g) * q)
    np.testing.assert_allclose(o, expect_o, rtol=1e-12, atol=1e-14)


def test_scalar_decay_is_geometric():
    """A scalar alpha_t (same on every channel) with beta = 0 gives S_t = alpha_t S_{t-1}."""
    rng = np.random.default_rng(3)
    T, H, Dk, Dv = 7, 1, 4, 4
    q, k, v, _, _ = _rand_inputs(rng, T, H, Dk, Dv)
    a = rng.uniform(0.3, 1.0, size=T)
    la = np.repeat(np.log(a)[:, None, None], Dk, axis=2)
    S0 = rng.standard_normal((1, H, Dk, Dv))
    for t in range(1, T + 1):
        _, S = oracle.recurrent(q[:t], k[:t], v[:t], la[:t], np.zeros((t, H)), S0)
        np.testing.assert_allclose(S, np.prod(a[:t]) * S0, rtol=1e-13)


# --- P3: alpha = 1, beta = 1, orthonormal keys => exact key -> value retrieval ----------------
def test_orthonormal_keys_retrieve_exactly():
    rng = np.random.default_rng(4)
    Dk, Dv, T, H = 8, 5, 6, 1
    Qm, _ = np.linalg.qr(rng.standard_normal((Dk, Dk)))
    keys = Qm[:, :T].T  # T orthonormal rows
    k = keys[:, None, :]
    v = rng.standard_normal((T, H, Dv))
    la = np.zeros((T, H, Dk))
    beta = np.ones((T, H))
    # query at step t = key of an earlier (or the same) step i(t)
    pick = [0, 1, 0, 2, 4, 5]
    q = keys[pick][:, None, :]
    o, S = oracle.recurrent(q, k, v, la, beta)
    for i in range(T):
        np.testing.assert_allclose(S[0, 0].T @ keys[i], v[i, 0], atol=1e-12)
    for t, i in enumerate(pick):
        # o_t uses the UPDATED state S_t (i == t must already see v_t)
        np.testing.assert_allclose(o[t, 0], v[i, 0], atol=1e-12)


def test_delta_rule_overwrites_same_key():
    """Writing (k, v1, b1) then (k, v2, b2) with ||k|| = 1 and alpha = 1 leaves
    S^T k = (1 - b2) b1 v1 + b2 v2 — the erase term of the delta rule with the right sign."""
    rng = np.random.default_rng(5)
    Dk, Dv = 6, 3
    kk = rng.standard_normal(Dk)
    kk /= np.linalg.norm(kk)
    k = np.stack([kk, kk])[:, None, :]
    v = rng.standard_normal((2, 1, Dv))
    b1, b2 = 0.7, 0.4
    beta = np.array([[b1], [b2]])
    q = k.copy()
    o, S = oracle.recurrent(q, k, v, np.zeros((2, 1, Dk)), beta)
    np.testing.assert_allclose(o[0, 0], b1 * v[0, 0], atol=1e-13)
    np.testing.assert_allclose(S[0, 0].T @ kk, (1 - b2) * b1 * v[0, 0] + b2 * v[1, 0], atol=1e-13)
    _, S1 = oracle.recurrent(q, k, v, np.zeros((2, 1, Dk)), np.ones((2, 1)))
    np.testing.assert_allclose(S1[0, 0].T @ kk, v[1, 0], atol=1e-13)  # beta = 1: full overwrite


# --- P4: a channel-uniform alpha reduces KDA to Gated DeltaNet ---------------------------------
def test_uniform_alpha_equals_gated_deltanet():
    """Gated DeltaNet (walkthrough §3.4 "Why this form"): S_t = a_t (I - b k k^T) S + b k v^T.
    KDA with Diag(alpha) = a_t I must give the same states: the decay multiplies the old state
    but not the new write."""
    rng = np.random.default_rng(6)
    T, Dk, Dv = 13, 5, 4
    q, k, v, _, beta = _rand_inputs(rng, T, 1, Dk, Dv)
    a = rng.uniform(0.5, 1.0, size=T)
    la = np.repeat(np.log(a)[:, None, None], Dk, axis=2)
    S0 = rng.standard_normal((1, 1, Dk, Dv))
    o, S = oracle.recurrent(q, k, v, la, beta, S0)
    St = S0[0, 0].copy()
    for t in range(T):
        kt, vt, bt = k[t, 0], v[t, 0], beta[t, 0]
        St = a[t] * (St - bt * np.outer(kt, kt @ St)) + bt * np.outer(kt, vt)
        np.testing.assert_allclose(o[t, 0], St.T @ q[t, 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S[0, 0], St, rtol=1e-12, atol=1e-13)


# --- brute force: explicit d_k x d_k transition products on tiny inputs -----------------------
def test_transition_matrix_product_brute_force():
    """S_T = P S_0 + H with P = prod_t (I - b_t k_t k_t^T) Diag(alpha_t) and
    H = sum_i (prod_{j>i} ...) b_i k_i v_i^T (walkthrough §3.4, intra-chunk unrolling),
    evaluated with explicit matrices."""
    rng = np.random.default_rng(7)
    T, Dk, Dv = 10, 4, 3
    q, k, v, la, beta = _rand_inputs(rng, T, 1, Dk, Dv, unit_keys=False)
    S0 = rng.standard_normal((1, 1, Dk, Dv))
    _, S = oracle.recurrent(q, k, v, la, beta, S0)
    mats = [(np.eye(Dk) - beta[t, 0] * np.outer(k[t, 0], k[t, 0])) @ np.diag(np.exp(la[t, 0]))
            for t in range(T)]
    P = np.eye(Dk)
    for t in range(T):
        P = mats[t] @ P
    Hm = np.zeros((Dk, Dv))
    for i in range(T):
        G = np.eye(Dk)
        for j in range(i + 1, T):
            G = mats[j] @ G
        Hm += G @ (beta[i, 0] * np.outer(k[i, 0], v[i, 0]))
    np.testing.assert_allclose(S[0, 0], P @ S0[0, 0] + Hm, rtol=1e-11, atol=1e-12)


# --- P5: chunk / call boundary: S at the end of one segment starts the next -------------------
def test_state_handoff_between_calls():
    rng = np.random.default_rng(8)
    T, H, Dk, Dv = 37, 2, 6, 5
    q, k, v, la, beta = _rand_inputs(rng, T, H, Dk, Dv)
    S0 = rng.standard_normal((1, H, Dk, Dv)) * 0.1
    o, S = oracle.recurrent(q, k, v, la, beta, S0)
    for cut in (1, 16, 23, 36):
        o1, S1 = oracle.recurrent(q[:cut], k[:cut], v[:cut], la[:cut], beta[:cut], S0)
        o2, S2 = oracle.recurrent(q[cut:], k[cut:], v[cut:], la[cut:], beta[cut:], S1)
        np.testing.assert_allclose(np.concatenate([o1, o2]), o, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(S2, S, rtol=1e-12, atol=1e-13)
        # the chunked form across the same cut
        o3, S3 = oracle.chunked(q[:cut], k[:cut], v[:cut], la[:cut], beta[:cut], S0, chunk=16)
        o4, S4 = oracle.chunked(q[cut:], k[cut:], v[cut:], la[cut:], beta[cut:], S3, chunk=16)
        np.testing.assert_allclose(S4, S, rtol=1e-11, atol=1e-12)


# --- P6: the chunkwise WY/UT form (Eq. 8/9) equals the recurrence -----------------------------
@pytest.mark.parametrize("C", [1, 4, 16, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 150])
def test_chunked_equals_recurrent(C, T):
    rng = np.random.default_rng(100 + C * 7 + T)
    H, Dk, Dv = 2, 16, 12
    q, k, v, la, beta = _rand_inputs(rng, T, H, Dk, Dv)
    S0 = rng.standard_normal((1, H, Dk, Dv)) * 0.05
    o_r, S_r = oracle.recurrent(q, k, v, la, beta, S0)
    o_c, S_c = oracle.chunked(q, k, v, la, beta, S0, chunk=C)
    scale_o = np.abs(o_r).max()
    scale_s = np.abs(S_r).max()
    assert np.abs(o_c - o_r).max() <= 1e-12 * scale_o
    assert np.abs(S_c - S_r).max() <= 1e-12 * scale_s


def test_chunked_equals_recurrent_varlen_and_strong_decay():
    rng = np.random.default_rng(11)
    lens = [5, 0, 64, 70, 1, 129]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, Dk, Dv = int(cu[-1]), 3, 8, 8
    q, k, v, la, beta = _rand_inputs(rng, T, H, Dk, Dv, decay_scale=3.0)
    S0 = rng.standard_normal((len(lens), H, Dk, Dv))
    o_r, S_r = oracle.recurrent(q, k, v, la, beta, S0, cu_seqlens=cu)
    o_c, S_c = oracle.chunked(q, k, v, la, beta, S0, cu_seqlens=cu, chunk=64)
    np.testing.assert_allclose(o_c, o_r, rtol=0, atol=1e-12 * np.abs(o_r).max())
    np.testing.assert_allclose(S_c, S_r, rtol=0, atol=1e-12 * np.abs(S_r).max())
    # the empty sequence keeps its initial state
    np.testing.assert_array_equal(S_r[1], S0[1])


def test_chunk_decay_index_reading():
    """Eq. 8 with the decay Gamma_{i->C} taken INCLUSIVE of position i (the product printed from
    j = i) disagrees with the recurrence; the exclusive reading used by the oracle agrees. This
    pins the reading of the garbled index."""
    rng = np.random.default_rng(12)
    T, Dk, Dv, C = 8, 4, 3, 8
    q, k, v, la, beta = _rand_inputs(rng, T, 1, Dk, Dv)
    _, S_r = oracle.recurrent(q, k, v, la, beta)
    g = np.cumsum(la[:, 0], axis=0)
    K = k[:, 0]
    A = np.tril(beta[:, 0][:, None] * ((np.exp(g) * K) @ (K * np.exp(-g)).T), -1)
    M = np.linalg.inv(np.eye(C) + A) * beta[:, 0][None, :]
    Wm, Um = M @ (np.exp(g) * K), M @ v[:, 0]
    excl = (np.exp(g[-1] - g) * K).T @ Um  # S_0 = 0, so V' = U
    incl = (np.exp(g[-1] - g + la[:, 0]) * K).T @ Um
    np.testing.assert_allclose(excl, S_r[0, 0], rtol=1e-12, atol=1e-13)
    assert np.abs(incl - S_r[0, 0]).max() > 1e-3
    del Wm


# --- P7: forward-substitution inverse equals a textbook dense inverse --------------------------
@pytest.mark.parametrize("C", [1, 2, 16, 64])
def test_unit_lower_inverse(C):
    rng = np.random.default_rng(200 + C)
    A = rng.standard_normal((C, C)) * 0.3
    X = oracle.unit_lower_inverse(A)
    ref = np.linalg.inv(np.eye(C) + np.tril(A, -1))
    np.testing.assert_allclose(X, ref, rtol=1e-10, atol=1e-12)
    assert np.array_equal(np.triu(X, 1), np.zeros((C, C)))


# --- P8: structure ---------------------------------------------------------------------------
def test_value_columns_are_independent():
    """Column j of S and o depends only on column j of v and S_0 (Eq. 1 mixes key channels only)."""
    rng = np.random.default_rng(13)
    T, H, Dk, Dv = 20, 2, 7, 6
    q, k, v, la, beta = _rand_inputs(rng, T, H, Dk, Dv)
    S0 = rng.standard_normal((1, H, Dk, Dv))
    o, S = oracle.recurrent(q, k, v, la, beta, S0)
    o_a, S_a = oracle.recurrent(q, k, v[..., :2], la, beta, S0[..., :2])
    o_b, S_b = oracle.recurrent(q, k, v[..., 2:], la, beta, S0[..., 2:])
    np.testing.assert_array_equal(np.concatenate([o_a, o_b], -1), o)
    np.testing.assert_array_equal(np.concatenate([S_a, S_b], -1), S)


def test_linear_in_values_and_state():
    """For fixed q, k, alpha, beta the map (v, S_0) -> (o, S_T) is linear (Eq. 1 is affine in S
    and the write is linear in v)."""
    rng = np.random.default_rng(14)
    T, H, Dk, Dv = 25, 1, 6, 5
    q, k, v1, la, beta = _rand_inputs(rng, T, H, Dk, Dv)
    v2 = rng.standard_normal(v1.shape)
    S1 = rng.standard_normal((1, H, Dk, Dv))
    S2 = rng.standard_normal((1, H, Dk, Dv))
    oa, Sa = oracle.recurrent(q, k, v1, la, beta, S1)
    ob, Sb = oracle.recurrent(q, k, v2, la, beta, S2)
    oc, Sc = oracle.recurrent(q, k, v1 - 2.5 * v2, la, beta, S1 - 2.5 * S2)
    np.testing.assert_allclose(oc, oa - 2.5 * ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Sc, Sa - 2.5 * Sb, rtol=1e-12, atol=1e-12)


def test_norm_bound_without_decay():
    """alpha = 1, beta in [0,1], ||k|| = 1: (I - b k k^T) is a contraction, so
    ||S_T||_F <= ||S_0||_F + sum_t b_t ||v_t||."""
    rng = np.random.default_rng(15)
    T, H, Dk, Dv = 200, 1, 8, 8
    q, k, v, _, beta = _rand_inputs(rng, T, H, Dk, Dv)
    S0 = rng.standard_normal((1, H, Dk, Dv))
    _, S = oracle.recurrent(q, k, v, np.zeros((T, H, Dk)), beta, S0)
    bound = np.linalg.norm(S0) + np.sum(beta[:, 0] * np.linalg.norm(v[:, 0], axis=-1))
    assert np.linalg.norm(S) <= bound


# --- P9: the Eq. 13 FLOP counter against the page's worked example ----------------------------
def test_eq13_flops_golden():
    with open(os.path.join(GOLDEN, "eq13_flops_example.json")) as f:
        gold = json.load(f)
    T, C, d = gold["T"], gold["C"], gold["d"]
    total = roofline.eq13_flops(T, C, d)
    assert total == 6 * 4096 * 128 * 128 + 3 * 4096 * 64 * 128 + 4096 * 64 * 64
    assert total == gold["exact_total"]
    # the page prints each term and the total rounded to the nearest few million
    terms = {"6Td^2": 6 * T * d * d, "3TCd": 3 * T * C * d, "TC^2": T * C * C}
    for name, val in terms.items():
        assert abs(val - gold["printed_terms_approx"][name]) <= 0.02 * val
    assert abs(sum(terms.values()) - total) == 0
    assert abs(total - gold["printed_total_approx"]) <= 0.01 * total
    assert 128 * 128 == gold["state_elements_per_head"]


# --- fused prologue: in-kernel L2 norm and the log-space decay gate ---------------------------
def test_prologue_gate_closed_forms():
    """softplus(0) = ln 2: with g = -dt_bias the decay is exactly -exp(A_log) * ln 2; a very
    negative pre-activation gives no decay; a large one gives log alpha ~ -exp(A_log) * x."""
    H, Dk = 3, 5
    A_log = np.log(np.array([1.0, 4.0, 16.0]))
    bias = np.linspace(-1, 1, H * Dk).reshape(H, Dk)
    q = np.ones((2, H, Dk))
    _, _, la = oracle.prologue(q, q, -bias[None].repeat(2, 0), A_log=A_log, dt_bias=bias)
    np.testing.assert_allclose(la, -np.exp(A_log)[None, :, None] * np.log(2.0) * np.ones_like(la),
                               rtol=1e-14)
    _, _, la = oracle.prologue(q, q, np.full((1, H, Dk), -60.0), A_log=A_log)
    assert np.all(la <= 0) and np.abs(la).max() < 1e-20
    _, _, la = oracle.prologue(q, q, np.full((1, H, Dk), 50.0), A_log=A_log)
    np.testing.assert_allclose(la, -np.exp(A_log)[None, :, None] * 50.0 * np.ones_like(la),
                               rtol=1e-12)


def test_prologue_l2norm_makes_the_operator_scale_invariant():
    """With in-kernel normalisation, positive rescaling of a token's q or k changes nothing, and
    the normalised keys have unit norm (up to eps)."""
    rng = np.random.default_rng(31)
    T, H, Dk, Dv = 12, 2, 8, 4
    q, k, v, la, beta = _rand_inputs(rng, T, H, Dk, Dv, unit_keys=False)
    s = rng.uniform(0.1, 10.0, size=(T, H, 1))
    q1, k1, _ = oracle.prologue(q, k, la, qk_l2norm=True, eps=0.0)
    q2, k2, _ = oracle.prologue(q * s, k * s[::-1], la, qk_l2norm=True, eps=0.0)
    np.testing.assert_allclose(np.linalg.norm(k1, axis=-1), 1.0, rtol=1e-14)
    o1, S1 = oracle.recurrent(q1, k1, v, la, beta)
    o2, S2 = oracle.recurrent(q2, k2, v, la, beta)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, S1, rtol=1e-12, atol=1e-13)


def test_output_norm_gate_worked_example():
    """o = (3, 4): mean square 12.5, RMS 5/sqrt(2) = 3.5355339..., so the normalised row is
    (0.8485281374, 1.1313708499) (= 3 sqrt(2)/5, 4 sqrt(2)/5); a zero gate halves it (sigmoid(0) =
    1/2) and the weight scales channel by channel."""
    y = oracle.output_norm_gate(np.array([[3.0, 4.0]]), eps=0.0)
    np.testing.assert_allclose(y, [[0.8485281374238570, 1.1313708498984760]], rtol=1e-14)
    y = oracle.output_norm_gate(np.array([[3.0, 4.0]]), gate=np.zeros((1, 2)),
                                weight=np.array([2.0, -1.0]), eps=0.0)
    np.testing.assert_allclose(y, [[0.8485281374238570, -0.5656854249492380]], rtol=1e-14)
    # eps enters under the square root: o = (1, 1), eps = 3 -> 1 / sqrt(1 + 3) = 1/2
    y = oracle.output_norm_gate(np.array([[1.0, 1.0]]), eps=3.0)
    np.testing.assert_allclose(y, [[0.5, 0.5]], rtol=1e-15)


def test_output_norm_gate_structure():
    """The RMS is per (token, head) row over the value channels: every row of the ungated output
    has unit RMS, positive rescaling of a row changes nothing, rows do not mix; a saturated gate
    passes the row through and a very negative one closes it."""
    rng = np.random.default_rng(41)
    o = rng.normal(size=(5, 3, 16)) * rng.uniform(0.01, 100.0, size=(5, 3, 1))
    y = oracle.output_norm_gate(o, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-13)
    s = rng.uniform(0.1, 10.0, size=(5, 3, 1))
    np.testing.assert_allclose(oracle.output_norm_gate(o * s, eps=0.0), y, rtol=1e-13)
    o2 = o.copy()
    o2[2, 1] *= -7.0
    y2 = oracle.output_norm_gate(o2, eps=0.0)
    mask = np.ones((5, 3), bool)
    mask[2, 1] = False
    np.testing.assert_array_equal(y2[mask], y[mask])
    np.testing.assert_allclose(y2[2, 1], -y[2, 1], rtol=1e-13)
    g_open = oracle.output_norm_gate(o, gate=np.full(o.shape, 40.0), eps=0.0)
    np.testing.assert_allclose(g_open, y, rtol=1e-15)
    g_shut = oracle.output_norm_gate(o, gate=np.full(o.shape, -800.0), eps=0.0)
    assert np.all(np.abs(g_shut) < 1e-300)


# --- backward pass: reverse-mode derivative of the recurrence ---------------------------------
def _loss(x, cu, d_o, d_fin):
    o, S = oracle.recurrent(x["q"], x["k"], x["v"], x["la"], x["beta"], x["s0"], cu_seqlens=cu)
    return float(np.sum(o * d_o) + np.sum(S * d_fin))


def _bwd_case(seed, lens, H, Dk, Dv):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    q, k, v, la, beta = _rand_inputs(rng, T, H, Dk, Dv, unit_keys=False)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    s0 = rng.standard_normal((len(lens), H, Dk, Dv))
    x = dict(q=q, k=k, v=v, la=la, beta=beta, s0=s0)
    d_o = rng.standard_normal((T, H, Dv))
    d_fin = rng.standard_normal((len(lens), H, Dk, Dv))
    g = oracle.recurrent_bwd(q, k, v, la, beta, d_o, initial_state=s0, d_final=d_fin,
                             cu_seqlens=cu)
    return x, cu, d_o, d_fin, dict(zip(("q", "k", "v", "la", "beta", "s0"), g))


def _central_difference(x, cu, d_o, d_fin, name, idx, h=1e-6):
    xp = {n: a.copy() for n, a in x.items()}
    xp[name][idx] += h
    lp = _loss(xp, cu, d_o, d_fin)
    xp[name][idx] -= 2 * h
    lm = _loss(xp, cu, d_o, d_fin)
    return (lp - lm) / (2 * h)


def test_backward_matches_finite_differences_everywhere():
    """Every partial derivative of <d_o, o> + <d_final, S_T> (q, k, v, log alpha, beta, S_0) on
    two short sequences equals its central finite difference; Dk != Dv catches transposes."""
    x, cu, d_o, d_fin, g = _bwd_case(51, [4, 3], 2, 3, 2)
    for name in ("q", "k", "v", "la", "beta", "s0"):
        for idx in np.ndindex(*x[name].shape):
            fd = _central_difference(x, cu, d_o, d_fin, name, idx)
            assert abs(fd - g[name][idx]) <= 1e-7 * max(1.0, abs(fd)), (name, idx, fd,
                                                                        g[name][idx])


def test_backward_across_recompute_segments():
    """A 75-token sequence crosses the oracle's 32-token recompute segments; sampled partial
    derivatives in every segment equal their finite differences."""
    x, cu, d_o, d_fin, g = _bwd_case(52, [75], 1, 4, 3)
    rng = np.random.default_rng(53)
    for name in ("q", "k", "v", "la", "beta"):
        for t in (0, 5, 31, 32, 33, 63, 64, 74):
            idx = (t, 0) if name == "beta" else (t, 0, int(rng.integers(x[name].shape[-1])))
            fd = _central_difference(x, cu, d_o, d_fin, name, idx)
            assert abs(fd - g[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx)
    for idx in ((0, 0, 0, 0), (0, 0, 3, 2)):
        fd = _central_difference(x, cu, d_o, d_fin, "s0", idx)
        assert abs(fd - g["s0"][idx]) <= 1e-6 * max(1.0, abs(fd))


def test_backward_closed_form_without_writes():
    """beta = 0: S_t = Gamma_t S_0 (pure decay), so d_q_t = S_t d_o_t, d_v = d_k = 0 and
    d_S_0 = sum_t Gamma_t q_t d_o_t^T + Gamma_T d_final (written out, no recurrence)."""
    rng = np.random.default_rng(54)
    T, H, Dk, Dv = 6, 1, 3, 2
    q, k, v, la, _ = _rand_inputs(rng, T, H, Dk, Dv)
    beta = np.zeros((T, H))
    s0 = rng.standard_normal((1, H, Dk, Dv))
    d_o = rng.standard_normal((T, H, Dv))
    d_fin = rng.standard_normal((1, H, Dk, Dv))
    dq, dk, dv, dla, db, ds0 = oracle.recurrent_bwd(q, k, v, la, beta, d_o, initial_state=s0,
                                                    d_final=d_fin)
    gam = np.exp(np.cumsum(la[:, 0], axis=0))  # [T, Dk]
    S_t = gam[:, :, None] * s0[0, 0][None]
    np.testing.assert_allclose(dq[:, 0], np.einsum("tkv,tv->tk", S_t, d_o[:, 0]), rtol=1e-13)
    assert np.all(dv == 0) and np.all(dk == 0)
    want = np.einsum("tk,tk,tv->kv", gam, q[:, 0], d_o[:, 0]) + gam[-1][:, None] * d_fin[0, 0]
    np.testing.assert_allclose(ds0[0, 0], want, rtol=1e-13)
