"""Pins for the float64 oracle: checks against what the pages and the mathematics
fix, each written independently of the oracle's own loop (explicit matrices,
the other state orientation, closed forms, library routines).

Every check uses d_k != d_v where the shapes allow, random non-trivial gates
and a non-zero initial state, so that a dropped term, a sign, an index or a
transposed operand in the oracle fails at least one of them.
"""

import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _rand_problem(seed, B=1, T=6, Hqk=1, Hv=1, dk=5, dv=3, s0=True):
    r = _rng(seed)
    q = _unit(r.standard_normal((B, T, Hqk, dk)))
    k = _unit(r.standard_normal((B, T, Hqk, dk)))
    v = r.standard_normal((B, T, Hv, dv))
    alpha = _sig(r.standard_normal((B, T, Hv, dk)) + 1.0)
    b = _sig(r.standard_normal((B, T, Hv, dk)))
    w = _sig(r.standard_normal((B, T, Hv, dv)))
    S0 = 0.5 * r.standard_normal((B, Hv, dk, dv)) if s0 else None
    return q, k, v, alpha, b, w, S0


# ---------------------------------------------------------------- worked example

def test_capital_overwrite_example():
    """Lesson 4.15 capital example: additive writes superpose, the delta rule
    with beta = 1 overwrites (read back with q = k after each write)."""
    g = json.load(open(os.path.join(GOLDEN, "capital_overwrite.json")))
    dk, dv = g["d_k"], g["d_v"]
    k = np.array(g["k"])
    assert abs(np.linalg.norm(k) - 1.0) < 1e-15
    kk = np.stack([k, k])[None, :, None, :]
    vv = np.stack([g["v_paris"], g["v_brasilia"]])[None, :, None, :]
    ones_k = np.ones((1, 2, 1, dk))
    ones_v = np.ones((1, 2, 1, dv))
    # additive fast weights: no erase (b = 0), no decay, full write
    o_add, _ = oracle.gdn2_forward(kk, kk, vv, ones_k, 0 * ones_k, ones_v)
    np.testing.assert_allclose(o_add[0, 1, 0], g["additive_readback_after_both"], atol=1e-14)
    # delta rule, beta = 1 (b = w = 1), no decay
    o_delta, _ = oracle.gdn2_forward(kk, kk, vv, ones_k, ones_k, ones_v)
    np.testing.assert_allclose(o_delta[0, 0, 0], g["delta_readback_after_first"], atol=1e-14)
    np.testing.assert_allclose(o_delta[0, 1, 0], g["delta_readback_after_both"], atol=1e-14)


def test_state_size_closed_form():
    """Lesson 3.6: about 3 MiB of float32 state per 48-head layer, ~144 MiB over 48 layers."""
    g = json.load(open(os.path.join(GOLDEN, "state_size.json")))
    q, k, v, a, b, w, _ = _rand_problem(0, T=1, Hqk=16, Hv=48, dk=128, dv=128, s0=False)
    _, ST = oracle.gdn2_forward(q, k, v, a, b, w)
    nbytes = ST[0].astype(np.float32).nbytes
    assert nbytes == g["state_bytes_per_layer"]
    assert nbytes / 2**20 == g["state_mib_per_layer"]
    assert nbytes * g["layers"] / 2**20 == g["state_mib_all_layers"]


# ----------------------------------------------------------- read-back identities

def test_full_erase_reads_back_gated_value():
    """b = 1 and unit k: (I - k kᵀ) removes what k read, so S_tᵀ k_t = w_t ⊙ v_t
    whatever alpha, S0 and the history were."""
    q, k, v, a, b, w, S0 = _rand_problem(1, T=7)
    q = k.copy()
    o, _ = oracle.gdn2_forward(q, k, v, a, np.ones_like(b), w, S0)
    np.testing.assert_allclose(o, w * v, atol=1e-13)


def test_partial_readback_deltanet():
    """DeltaNet section: reading again with the same unit key after a write
    gives (1 - beta) S̄ᵀk + beta v (tied gates, alpha = 1 so S̄ = S_{t-1})."""
    q, k, v, a, b, w, S0 = _rand_problem(2, T=5)
    beta = _sig(_rng(20).standard_normal((1, 5, 1)))
    alpha, bb, ww = oracle.expand_tied_gates("kda", np.ones_like(a), beta, 5, 3)
    o, _ = oracle.gdn2_forward(k, k, v, alpha, bb, ww, S0)
    S_prev = S0[0, 0]
    for t in range(5):
        if t > 0:
            _, ST = oracle.gdn2_forward(k[:, :t], k[:, :t], v[:, :t], alpha[:, :t], bb[:, :t],
                                        ww[:, :t], S0)
            S_prev = ST[0, 0]
        bt = beta[0, t, 0]
        expect = (1 - bt) * S_prev.T @ k[0, t, 0] + bt * v[0, t, 0]
        np.testing.assert_allclose(o[0, t, 0], expect, atol=1e-13)


def test_locality_orthogonal_query():
    """DeltaNet section: with alpha = 1 a query orthogonal to the written key
    reads the same value before and after the write."""
    q, k, v, a, b, w, S0 = _rand_problem(3, T=4, dk=6)
    ones = np.ones_like(a)
    qo = q.copy()
    for t in range(4):
        kt = k[0, t, 0]
        x = qo[0, t, 0] - (qo[0, t, 0] @ kt) * kt
        qo[0, t, 0] = x / np.linalg.norm(x)
    o, _ = oracle.gdn2_forward(qo, k, v, ones, b, w, S0)
    S_prev = S0[0, 0]
    for t in range(4):
        np.testing.assert_allclose(o[0, t, 0], S_prev.T @ qo[0, t, 0], atol=1e-13)
        _, ST = oracle.gdn2_forward(qo[:, :t + 1], k[:, :t + 1], v[:, :t + 1], ones[:, :t + 1],
                                    b[:, :t + 1], w[:, :t + 1], S0)
        S_prev = ST[0, 0]


def test_eigenvalue_along_key():
    """Structured transition: with alpha = 1 and no write, a state k xᵀ is scaled
    by 1 - eᵀk (1 - beta for tied gates, unit k) and a state u xᵀ with u ⟂ e is
    left unchanged."""
    r = _rng(4)
    dk, dv = 6, 4
    k = _unit(r.standard_normal(dk))
    bvec = _sig(r.standard_normal(dk))
    x = r.standard_normal(dv)
    e = bvec * k
    kk = k[None, None, None, :]
    ones = np.ones((1, 1, 1, dk))
    zero_w = np.zeros((1, 1, 1, dv))
    S0 = np.outer(k, x)[None, None]
    _, ST = oracle.gdn2_forward(kk, kk, np.ones((1, 1, 1, dv)), ones, bvec[None, None, None], zero_w, S0)
    np.testing.assert_allclose(ST[0, 0], (1 - e @ k) * np.outer(k, x), atol=1e-14)
    u = r.standard_normal(dk)
    u -= (u @ e) / (e @ e) * e
    S0u = np.outer(u, x)[None, None]
    _, STu = oracle.gdn2_forward(kk, kk, np.ones((1, 1, 1, dv)), ones, bvec[None, None, None], zero_w, S0u)
    np.testing.assert_allclose(STu[0, 0], np.outer(u, x), atol=1e-14)
    # tied: eigenvalue 1 - beta
    beta = 0.3
    _, STt = oracle.gdn2_forward(kk, kk, np.ones((1, 1, 1, dv)), ones, beta * ones, zero_w, S0)
    np.testing.assert_allclose(STt[0, 0], (1 - beta) * np.outer(k, x), atol=1e-14)


# --------------------------------------------------------------------- reductions

def _kda_loop_dv_dk(q, k, v, alpha, beta, S0_dv_dk, s):
    """KDA as five steps in the d_v x d_k orientation of the hada.io page
    (section "Kimi Delta Attention"): S̃ = S D, v̂ = S̃ k, e = beta (v - v̂),
    S = S̃ + e kᵀ, o = S (s q)."""
    T = q.shape[0]
    S = S0_dv_dk.copy()
    outs = []
    for t in range(T):
        St = S @ np.diag(alpha[t])
        vhat = St @ k[t]
        e = beta[t] * (v[t] - vhat)
        S = St + np.outer(e, k[t])
        outs.append(S @ (s * q[t]))
    return np.array(outs), S


def test_kda_reduction():
    """b = w = beta (scalar) recovers KDA; read scale d_k^-1/2 as on the hada.io page."""
    dk, dv, T = 5, 3, 8
    q, k, v, a, _, _, S0 = _rand_problem(5, T=T, dk=dk, dv=dv)
    beta = _sig(_rng(50).standard_normal((1, T, 1)))
    alpha, bb, ww = oracle.expand_tied_gates("kda", a, beta, dk, dv)
    s = dk ** -0.5
    o, ST = oracle.gdn2_forward(q, k, v, alpha, bb, ww, S0, scale=s)
    o_ref, S_ref = _kda_loop_dv_dk(q[0, :, 0], k[0, :, 0], v[0, :, 0], a[0, :, 0], beta[0, :, 0],
                                   S0[0, 0].T, s)
    np.testing.assert_allclose(o[0, :, 0], o_ref, atol=1e-13)
    np.testing.assert_allclose(ST[0, 0], S_ref.T, atol=1e-13)


def test_gated_deltanet_reduction():
    """Scalar alpha and scalar beta: forget, predict, correct, write (hada.io,
    section "Gated DeltaNet"), in the d_v x d_k orientation, o = S q."""
    dk, dv, T = 4, 6, 8
    q, k, v, _, _, _, S0 = _rand_problem(6, T=T, dk=dk, dv=dv)
    r = _rng(60)
    a_s = _sig(r.standard_normal((1, T, 1)) + 2)
    beta = _sig(r.standard_normal((1, T, 1)))
    alpha, bb, ww = oracle.expand_tied_gates("gdn", a_s, beta, dk, dv)
    o, ST = oracle.gdn2_forward(q, k, v, alpha, bb, ww, S0)
    S = S0[0, 0].T.copy()
    for t in range(T):
        St = a_s[0, t, 0] * S
        vhat = St @ k[0, t, 0]
        e = beta[0, t, 0] * (v[0, t, 0] - vhat)
        S = St + np.outer(e, k[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], S @ q[0, t, 0], atol=1e-13)
    np.testing.assert_allclose(ST[0, 0], S.T, atol=1e-13)


def test_deltanet_reduction():
    """alpha = 1: e_t = beta (v_t - S_{t-1} k_t), S_t = S_{t-1} + e_t k_tᵀ."""
    dk, dv, T = 5, 4, 7
    q, k, v, a, _, _, S0 = _rand_problem(7, T=T, dk=dk, dv=dv)
    beta = _sig(_rng(70).standard_normal((1, T, 1)))
    alpha, bb, ww = oracle.expand_tied_gates("kda", np.ones_like(a), beta, dk, dv)
    o, ST = oracle.gdn2_forward(q, k, v, alpha, bb, ww, S0)
    S = S0[0, 0].T.copy()
    for t in range(T):
        e = beta[0, t, 0] * (v[0, t, 0] - S @ k[0, t, 0])
        S = S + np.outer(e, k[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], S @ q[0, t, 0], atol=1e-13)
    np.testing.assert_allclose(ST[0, 0], S.T, atol=1e-13)


def test_linear_attention_when_no_erase():
    """b = 0, alpha = 1, w = 1: additive linear attention,
    o_t = Σ_{i<=t} (k_iᵀ q_t) v_i + S0ᵀ q_t (masked (Q Kᵀ) V)."""
    dk, dv, T = 5, 3, 9
    q, k, v, a, b, w, S0 = _rand_problem(8, T=T, dk=dk, dv=dv)
    o, ST = oracle.gdn2_forward(q, k, v, np.ones_like(a), np.zeros_like(b), np.ones_like(w), S0)
    Q, K, V = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    ref = np.tril(Q @ K.T) @ V + Q @ S0[0, 0]
    np.testing.assert_allclose(o[0, :, 0], ref, atol=1e-13)
    np.testing.assert_allclose(ST[0, 0], S0[0, 0] + K.T @ V, atol=1e-13)


def test_gated_additive_when_no_erase():
    """b = 0 with per-channel decay: o_t = Σ_{i<=t} Σ_c q_tc k_ic Π_{i<s<=t} α_sc · z_i
    + Σ_c q_tc Π_{s<=t} α_sc S0[c,:]."""
    dk, dv, T = 4, 3, 6
    q, k, v, a, b, w, S0 = _rand_problem(9, T=T, dk=dk, dv=dv)
    o, ST = oracle.gdn2_forward(q, k, v, a, np.zeros_like(b), w, S0)
    Q, K, A, Z = q[0, :, 0], k[0, :, 0], a[0, :, 0], (w * v)[0, :, 0]
    for t in range(T):
        acc = (Q[t] * np.prod(A[:t + 1], axis=0)) @ S0[0, 0]
        for i in range(t + 1):
            dec = np.prod(A[i + 1:t + 1], axis=0) if i < t else np.ones(dk)
            acc = acc + np.sum(Q[t] * K[i] * dec) * Z[i]
        np.testing.assert_allclose(o[0, t, 0], acc, atol=1e-13)


# ------------------------------------------------------------------- brute force

@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_bruteforce_unrolled_transitions(T):
    """Explicit d_k x d_k transitions A_t = (I - k_t e_tᵀ) Diag(alpha_t) (the
    diagonal-plus-low-rank view) and the unrolled sum
    S_t = (A_t⋯A_1) S0 + Σ_j (A_t⋯A_{j+1}) k_j z_jᵀ, o_t = s S_tᵀ q_t."""
    dk, dv = 5, 3
    q, k, v, a, b, w, S0 = _rand_problem(10 + T, T=T, dk=dk, dv=dv)
    s = 0.7
    o, ST = oracle.gdn2_forward(q, k, v, a, b, w, S0, scale=s)
    Q, K, V, A, Bg, W = q[0, :, 0], k[0, :, 0], v[0, :, 0], a[0, :, 0], b[0, :, 0], w[0, :, 0]
    trans = [(np.eye(dk) - np.outer(K[t], Bg[t] * K[t])) @ np.diag(A[t]) for t in range(T)]
    for t in range(T):
        P = np.eye(dk)
        for s_ in range(t, -1, -1):
            P = P @ trans[s_]
        St = P @ S0[0, 0]
        for j in range(t + 1):
            Pj = np.eye(dk)
            for s_ in range(t, j, -1):
                Pj = Pj @ trans[s_]
            St = St + Pj @ np.outer(K[j], W[j] * V[j])
        np.testing.assert_allclose(o[0, t, 0], s * St.T @ Q[t], atol=1e-13)
        if t == T - 1:
            np.testing.assert_allclose(ST[0, 0], St, atol=1e-13)


def test_linearity_in_state_and_write():
    """S_T and o are jointly linear in (S0, Z): f(S0, Z) = f(S0, 0) + f(0, Z)."""
    q, k, v, a, b, w, S0 = _rand_problem(20, T=8, dk=6, dv=4)
    o1, S1 = oracle.gdn2_forward(q, k, v, a, b, w, S0)
    o2, S2 = oracle.gdn2_forward(q, k, v, a, b, np.zeros_like(w), S0)
    o3, S3 = oracle.gdn2_forward(q, k, v, a, b, w, None)
    np.testing.assert_allclose(o1, o2 + o3, atol=1e-13)
    np.testing.assert_allclose(S1, S2 + S3, atol=1e-13)


def test_split_sequence_carries_state():
    """The recurrence is a left fold: running [0,t) then [t,T) from the carried
    state equals one run over [0,T)."""
    q, k, v, a, b, w, S0 = _rand_problem(21, T=9)
    o, ST = oracle.gdn2_forward(q, k, v, a, b, w, S0)
    oa, Sa = oracle.gdn2_forward(q[:, :4], k[:, :4], v[:, :4], a[:, :4], b[:, :4], w[:, :4], S0)
    ob, Sb = oracle.gdn2_forward(q[:, 4:], k[:, 4:], v[:, 4:], a[:, 4:], b[:, 4:], w[:, 4:], Sa)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, atol=1e-13)
    np.testing.assert_allclose(Sb, ST, atol=1e-13)


def test_empty_sequence_returns_initial_state():
    q, k, v, a, b, w, S0 = _rand_problem(22, T=0)
    o, ST = oracle.gdn2_forward(q, k, v, a, b, w, S0)
    assert o.shape == (1, 0, 1, 3)
    np.testing.assert_array_equal(ST, S0)


def test_grouped_heads_contiguous_mapping():
    """Each QK head serves H_v/H_qk consecutive V heads: V head h reads QK head
    h // (H_v/H_qk). Checked against separate single-head runs, with B = 2."""
    q, k, v, a, b, w, S0 = _rand_problem(23, B=2, T=5, Hqk=2, Hv=6, dk=4, dv=3)
    o, ST = oracle.gdn2_forward(q, k, v, a, b, w, S0)
    for bi in range(2):
        for h in range(6):
            hq = h // 3
            sl = (slice(bi, bi + 1), slice(None))
            oh, Sh = oracle.gdn2_forward(q[bi:bi + 1, :, hq:hq + 1], k[bi:bi + 1, :, hq:hq + 1],
                                         v[bi:bi + 1, :, h:h + 1], a[bi:bi + 1, :, h:h + 1],
                                         b[bi:bi + 1, :, h:h + 1], w[bi:bi + 1, :, h:h + 1],
                                         S0[bi:bi + 1, h:h + 1])
            np.testing.assert_allclose(o[sl][0, :, h], oh[0, :, 0], atol=1e-14)
            np.testing.assert_allclose(ST[bi, h], Sh[0, 0], atol=1e-14)


def test_threads_do_not_change_result():
    q, k, v, a, b, w, S0 = _rand_problem(24, B=3, T=6, Hqk=2, Hv=4, dk=4, dv=5)
    o1, S1 = oracle.gdn2_forward(q, k, v, a, b, w, S0, threads=1)
    o4, S4 = oracle.gdn2_forward(q, k, v, a, b, w, S0, threads=4)
    np.testing.assert_array_equal(o1, o4)
    np.testing.assert_array_equal(S1, S4)


def test_scale_is_linear():
    q, k, v, a, b, w, S0 = _rand_problem(25)
    o1, S1 = oracle.gdn2_forward(q, k, v, a, b, w, S0, scale=1.0)
    o2, S2 = oracle.gdn2_forward(q, k, v, a, b, w, S0, scale=0.25)
    np.testing.assert_allclose(o2, 0.25 * o1, atol=1e-15)
    np.testing.assert_array_equal(S1, S2)


# --------------------------------------------------------------- preprocessing

def test_causal_conv_matches_numpy_convolve():
    r = _rng(30)
    B, T, C = 2, 11, 5
    x = r.standard_normal((B, T, C))
    W = r.standard_normal((C, 4))
    y = oracle.causal_conv4(x, W)
    for bi in range(B):
        for c in range(C):
            ref = np.convolve(x[bi, :, c], W[c][::-1])[:T]
            np.testing.assert_allclose(y[bi, :, c], ref, atol=1e-14)


def test_conv_current_token_tap_and_causality():
    """W[c][3] weights the current token; nothing reads the future."""
    x = np.zeros((1, 6, 1))
    x[0, 2, 0] = 1.0
    W = np.array([[1.0, 2.0, 3.0, 4.0]])
    y = oracle.causal_conv4(x, W)
    np.testing.assert_array_equal(y[0, :, 0], [0, 0, 4, 3, 2, 1])


def test_conv_history_taps_closed_form():
    """With only tap j set, y_t = W[c][j]·x_{t−3+j}: the first outputs read the
    history rows oldest first (row 0 = token −3), then the tokens themselves."""
    hist = np.array([[[10.0], [20.0], [30.0]]])      # tokens −3, −2, −1
    x = np.array([[[1.0], [2.0], [3.0], [4.0]]])
    for j, ref in ((0, [10, 20, 30, 1]), (1, [20, 30, 1, 2]), (2, [30, 1, 2, 3]), (3, [1, 2, 3, 4])):
        W = np.zeros((1, 4))
        W[0, j] = 2.0
        y = oracle.causal_conv4(x, W, hist)
        np.testing.assert_array_equal(y[0, :, 0], 2.0 * np.array(ref, dtype=float))


def test_conv_split_equals_whole_and_state_rows():
    """Convolving a sequence in pieces, each starting from the history the
    previous piece leaves (conv_state_after), equals one conv of the whole
    sequence: the conv is causal over the token stream. Pieces shorter than
    three tokens shift the older history through."""
    r = _rng(33)
    B, T, Hqk, Hv, dk, dv = 2, 13, 1, 2, 3, 2
    q = r.standard_normal((B, T, Hqk, dk))
    k = r.standard_normal((B, T, Hqk, dk))
    v = r.standard_normal((B, T, Hv, dv))
    W = r.standard_normal((2 * Hqk * dk + Hv * dv, 4))
    whole = oracle.preprocess(q, k, v, W, l2norm_qk=True)
    for cuts in ([0, 5, 13], [0, 1, 2, 3, 13], [0, 2, 4, 6, 7, 13], [0, 13, 13]):
        state = None
        parts = []
        for t0, t1 in zip(cuts[:-1], cuts[1:]):
            sl = slice(t0, t1)
            parts.append(oracle.preprocess(q[:, sl], k[:, sl], v[:, sl], W, l2norm_qk=True, conv_state=state))
            state = oracle.conv_state_after(q[:, sl], k[:, sl], v[:, sl], state)
        for i in range(3):
            got = np.concatenate([p[i] for p in parts], axis=1)
            np.testing.assert_allclose(got, whole[i], rtol=0, atol=1e-13)
        # the final history holds the inputs of tokens T−3, T−2, T−1, channels q | k | v
        last = np.concatenate([q[:, -3:].reshape(B, 3, -1), k[:, -3:].reshape(B, 3, -1),
                               v[:, -3:].reshape(B, 3, -1)], axis=2)
        np.testing.assert_array_equal(state, last)
    # one token after a given history: rows 1, 2 of it, then the token
    h = r.standard_normal((B, 3, 2 * Hqk * dk + Hv * dv))
    s1 = oracle.conv_state_after(q[:, :1], k[:, :1], v[:, :1], h)
    np.testing.assert_array_equal(s1[:, :2], h[:, 1:])
    np.testing.assert_array_equal(s1[:, 2], oracle.conv_inputs(q[:, :1], k[:, :1], v[:, :1])[:, 0])


def test_l2norm_matches_numpy():
    r = _rng(31)
    x = r.standard_normal((3, 7, 9))
    y = oracle.l2norm(x)
    ref = x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + oracle.L2NORM_EPS)
    np.testing.assert_allclose(y, ref, rtol=1e-15)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-6)


def test_preprocess_order_conv_then_norm():
    r = _rng(32)
    B, T, Hqk, Hv, dk, dv = 1, 7, 2, 4, 3, 2
    q = r.standard_normal((B, T, Hqk, dk))
    k = r.standard_normal((B, T, Hqk, dk))
    v = r.standard_normal((B, T, Hv, dv))
    W = r.standard_normal((2 * Hqk * dk + Hv * dv, 4))
    qp, kp, vp = oracle.preprocess(q, k, v, W, l2norm_qk=True)
    nq = Hqk * dk
    qc = oracle.causal_conv4(q.reshape(B, T, nq), W[:nq]).reshape(q.shape)
    kc = oracle.causal_conv4(k.reshape(B, T, nq), W[nq:2 * nq]).reshape(k.shape)
    vc = oracle.causal_conv4(v.reshape(B, T, Hv * dv), W[2 * nq:]).reshape(v.shape)
    np.testing.assert_allclose(qp, qc / np.linalg.norm(qc, axis=-1, keepdims=True), rtol=1e-5)
    np.testing.assert_allclose(kp, kc / np.linalg.norm(kc, axis=-1, keepdims=True), rtol=1e-5)
    np.testing.assert_array_equal(vp, vc)


def test_gates_for_value_heads_mapping_and_group_symmetry():
    """Value head h takes the gates of QK head h // (H_v/H_qk) (contiguous
    groups); and with gates shared, the heads of one group that also get the
    same v and w run identical recurrences (a consequence of sharing q, k and
    the key-side gates), while heads of different groups do not."""
    B, T, Hqk, Hv, d = 1, 6, 2, 6, 4
    g = np.arange(B * T * Hqk * d, dtype=float).reshape(B, T, Hqk, d)
    e = oracle.gates_for_value_heads(g, Hv)
    assert e.shape == (B, T, Hv, d)
    for h in range(Hv):
        np.testing.assert_array_equal(e[:, :, h], g[:, :, h // 3])
    s = np.arange(4, dtype=float).reshape(2, 2)          # one step: [B, H_qk]
    np.testing.assert_array_equal(oracle.gates_for_value_heads(s, 4, axis=1), [[0, 0, 1, 1], [2, 2, 3, 3]])
    r = _rng(34)
    q = _unit(r.standard_normal((B, T, Hqk, d)))
    k = _unit(r.standard_normal((B, T, Hqk, d)))
    v1 = r.standard_normal((B, T, 1, d))
    w1 = 1.0 / (1.0 + np.exp(-r.standard_normal((B, T, 1, d))))
    v, w = np.repeat(v1, Hv, axis=2), np.repeat(w1, Hv, axis=2)
    a = oracle.gates_for_value_heads(1.0 / (1.0 + np.exp(-3.0 - r.standard_normal((B, T, Hqk, d)))), Hv)
    b = oracle.gates_for_value_heads(1.0 / (1.0 + np.exp(-r.standard_normal((B, T, Hqk, d)))), Hv)
    qv, kv = np.repeat(q, 3, axis=2), np.repeat(k, 3, axis=2)
    o, S = oracle.gdn2_forward(qv, kv, v, a, b, w)
    for h in (1, 2):
        np.testing.assert_array_equal(o[:, :, h], o[:, :, 0])
        np.testing.assert_array_equal(S[:, h], S[:, 0])
    assert np.abs(o[:, :, 3] - o[:, :, 0]).max() > 1e-3


@pytest.mark.parametrize("C", [4, 16])
def test_chunk_algebra_equals_token_loop(C):
    """The chunked form the prefill kernels compute ("Chunkwise KDA" of the
    hada.io page, with the decoupled gates of the GDN-2 summary, Metodologia
    §3), written out in float64 from its equations, equals the token loop to
    rounding: per chunk with entry state S and γ_i = Π_{s≤i} α_s,
        T_ij = Σ_c e_ic k_jc γ_ic/γ_jc (j < i),  Aqk_ij = Σ_c q_ic k_jc γ_ic/γ_jc (j ≤ i),
        Y = (I+T)⁻¹ Ē,  U_w = (I+T)⁻¹ Z,  U = U_w − Y S,
        O = Q̄ S + Aqk U,  S ← Diag(γ_C) S + K_endᵀ U,
    and the state update is the affine map S ← (Diag(γ_C) − K_endᵀ Y) S + K_endᵀ U_w."""
    r = _rng(40 + C)
    T, dk, dv = 3 * C + 1, 5, 3                      # a ragged last chunk
    q = _unit(r.standard_normal((T, dk)))
    k = _unit(r.standard_normal((T, dk)))
    v = r.standard_normal((T, dv))
    a = _sig(r.standard_normal((T, dk)) + 2.0)
    b = _sig(r.standard_normal((T, dk)))
    w = _sig(r.standard_normal((T, dv)))
    S0 = 0.1 * r.standard_normal((dk, dv))
    o_ref, S_ref = oracle.gdn2_forward(q[None, :, None], k[None, :, None], v[None, :, None], a[None, :, None],
                                       b[None, :, None], w[None, :, None], S0[None, None])
    S = S0.copy()
    out = []
    for t0 in range(0, T, C):
        sl = slice(t0, min(T, t0 + C))
        qc, kc, vc, ac, bc, wc = q[sl], k[sl], v[sl], a[sl], b[sl], w[sl]
        L = qc.shape[0]
        g = np.cumprod(ac, axis=0)                   # γ_i per key channel
        e, z = bc * kc, wc * vc
        Eb, Qb = e * g, qc * g                       # Ē, Q̄
        Kt = kc / g                                  # K̃ (γ_i/γ_j = Ē_i·K̃_j)
        Tm = np.tril(Eb @ Kt.T, -1)
        Aqk = np.tril(Qb @ Kt.T)
        Ainv = np.linalg.inv(np.eye(L) + Tm)
        Y, Uw = Ainv @ Eb, Ainv @ z
        U = Uw - Y @ S
        out.append(Qb @ S + Aqk @ U)
        Kend = kc * (g[-1] / g)                      # k_j ⊙ Π_{j<s≤L} α_s
        S_aff = (np.diag(g[-1]) - Kend.T @ Y) @ S + Kend.T @ Uw
        S = g[-1][:, None] * S + Kend.T @ U
        np.testing.assert_allclose(S_aff, S, rtol=0, atol=1e-12)
    o = np.concatenate(out)
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, S_ref[0, 0], rtol=0, atol=1e-12)


def test_rel_err_metric():
    ref = np.array([3.0, -4.0])
    assert oracle.rel_err(ref, ref) == 0.0
    got = ref + np.array([0.0, 0.5])
    assert abs(oracle.rel_err(got, ref) - 0.5 / np.sqrt(12.5)) < 1e-15


def test_gates_from_logits_closed_forms():
    """σ(0) = 1/2, σ(ln 3) = 3/4 and σ(−ln 3) = 1/4 exactly in closed form;
    σ(x) + σ(−x) = 1; increasing; saturates to 0 and 1 without NaN."""
    s = oracle.gates_from_logits(np.array([0.0, np.log(3.0), -np.log(3.0)]))
    np.testing.assert_allclose(s, [0.5, 0.75, 0.25], rtol=0, atol=1e-15)
    x = _rng(50).standard_normal(1000) * 6.0
    np.testing.assert_allclose(oracle.gates_from_logits(x) + oracle.gates_from_logits(-x), 1.0, rtol=0,
                               atol=1e-15)
    xs = np.sort(x)
    assert np.all(np.diff(oracle.gates_from_logits(xs)) >= 0)
    ext = oracle.gates_from_logits(np.array([-1000.0, 1000.0]))
    assert ext[0] == 0.0 and ext[1] == 1.0
    # the odds: σ(x) / σ(−x) = e^x
    xm = x[np.abs(x) < 30]
    np.testing.assert_allclose(oracle.gates_from_logits(xm) / oracle.gates_from_logits(-xm), np.exp(xm),
                               rtol=1e-12)
