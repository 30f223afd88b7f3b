"""Pins of the backward oracle (oracle.gdn2_backward) against what mathematics
fixes without it ("Resumo Técnico: Gated DeltaNet-2", Metodologia §1 and §3;
the gradient is that of L = <dO, o> + <dS_T, S_T>):

* central finite differences of the forward oracle (a separate code path),
  for every input, on a problem small enough to perturb every element, and
  on sampled elements of one longer than the 64-token recomputation blocks;
* exact adjoint identities: o and S_T are jointly linear in (S0, v) at fixed
  q, k, α, b, w, so L = <dS0, S0> + <dv, v>; o is linear in q and S_T does not
  depend on it, so <dO, o> = <dq, q>; with S0 = 0, L is linear in w, so
  L = <dw, w>;
* the chain rules through the tied gates (KDA, Gated DeltaNet), the gates
  owned by query/key heads and gate logits, against finite differences of
  the forward oracle run on the expanded gates."""

import numpy as np
import pytest

import oracle


def _problem(rng, B=1, T=7, H_qk=1, H_v=2, d=4, s0=True):
    q = rng.standard_normal((B, T, H_qk, d))
    k = rng.standard_normal((B, T, H_qk, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    x = dict(q=q, k=k, v=rng.standard_normal((B, T, H_v, d)),
             alpha=rng.uniform(0.3, 0.99, (B, T, H_v, d)), b=rng.uniform(0.05, 0.95, (B, T, H_v, d)),
             w=rng.uniform(0.05, 0.95, (B, T, H_v, d)),
             S0=rng.standard_normal((B, H_v, d, d)) * 0.5 if s0 else None)
    up = dict(dO=rng.standard_normal((B, T, H_v, d)), dS_T=rng.standard_normal((B, H_v, d, d)))
    return x, up


def _loss(x, up, scale):
    o, S = oracle.gdn2_forward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], scale=scale)
    return float(np.sum(up["dO"] * o) + np.sum(up["dS_T"] * S))


def _fd_check(x, up, g, names, scale=1.0, sample=None, rng=None, h=1e-6, tol=1e-6):
    for name in names:
        flat = x[name].reshape(-1)
        idx = range(flat.size) if sample is None else rng.choice(flat.size, size=sample, replace=False)
        gf = g[name].reshape(-1)
        worst = 0.0
        for i in idx:
            keep = flat[i]
            flat[i] = keep + h
            lp = _loss(x, up, scale)
            flat[i] = keep - h
            lm = _loss(x, up, scale)
            flat[i] = keep
            fd = (lp - lm) / (2 * h)
            worst = max(worst, abs(fd - gf[i]))
        ref = max(float(np.sqrt(np.mean(g[name] ** 2))), 1e-3)
        assert worst / ref <= tol, f"d{name}: finite differences differ by {worst:.3e} (RMS {ref:.3e})"


@pytest.mark.parametrize("scale", [1.0, 0.5])
def test_backward_matches_finite_differences_every_element(scale):
    rng = np.random.default_rng(1)
    x, up = _problem(rng)
    g = oracle.gdn2_backward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], up["dO"], up["dS_T"],
                             scale=scale)
    _fd_check(x, up, g, ["q", "k", "v", "alpha", "b", "w", "S0"], scale=scale)


def test_backward_matches_finite_differences_across_recompute_blocks():
    """T = 150 spans three 64-token recomputation blocks; grouped heads
    (2 QK / 6 V) so dq and dk sum over the value heads of a group."""
    rng = np.random.default_rng(2)
    x, up = _problem(rng, B=2, T=150, H_qk=2, H_v=6, d=4)
    g = oracle.gdn2_backward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], up["dO"], up["dS_T"])
    _fd_check(x, up, g, ["q", "k", "v", "alpha", "b", "w", "S0"], sample=40, rng=rng)


def test_adjoint_identities():
    rng = np.random.default_rng(3)
    x, up = _problem(rng, B=2, T=90, H_qk=2, H_v=4, d=16)
    o, S = oracle.gdn2_forward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"])
    g = oracle.gdn2_backward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], up["dO"], up["dS_T"])
    L = np.sum(up["dO"] * o) + np.sum(up["dS_T"] * S)
    scale_ = max(abs(L), 1.0)
    # jointly linear in (S0, v)
    assert abs(np.sum(g["S0"] * x["S0"]) + np.sum(g["v"] * x["v"]) - L) <= 1e-10 * scale_ * 100
    # linear in q; S_T does not depend on q
    assert abs(np.sum(g["q"] * x["q"]) - np.sum(up["dO"] * o)) <= 1e-10 * scale_ * 100
    # with S0 = 0: linear in w
    g0 = oracle.gdn2_backward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], None, up["dO"], up["dS_T"])
    o0, S0_ = oracle.gdn2_forward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], None)
    L0 = np.sum(up["dO"] * o0) + np.sum(up["dS_T"] * S0_)
    assert abs(np.sum(g0["w"] * x["w"]) - L0) <= 1e-8 * max(abs(L0), 1.0)
    # no upstream gradient of the state: dS_T = None is zeros
    g1 = oracle.gdn2_backward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], up["dO"], None)
    g2 = oracle.gdn2_backward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], up["dO"],
                              np.zeros_like(up["dS_T"]))
    for key in g1:
        np.testing.assert_array_equal(g1[key], g2[key])


@pytest.mark.parametrize("mode", ["kda", "gdn"])
def test_tied_gate_chain_rule(mode):
    """dβ and the scalar dα of the tied forms against finite differences of
    the forward oracle run on the expanded gates."""
    rng = np.random.default_rng(4)
    B, T, H, d = 1, 9, 2, 4
    x, up = _problem(rng, B=B, T=T, H_qk=1, H_v=H, d=d)
    beta = rng.uniform(0.1, 0.9, (B, T, H))
    a_t = rng.uniform(0.5, 0.99, (B, T, H) if mode == "gdn" else (B, T, H, d))

    def loss(a_, be):
        al, b_, w_ = oracle.expand_tied_gates(mode, a_, be, d, d)
        return _loss(dict(x, alpha=al, b=b_, w=w_), up, 1.0)

    al, b_, w_ = oracle.expand_tied_gates(mode, a_t, beta, d, d)
    g = oracle.gdn2_backward(x["q"], x["k"], x["v"], al, b_, w_, x["S0"], up["dO"], up["dS_T"])
    da, dbeta = oracle.tied_gate_grads(mode, g["alpha"], g["b"], g["w"])
    h = 1e-6
    for arr, grad in ((a_t, da), (beta, dbeta)):
        flat, gf = arr.reshape(-1), grad.reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            lp = loss(a_t, beta)
            flat[i] = keep - h
            lm = loss(a_t, beta)
            flat[i] = keep
            assert abs((lp - lm) / (2 * h) - gf[i]) <= 1e-6 * max(1.0, abs(gf[i]))


def test_qk_head_gates_and_logits_chain_rule():
    """Gates owned by query/key heads and given as logits: the summed and
    σ'-scaled per-channel gradients against finite differences of the
    forward oracle on σ of the expanded logits."""
    rng = np.random.default_rng(5)
    B, T, H_qk, H_v, d = 1, 8, 1, 3, 4
    x, up = _problem(rng, B=B, T=T, H_qk=H_qk, H_v=H_v, d=d)
    xa = rng.normal(2.0, 1.0, (B, T, H_qk, d))     # logits of α per QK head
    xb = rng.normal(0.0, 1.0, (B, T, H_qk, d))     # logits of b per QK head
    xw = rng.normal(0.0, 1.0, (B, T, H_v, d))      # logits of w per value head

    def gates(xa_, xb_, xw_):
        return (oracle.gates_for_value_heads(oracle.gates_from_logits(xa_), H_v),
                oracle.gates_for_value_heads(oracle.gates_from_logits(xb_), H_v), oracle.gates_from_logits(xw_))

    al, b_, w_ = gates(xa, xb, xw)
    g = oracle.gdn2_backward(x["q"], x["k"], x["v"], al, b_, w_, x["S0"], up["dO"], up["dS_T"])
    dxa = oracle.logit_grads(oracle.grads_for_qk_heads(g["alpha"], H_qk), xa)
    dxb = oracle.logit_grads(oracle.grads_for_qk_heads(g["b"], H_qk), xb)
    dxw = oracle.logit_grads(g["w"], xw)
    h = 1e-6
    for arr, grad in ((xa, dxa), (xb, dxb), (xw, dxw)):
        flat, gf = arr.reshape(-1), grad.reshape(-1)
        for i in range(0, flat.size, 3):
            keep = flat[i]
            flat[i] = keep + h
            a1, b1, w1 = gates(xa, xb, xw)
            lp = _loss(dict(x, alpha=a1, b=b1, w=w1), up, 1.0)
            flat[i] = keep - h
            a1, b1, w1 = gates(xa, xb, xw)
            lm = _loss(dict(x, alpha=a1, b=b1, w=w1), up, 1.0)
            flat[i] = keep
            assert abs((lp - lm) / (2 * h) - gf[i]) <= 1e-6 * max(1.0, abs(gf[i]))
