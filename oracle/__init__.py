"""Float64 CPU oracle for the Gated DeltaNet-2 recurrence.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. It shares no code
with the CUDA library (``delta_rule_linear_gdn_b200``) and neither imports the
other.

Functions and the passages they follow:

* :func:`gdn2_forward` -- the token-by-token recurrence of
  "Resumo Técnico: Gated DeltaNet-2", Metodologia §1 "Regra Delta Portão-2":
  ``S_t = (I - k_t (b_t ⊙ k_t)^T) Diag(α_t) S_{t-1} + k_t (w_t ⊙ v_t)^T``,
  read after the write as ``o_t = s · S_t^T q_t`` (C++ loop in
  ``gdn2_oracle.cpp``).
* :func:`expand_tied_gates` -- the reductions of the same section: tying
  ``b_t`` and ``w_t`` to one scalar ``β_t`` gives KDA; tying ``α_t`` to a
  scalar as well gives Gated DeltaNet.
* :func:`gates_for_value_heads` -- gates shared per query/key head, given to
  each value head of the group (its contiguous head grouping).
* :func:`causal_conv4` -- depthwise causal convolution with kernel 4
  ("Gated DeltaNet: o mixer em 48 das 64 camadas", Conceito).
* :func:`l2norm` -- row-wise L2 normalisation of queries and keys (the pages
  assume normalised keys: "Uma análise das variantes de atenção linear da
  família DeltaNet", Notação e ordem da derivação).
* :func:`preprocess` -- conv then L2 norm, in that order.
* :func:`conv_state_after` -- the conv's three-token history after a call, so
  that a sequence split into calls (prefill pieces, decode steps) convolves
  exactly as one call over all its tokens (same page: the conv is causal
  over the token stream, which a split does not change).
* :func:`gdn2_backward` -- the gradients of ``<dO, o> + <dS_T, S_T>`` with
  respect to every input of :func:`gdn2_forward`: reverse-mode
  differentiation of the same token loop, written out step by step in C++
  (``gdn2_oracle_bwd.cpp``); "Resumo Técnico: Gated DeltaNet-2", Metodologia
  §3, "Passagem de Retropropagação Consciente de Portões".
* :func:`tied_gate_grads`, :func:`grads_for_qk_heads`, :func:`logit_grads` --
  the chain rule through the tied gates, the gates shared per query/key head
  and the sigmoid of gate logits (sums and products of the per-channel
  gradients, the transposes of :func:`expand_tied_gates`,
  :func:`gates_for_value_heads` and :func:`gates_from_logits`).
* :func:`gates_from_logits` -- the gates as the sigmoid of their projections'
  outputs ("BigSaaS – Posts", section "Implementação Prática: Como Funciona a
  Camada de Atenção do DeltaNet-2": erase and write gates pass through a
  sigmoid so that they lie between 0 and 1).

Pins: every function above is checked in ``tests/test_oracle_pins.py`` against
closed forms, special cases and brute force (no function is parity-unpinned).
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.cpp")
_SRC_BWD = os.path.join(_HERE, "gdn2_oracle_bwd.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

L2NORM_EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile the C++ oracle with g++ (plain -O2, IEEE double)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_BWD))
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < newest:
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", _SRC, _SRC_BWD, "-o", _LIB_PATH]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_gdn2_forward.argtypes = [ctypes.c_int] * 6 + [ctypes.c_double] + [dp] * 9 + [ctypes.c_int]
        lib.oracle_gdn2_forward.restype = ctypes.c_int
        lib.oracle_causal_conv4.argtypes = [ctypes.c_int] * 3 + [dp] * 3
        lib.oracle_causal_conv4.restype = ctypes.c_int
        lib.oracle_l2norm.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_double, dp, dp]
        lib.oracle_l2norm.restype = ctypes.c_int
        lib.oracle_gdn2_backward.argtypes = [ctypes.c_int] * 6 + [ctypes.c_double] + [dp] * 16 + [ctypes.c_int]
        lib.oracle_gdn2_backward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def gdn2_forward(q, k, v, alpha, b, w, S0=None, scale: float = 1.0, threads: int = 0):
    """Run the recurrence. Shapes: q,k [B,T,Hqk,dk]; v [B,T,Hv,dv];
    alpha,b [B,T,Hv,dk]; w [B,T,Hv,dv]; S0 [B,Hv,dk,dv] or None.
    Returns (o [B,T,Hv,dv], S_T [B,Hv,dk,dv]) in float64."""
    q, k, v, alpha, b, w = (_f64(x) for x in (q, k, v, alpha, b, w))
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    assert k.shape == q.shape and v.shape[:2] == (B, T)
    assert alpha.shape == (B, T, Hv, dk) and b.shape == (B, T, Hv, dk) and w.shape == (B, T, Hv, dv)
    if S0 is not None:
        S0 = _f64(S0)
        assert S0.shape == (B, Hv, dk, dv)
    o = np.zeros((B, T, Hv, dv), dtype=np.float64)
    ST = np.zeros((B, Hv, dk, dv), dtype=np.float64)
    rc = _load().oracle_gdn2_forward(B, T, Hqk, Hv, dk, dv, float(scale), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o), _ptr(ST),
                                     int(threads))
    if rc != 0:
        raise ValueError("oracle_gdn2_forward rejected its arguments")
    return o, ST


def gdn2_backward(q, k, v, alpha, b, w, S0, dO, dS_T=None, scale: float = 1.0, threads: int = 0):
    """Gradients of L = <dO, o> + <dS_T, S_T> for the inputs of
    :func:`gdn2_forward` (same shapes; per-channel gates per value head).
    S0 and dS_T may be None (zeros). Returns a dict with keys q, k, v, alpha,
    b, w, S0 (float64)."""
    q, k, v, alpha, b, w, dO = (_f64(x) for x in (q, k, v, alpha, b, w, dO))
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    assert k.shape == q.shape and v.shape[:2] == (B, T) and dO.shape == v.shape
    assert alpha.shape == (B, T, Hv, dk) and b.shape == (B, T, Hv, dk) and w.shape == (B, T, Hv, dv)
    S0 = None if S0 is None else _f64(S0)
    dS_T = None if dS_T is None else _f64(dS_T)
    for s_ in (S0, dS_T):
        assert s_ is None or s_.shape == (B, Hv, dk, dv)
    g = {"q": np.zeros_like(q), "k": np.zeros_like(k), "v": np.zeros_like(v), "alpha": np.zeros_like(alpha),
         "b": np.zeros_like(b), "w": np.zeros_like(w), "S0": np.zeros((B, Hv, dk, dv))}
    rc = _load().oracle_gdn2_backward(B, T, Hqk, Hv, dk, dv, float(scale), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(dO), _ptr(dS_T),
                                      _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]), _ptr(g["alpha"]), _ptr(g["b"]),
                                      _ptr(g["w"]), _ptr(g["S0"]), int(threads))
    if rc != 0:
        raise ValueError("oracle_gdn2_backward rejected its arguments")
    return g


def tied_gate_grads(mode: str, dalpha, db, dw):
    """Chain rule through :func:`expand_tied_gates`: "kda" gives dβ = Σ_c db_c +
    Σ_v dw_v (per token and head) and the per-channel dα; "gdn" also sums dα
    over the channels. Returns (dalpha, dbeta)."""
    dalpha, db, dw = _f64(dalpha), _f64(db), _f64(dw)
    dbeta = db.sum(axis=-1) + dw.sum(axis=-1)
    if mode == "gdn":
        dalpha = dalpha.sum(axis=-1)
    elif mode != "kda":
        raise ValueError(mode)
    return dalpha, dbeta


def grads_for_qk_heads(g, H_qk: int, axis: int = 2):
    """Chain rule through :func:`gates_for_value_heads`: the gradient of a gate
    shared by the value heads of a query/key head is the sum over those heads."""
    g = _f64(g)
    H_v = g.shape[axis]
    assert H_v % H_qk == 0
    shape = g.shape[:axis] + (H_qk, H_v // H_qk) + g.shape[axis + 1:]
    return g.reshape(shape).sum(axis=axis + 1)


def logit_grads(dgate, x):
    """Chain rule through :func:`gates_from_logits`: dL/dx = dL/dσ · σ(x)(1 − σ(x))."""
    s = gates_from_logits(x)
    return _f64(dgate) * s * (1.0 - s)


def expand_tied_gates(mode: str, alpha, beta, d_k: int, d_v: int):
    """Per-channel gates of a tied variant.

    mode "kda": alpha [...,dk] per channel, beta [...] scalar -> b = beta·1_dk, w = beta·1_dv.
    mode "gdn": alpha [...] scalar and beta [...] scalar -> alpha·1_dk as well.
    Returns (alpha [..., dk], b [..., dk], w [..., dv]) in float64.
    """
    beta = _f64(beta)
    b = np.repeat(beta[..., None], d_k, axis=-1)
    w = np.repeat(beta[..., None], d_v, axis=-1)
    alpha = _f64(alpha)
    if mode == "gdn":
        alpha = np.repeat(alpha[..., None], d_k, axis=-1)
    elif mode != "kda":
        raise ValueError(mode)
    return alpha, b, w


def gates_for_value_heads(g, H_v: int, axis: int = 2):
    """Gates owned by query/key heads, head axis ``axis`` ([B,T,H_qk,...]; 1
    for one step's [B,H_qk,...]), repeated for the value heads that read each
    QK head: value head h takes QK head h // (H_v / H_qk), the contiguous
    grouping of "Gated DeltaNet: o mixer em 48 das 64 camadas", Conceito."""
    g = _f64(g)
    H_qk = g.shape[axis]
    assert H_v % H_qk == 0
    return np.repeat(g, H_v // H_qk, axis=axis)


def causal_conv4(x, W, history=None):
    """x [B,T,C], W [C,4] -> y [B,T,C] (depthwise causal conv).

    ``history`` [B,3,C] holds the three inputs before token 0, oldest first
    (None: zeros). The conv is then the zero-history conv of the stream
    ``history ++ x`` with its first three outputs dropped: the definition of a
    conv that continues over earlier tokens."""
    x = _f64(x)
    W = _f64(W)
    B, T, C = x.shape
    assert W.shape == (C, 4)
    if history is not None:
        h = _f64(history)
        assert h.shape == (B, 3, C)
        return causal_conv4(np.concatenate([h, x], axis=1), W)[:, 3:]
    y = np.zeros_like(x)
    if _load().oracle_causal_conv4(B, T, C, _ptr(x), _ptr(W), _ptr(y)) != 0:
        raise ValueError("oracle_causal_conv4 rejected its arguments")
    return y


def conv_inputs(q, k, v):
    """The conv's input channels per token: [B,T, Hqk·dk | Hqk·dk | Hv·dv]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hqk, dk = q.shape
    nq, nv = Hqk * dk, v.shape[2] * v.shape[3]
    return np.concatenate([q.reshape(B, T, nq), k.reshape(B, T, nq), v.reshape(B, T, nv)], axis=2)


def conv_state_after(q, k, v, conv_state=None):
    """The conv history after the last token: the last three rows of
    ``conv_state ++ inputs`` ([B,3,C], oldest first; zeros stand in for a
    missing ``conv_state``)."""
    x = conv_inputs(q, k, v)
    B, _, C = x.shape
    h = np.zeros((B, 3, C)) if conv_state is None else _f64(conv_state)
    return np.concatenate([h, x], axis=1)[:, -3:]


def l2norm(x, eps: float = L2NORM_EPS):
    """Normalise the last axis: x · (Σx² + eps)^(-1/2)."""
    x = _f64(x)
    d = x.shape[-1]
    n = x.size // d if d else 0
    y = np.zeros_like(x)
    if _load().oracle_l2norm(n, d, float(eps), _ptr(x), _ptr(y)) != 0:
        raise ValueError("oracle_l2norm rejected its arguments")
    return y


def preprocess(q, k, v, conv_w=None, l2norm_qk: bool = False, conv_state=None):
    """Optional depthwise causal conv on q, k, v (weights [Hqk·dk + Hqk·dk + Hv·dv, 4],
    rows ordered q | k | v; history ``conv_state`` [B,3,channels] in the same
    channel order, None for zeros), then optional L2 normalisation of q and k."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if conv_w is not None:
        W = _f64(conv_w)
        nq = Hqk * dk
        assert W.shape == (2 * nq + Hv * dv, 4)
        h = [None] * 3
        if conv_state is not None:
            hs = _f64(conv_state)
            h = [hs[:, :, :nq], hs[:, :, nq:2 * nq], hs[:, :, 2 * nq:]]
        q = causal_conv4(q.reshape(B, T, nq), W[:nq], h[0]).reshape(q.shape)
        k = causal_conv4(k.reshape(B, T, nq), W[nq:2 * nq], h[1]).reshape(k.shape)
        v = causal_conv4(v.reshape(B, T, Hv * dv), W[2 * nq:], h[2]).reshape(v.shape)
    if l2norm_qk:
        q = l2norm(q)
        k = l2norm(k)
    return q, k, v


def gates_from_logits(x):
    """σ(x) = 1 / (1 + e^(−x)) elementwise, float64 (x: gate logits)."""
    x = _f64(x)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def rel_err(got, ref) -> float:
    """max |got - ref| / RMS(ref): the parity metric for every floating output."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    err = float(np.max(np.abs(got - ref)))
    return err / rms if rms > 0 else err
