"""Helpers shared by the GPU parity tests: run the oracle on the same inputs the
CUDA path sees and compare with the max|err|/RMS(ref) metric."""

import numpy as np
import torch

import oracle

TOL_FP32 = 1e-4   # fp32 path
TOL_BF16 = 2e-2   # bf16 operands, fp32 accumulate


def np64(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.astype(np.float64, copy=False)
    return t.detach().to(torch.float64).cpu().numpy()


def oracle_gates(mode, alpha, b, w, d_k, d_v, gate_logits=False, H_v=None, head_axis=2):
    """Per-channel float64 gates for the oracle from the tensors the kernel gets
    (bf16 logits pass through the oracle's sigmoid first; with ``H_v``, alpha
    and b are owned by QK heads and given to each value head of the group)."""
    f = oracle.gates_from_logits if gate_logits else (lambda x: x)
    alpha, b = f(np64(alpha)), f(np64(b))
    w = None if w is None else f(np64(w))
    if H_v is not None:
        alpha = oracle.gates_for_value_heads(alpha, H_v, head_axis)
        b = oracle.gates_for_value_heads(b, H_v, head_axis)
    if mode == "full":
        return alpha, b, w
    return oracle.expand_tied_gates(mode, alpha, b, d_k, d_v)


def oracle_chunk(inp, gate_mode="full", scale=1.0, l2norm_qk=False, S0=None, threads=0,
                 heads=None, gate_logits=False, conv_state=None, gates_per_qk_head=False):
    """Oracle (o, S_T) for a chunk_fwd input dict (``conv_state``: the conv
    history before token 0, or None). ``heads`` optionally restricts to a list of
    (sequence, value head) pairs; returns dict keyed by pair then."""
    q, k, v = np64(inp["q"]), np64(inp["k"]), np64(inp["v"])
    d_k, d_v = q.shape[-1], v.shape[-1]
    conv_w = np64(inp.get("conv_w"))
    conv_state = np64(conv_state)
    S0 = np64(inp.get("S0")) if S0 is None else np64(S0)
    alpha, b, w = oracle_gates(gate_mode, inp["alpha"], inp["b"], inp.get("w"), d_k, d_v, gate_logits,
                               H_v=v.shape[2] if gates_per_qk_head else None)
    if heads is None:
        qp, kp, vp = oracle.preprocess(q, k, v, conv_w, l2norm_qk, conv_state)
        return oracle.gdn2_forward(qp, kp, vp, alpha, b, w, S0, scale=scale, threads=threads)
    assert conv_state is None, "per-head oracle runs take no conv history"
    Hqk, Hv = q.shape[2], v.shape[2]
    g = Hv // Hqk
    out = {}
    for (bi, h) in heads:
        hq = h // g
        qh, kh = q[bi:bi + 1, :, hq:hq + 1], k[bi:bi + 1, :, hq:hq + 1]
        vh = v[bi:bi + 1, :, h:h + 1]
        cw = None
        if conv_w is not None:
            n = Hqk * d_k
            cw = np.concatenate([conv_w[hq * d_k:(hq + 1) * d_k], conv_w[n + hq * d_k:n + (hq + 1) * d_k],
                                 conv_w[2 * n + h * d_v:2 * n + (h + 1) * d_v]])
        qp, kp, vp = oracle.preprocess(qh, kh, vh, cw, l2norm_qk)
        s0 = None if S0 is None else S0[bi:bi + 1, h:h + 1]
        out[(bi, h)] = oracle.gdn2_forward(qp, kp, vp, alpha[bi:bi + 1, :, h:h + 1], b[bi:bi + 1, :, h:h + 1],
                                           w[bi:bi + 1, :, h:h + 1], s0, scale=scale, threads=threads)
    return out


def to_cuda(inp):
    return {k_: (None if t is None else t.cuda()) for k_, t in inp.items()}


def assert_bf16_rounding(o_bf16, o_f32, what):
    """A bf16 output must be the fp32 result rounded to nearest bf16 (1 ulp slack):
    the tolerance bar applies to the kernel's arithmetic, and rounding the output
    to bf16 adds at most 2^-9 relative per element on top of it."""
    assert o_bf16.dtype == torch.bfloat16 and o_f32.dtype == torch.float32
    diff = (o_bf16.float() - o_f32.to(torch.bfloat16).float()).abs()
    ulp = o_f32.abs() * 2.0 ** -7 + 1e-30
    bad = int((diff > ulp).sum())
    assert bad == 0, f"{what}: {bad} bf16 outputs are not the rounded fp32 result"


def assert_close(got, ref, tol, what):
    err = oracle.rel_err(np64(got) if torch.is_tensor(got) else got, ref)
    assert np.isfinite(err) and err <= tol, f"{what}: max|err|/RMS(ref) = {err:.3e} > {tol:.1e}"
    return err


def split_packed(inp, cu, n):
    """Sequence n of a packed input dict ([1, T, ...] tensors, offsets cu) as
    its own one-sequence input dict (S0 row n). Fresh copies: a slice of a
    per-token scalar gate can start off the 16-byte alignment the C calls ask
    for."""
    t0, t1 = int(cu[n]), int(cu[n + 1])
    out = {}
    for key, t in inp.items():
        if t is None or key == "conv_w":
            out[key] = t
        elif key == "S0":
            out[key] = t[n:n + 1].clone()
        else:
            out[key] = t[:, t0:t1].clone()
    return out


def oracle_packed(inp, cu, conv_state=None, **kw):
    """Oracle (o [1,T,H_v,d_v], S_T [N,H_v,d_k,d_v]) of packed sequences: each
    sequence on its own, from its own state and conv history."""
    N = len(cu) - 1
    os_, Ss = [], []
    for n in range(N):
        part = split_packed(inp, cu, n)
        hist = None if conv_state is None else conv_state[n:n + 1]
        o, S = oracle_chunk(part, conv_state=hist, **kw)
        os_.append(o)
        Ss.append(S)
    return np.concatenate(os_, axis=1), np.concatenate(Ss, axis=0)
