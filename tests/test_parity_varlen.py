"""Sequences of different lengths packed along T (cu_seqlens): each sequence
starts its own chunks, state and conv history. Both prefill paths against the
float64 oracle run sequence by sequence, and bit for bit against separate
calls, one per sequence."""

from dataclasses import replace

import numpy as np
import pytest
import torch

from delta_rule_linear_gdn_b200 import gdn2
from delta_rule_linear_gdn_b200.inputs import make_conv_state, make_inputs, workload
from tests.gpu_util import (TOL_BF16, TOL_FP32, assert_close, np64, oracle_packed, split_packed, to_cuda)

import oracle

pytestmark = pytest.mark.gpu

PATHS = {
    "tensor_core": (dict(H_qk=2, H_v=6, d=128, chunk=64, qkv_dtype="bf16"), TOL_BF16),
    "fp32": (dict(H_qk=2, H_v=4, d=32, chunk=16, qkv_dtype="f32"), TOL_FP32),
}


def packed_inputs(path, lens, seed, conv=False, **kw):
    """Seeded inputs for sequences of lengths ``lens`` packed into one row,
    with one initial state per sequence."""
    over, tol = PATHS[path]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(int).tolist()
    w = replace(workload(0), B=1, T=cu[-1], s0="zeros", conv=conv, **over)
    inp = make_inputs(w, seed=seed, **kw)
    ws = replace(w, B=len(lens), T=1, s0="normal")
    inp["S0"] = make_inputs(ws, seed=seed + 1)["S0"]
    return w, cu, inp, tol


def run(c, cu=None, **kw):
    o, S = gdn2.chunk_fwd(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], c["S0"], conv_w=c["conv_w"],
                          o_dtype=torch.float32, cu_seqlens=cu, **kw)
    return o, S


def separate(c, cu, hist=None, hist_out=None, **kw):
    """One call per sequence: o concatenated, S_T stacked, histories written."""
    os_, Ss = [], []
    for n in range(len(cu) - 1):
        part = split_packed(c, cu, n)
        o, S = run(part, conv_state_in=None if hist is None else hist[n:n + 1].clone(),
                   conv_state_out=None if hist_out is None else hist_out[n:n + 1], **kw)
        os_.append(o)
        Ss.append(S)
    return torch.cat(os_, 1), torch.cat(Ss, 0)


@pytest.mark.parametrize("path", ["tensor_core", "fp32"])
@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
def test_packed_equals_separate_and_oracle(path, gate_mode):
    """Lengths with ragged tails, an empty sequence and a one-token sequence."""
    lens = [130, 0, 1, 200, 64]
    w, cu, inp, tol = packed_inputs(path, lens, seed=70, gate_mode=gate_mode)
    c = to_cuda(inp)
    kw = dict(chunk=w.chunk, gate_mode=gate_mode)
    o, S = run(c, cu, **kw)
    o_sep, S_sep = separate(c, cu, **kw)
    torch.cuda.synchronize()
    torch.testing.assert_close(o, o_sep, rtol=0, atol=0)
    torch.testing.assert_close(S, S_sep, rtol=0, atol=0)
    torch.testing.assert_close(S[1], c["S0"][1], rtol=0, atol=0)     # the empty sequence keeps its state
    o_ref, S_ref = oracle_packed(inp, cu, gate_mode=gate_mode)
    assert_close(o, o_ref, tol, "o")
    assert_close(S, S_ref, tol, "S_T")


@pytest.mark.parametrize("path", ["tensor_core", "fp32"])
def test_packed_conv_histories(path):
    """Conv + L2 norm in the prep's load: at every sequence start the conv reads
    that sequence's own history (never the previous sequence's tokens), and
    each sequence's history after its last token is written."""
    lens = [70, 2, 0, 129, 5]
    w, cu, inp, tol = packed_inputs(path, lens, seed=71, conv=True)
    hist = make_conv_state(replace(w, B=len(lens)), seed=72)
    c = to_cuda(inp)
    h_in = hist.cuda()
    h_out = torch.full_like(h_in, float("nan"))
    h_sep = torch.full_like(h_in, float("nan"))
    kw = dict(chunk=w.chunk, l2norm_qk=True)
    o, S = run(c, cu, conv_state_in=h_in, conv_state_out=h_out, **kw)
    o_sep, S_sep = separate(c, cu, hist=h_in, hist_out=h_sep, **kw)
    torch.cuda.synchronize()
    torch.testing.assert_close(o, o_sep, rtol=0, atol=0)
    torch.testing.assert_close(S, S_sep, rtol=0, atol=0)
    torch.testing.assert_close(h_out, h_sep, rtol=0, atol=0)
    o_ref, S_ref = oracle_packed(inp, cu, conv_state=hist, l2norm_qk=True)
    assert_close(o, o_ref, tol, "o")
    assert_close(S, S_ref, tol, "S_T")
    for n in range(len(lens)):
        part = split_packed(inp, cu, n)
        want = oracle.conv_state_after(np64(part["q"]), np64(part["k"]), np64(part["v"]), np64(hist[n:n + 1]))
        got = h_out[n:n + 1].cpu().to(torch.float64).numpy()
        assert np.array_equal(got, want), f"history of sequence {n}"


@pytest.mark.parametrize("gate_logits", [False, True])
def test_packed_gate_layouts(gate_logits):
    """Gates per QK head, as values or logits, in a packed call."""
    lens = [100, 37, 65]
    w, cu, inp, tol = packed_inputs("tensor_core", lens, seed=73, gate_logits=gate_logits, gates_per_qk_head=True)
    c = to_cuda(inp)
    kw = dict(chunk=64, gate_logits=gate_logits, gates_per_qk_head=True)
    o, S = run(c, cu, **kw)
    o_sep, S_sep = separate(c, cu, **kw)
    torch.cuda.synchronize()
    torch.testing.assert_close(o, o_sep, rtol=0, atol=0)
    torch.testing.assert_close(S, S_sep, rtol=0, atol=0)
    o_ref, S_ref = oracle_packed(inp, cu, gate_logits=gate_logits, gates_per_qk_head=True)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(S, S_ref, TOL_BF16, "S_T")


def test_packed_long_and_many():
    """A long sequence (65 chunks, which alone would run the pipelined
    schedule) beside a short one; and the most sequences one call takes, of
    0 to 40 tokens each."""
    lens = [4100, 61]
    w, cu, inp, tol = packed_inputs("tensor_core", lens, seed=74)
    c = to_cuda(inp)
    o, S = run(c, cu, chunk=64)
    o_sep, S_sep = separate(c, cu, chunk=64)
    torch.cuda.synchronize()
    torch.testing.assert_close(o, o_sep, rtol=0, atol=0)
    torch.testing.assert_close(S, S_sep, rtol=0, atol=0)

    rng = np.random.default_rng(75)
    lens = rng.integers(0, 41, size=gdn2.MAX_SEQS).tolist()
    w, cu, inp, tol = packed_inputs("tensor_core", lens, seed=76)
    c = to_cuda(inp)
    o, S = run(c, cu, chunk=64)
    torch.cuda.synchronize()
    sample = [0, 1, 57, 200, gdn2.MAX_SEQS - 1]
    for n in sample:
        part = split_packed(inp, cu, n)
        o_ref, S_ref = oracle_packed(part, [0, cu[n + 1] - cu[n]])
        if cu[n + 1] > cu[n]:
            assert_close(o[:, cu[n]:cu[n + 1]], o_ref, TOL_BF16, f"o of sequence {n}")
        assert_close(S[n:n + 1], S_ref, TOL_BF16, f"S_T of sequence {n}")


def test_binding_shapes_for_packed_sequences():
    lens = [5, 7]
    w, cu, inp, tol = packed_inputs("fp32", lens, seed=77)
    c = to_cuda(inp)
    with pytest.raises(ValueError):     # one state for two sequences
        run(dict(c, S0=c["S0"][:1].contiguous()), cu, chunk=16)
    with pytest.raises(gdn2.GDN2Error):  # offsets that do not end at T
        run(c, [0, 5, 11], chunk=16)


def test_packed_without_states_and_fp32_arithmetic_on_bf16():
    """No initial states (zeros) and no final states requested, on the
    tensor-core path; and GDN2_PREC_FP32 on bf16 inputs (the fp32 path reads
    bf16 q, k, v) against the 1e-4 bar."""
    lens = [90, 3, 0, 70]
    w, cu, inp, tol = packed_inputs("tensor_core", lens, seed=78)
    inp["S0"] = None
    c = to_cuda(inp)
    o, S = gdn2.chunk_fwd(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], None, chunk=64,
                          o_dtype=torch.float32, cu_seqlens=cu, want_state=False)
    torch.cuda.synchronize()
    assert S is None
    o_ref, _ = oracle_packed(inp, cu)
    assert_close(o, o_ref, TOL_BF16, "o without states")
    o32, S32 = gdn2.chunk_fwd(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], None, chunk=64,
                              o_dtype=torch.float32, cu_seqlens=cu, precision="fp32")
    torch.cuda.synchronize()
    o_ref2, S_ref2 = oracle_packed(inp, cu)
    assert_close(o32, o_ref2, TOL_FP32, "o fp32 path")
    assert_close(S32, S_ref2, TOL_FP32, "S_T fp32 path")
    assert torch.count_nonzero(S32[2]) == 0                      # the empty sequence: zero state
