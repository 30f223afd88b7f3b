"""Decay and erase gates shared per query/key head (gates_per_qk_head): every
path against the float64 oracle, and bit for bit against the same call with
each gate row repeated for the value heads of its group."""

from dataclasses import replace

import pytest
import torch

from delta_rule_linear_gdn_b200 import gdn2
from delta_rule_linear_gdn_b200.inputs import make_decode_pool, make_inputs, workload
from tests.gpu_util import TOL_BF16, TOL_FP32, assert_close, np64, oracle_chunk, oracle_gates, to_cuda

import oracle

pytestmark = pytest.mark.gpu


def repeated(c, H_v, axis=2):
    """The per-QK-head alpha and b given to every value head of the group."""
    out = dict(c)
    for key in ("alpha", "b"):
        g = c[key]
        out[key] = g.repeat_interleave(H_v // g.shape[axis], dim=axis).contiguous()
    return out


def run(c, **kw):
    o, S = gdn2.chunk_fwd(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], c["S0"], conv_w=c["conv_w"], **kw)
    torch.cuda.synchronize()
    return o, S


CASES = [
    # (path, workload overrides, tolerance)
    ("tensor_core", dict(T=200, B=2, H_qk=2, H_v=6, d=128, chunk=64, qkv_dtype="bf16", s0="normal"), TOL_BF16),
    ("fp32", dict(T=77, B=2, H_qk=2, H_v=4, d=32, chunk=16, qkv_dtype="f32", s0="normal"), TOL_FP32),
]


@pytest.mark.parametrize("path,over,tol", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
def test_chunk_qk_gates(path, over, tol, gate_mode):
    w = replace(workload(0), **over)
    inp = make_inputs(w, seed=60, gate_mode=gate_mode, gates_per_qk_head=True)
    assert inp["alpha"].shape[2] == w.H_qk
    c = to_cuda(inp)
    kw = dict(chunk=w.chunk, gate_mode=gate_mode, o_dtype=torch.float32)
    o, S = run(c, gates_per_qk_head=True, **kw)
    o_rep, S_rep = run(repeated(c, w.H_v), **kw)
    torch.testing.assert_close(o, o_rep, rtol=0, atol=0)
    torch.testing.assert_close(S, S_rep, rtol=0, atol=0)
    o_ref, S_ref = oracle_chunk(inp, gate_mode=gate_mode, gates_per_qk_head=True)
    assert_close(o, o_ref, tol, "o")
    assert_close(S, S_ref, tol, "S_T")


@pytest.mark.parametrize("gate_logits", [False, True])
def test_qk_gates_long_sequence_overlapped(gate_logits):
    """A sequence long enough for the pipelined segments (the α tile of each
    item by TMA from the QK head's rows), with gate values and with logits."""
    w = replace(workload("prefill_t4096"), T=4096 + 37, H_qk=2, H_v=6, s0="normal")
    inp = make_inputs(w, seed=61, gate_logits=gate_logits, gates_per_qk_head=True)
    c = to_cuda(inp)
    kw = dict(chunk=64, gate_logits=gate_logits)
    o, S = run(c, gates_per_qk_head=True, **kw)
    o_rep, S_rep = run(repeated(c, w.H_v), **kw)
    torch.testing.assert_close(o, o_rep, rtol=0, atol=0)
    torch.testing.assert_close(S, S_rep, rtol=0, atol=0)
    heads = [(0, 0), (0, 4)]
    ref = oracle_chunk(inp, heads=heads, gate_logits=gate_logits, gates_per_qk_head=True)
    for (bi, h) in heads:
        o_ref, S_ref = ref[(bi, h)]
        assert_close(o[bi:bi + 1, :, h:h + 1].float(), o_ref, TOL_BF16, f"o[{bi},{h}]")
        assert_close(S[bi:bi + 1, h:h + 1], S_ref, TOL_BF16, f"S_T[{bi},{h}]")


@pytest.mark.parametrize("d,qkv", [(128, "bf16"), (32, "f32")])
@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
def test_decode_qk_gates(d, qkv, gate_mode):
    w = replace(workload("decode_b64"), B=3, H_qk=2, H_v=6, d=d, qkv_dtype=qkv)
    pool = make_decode_pool(w, pool=2, seed=62, gate_mode=gate_mode, gates_per_qk_head=True)
    step = {k_: (None if pool[k_] is None else pool[k_][0].cuda()) for k_ in ("q", "k", "v", "alpha", "b", "w")}
    S0 = pool["S0"].cuda()
    S1, S2 = S0.clone(), S0.clone()
    o = gdn2.decode_step(step["q"], step["k"], step["v"], step["alpha"], step["b"], step["w"], S1,
                         gate_mode=gate_mode, o_dtype=torch.float32, gates_per_qk_head=True)
    rep = repeated(step, w.H_v, axis=1)
    o_rep = gdn2.decode_step(rep["q"], rep["k"], rep["v"], rep["alpha"], rep["b"], rep["w"], S2,
                             gate_mode=gate_mode, o_dtype=torch.float32)
    torch.cuda.synchronize()
    torch.testing.assert_close(o, o_rep, rtol=0, atol=0)
    torch.testing.assert_close(S1, S2, rtol=0, atol=0)
    a, b, w_ = oracle_gates(gate_mode, step["alpha"], step["b"], step["w"], d, d, H_v=w.H_v, head_axis=1)
    o_ref, S_ref = oracle.gdn2_forward(np64(step["q"])[:, None], np64(step["k"])[:, None], np64(step["v"])[:, None],
                                       a[:, None], b[:, None], w_[:, None], np64(S0))
    assert_close(o, o_ref[:, 0], TOL_FP32, "decode o")
    assert_close(S1, S_ref, TOL_FP32, "decode S")


def test_binding_rejects_gates_of_the_wrong_heads():
    """Per-value-head gates passed as per-QK-head ones (or the reverse) are
    refused before any launch: the kernels would index past them."""
    w = replace(workload(0), T=16, B=1, H_qk=1, H_v=2, d=16, chunk=16)
    c = to_cuda(make_inputs(w, seed=63))
    with pytest.raises(ValueError):
        run(c, chunk=16, gates_per_qk_head=True)
    cq = to_cuda(make_inputs(w, seed=63, gates_per_qk_head=True))
    with pytest.raises(ValueError):
        run(cq, chunk=16)


def test_noalloc_with_qk_gates():
    """The allocation-free call with gates per QK head: 79 chunks of 6
    sequence-heads do not fit its 32 MiB scratch (74 do), so it runs in plain
    segments; same results as the workspace call, bit for bit."""
    w = replace(workload("prefill_t4096"), T=5000, H_qk=2, H_v=6, s0="normal")
    inp = make_inputs(w, seed=64, gates_per_qk_head=True)
    c = to_cuda(inp)
    o, S = run(c, chunk=64, gates_per_qk_head=True)
    o2 = torch.empty_like(o)
    S2 = torch.empty_like(S)
    gdn2.chunk_fwd_noalloc(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], c["S0"], o=o2, S_T=S2,
                           chunk=64, gates_per_qk_head=True)
    torch.cuda.synchronize()
    torch.testing.assert_close(o2, o, rtol=0, atol=0)
    torch.testing.assert_close(S2, S, rtol=0, atol=0)


@pytest.mark.parametrize("gate_mode", ["kda", "gdn"])
@pytest.mark.parametrize("gate_logits", [False, True])
@pytest.mark.parametrize("qk", [False, True])
def test_tied_gates_by_tma_box(gate_mode, gate_logits, qk):
    """The layer's head counts (16 QK / 48 V heads): a row of gates is a
    multiple of 16 bytes, so the tensor-core prep takes the tied layouts'
    scalar gates (β, and α in the Gated DeltaNet layout) by TMA boxes one item
    ahead. Two sequences with a ragged tail, values and logits, gates per value
    head and per QK head (bit for bit the same call with the rows repeated),
    every head against the oracle."""
    w = replace(workload("prefill_t4096"), T=200, B=2, s0="normal")
    inp = make_inputs(w, seed=62, gate_mode=gate_mode, gate_logits=gate_logits, gates_per_qk_head=qk)
    c = to_cuda(inp)
    kw = dict(chunk=64, gate_mode=gate_mode, gate_logits=gate_logits, o_dtype=torch.float32)
    o, S = run(c, gates_per_qk_head=qk, **kw)
    if qk:
        o_rep, S_rep = run(repeated(c, w.H_v), **kw)
        torch.testing.assert_close(o, o_rep, rtol=0, atol=0)
        torch.testing.assert_close(S, S_rep, rtol=0, atol=0)
    o_ref, S_ref = oracle_chunk(inp, gate_mode=gate_mode, gate_logits=gate_logits, gates_per_qk_head=qk)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(S, S_ref, TOL_BF16, "S_T")
