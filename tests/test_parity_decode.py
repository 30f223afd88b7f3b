"""Recurrent decode step (gdn2_decode_step) against the float64 oracle."""

from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_gdn_b200 import gdn2
from delta_rule_linear_gdn_b200.inputs import make_decode_pool, make_inputs, workload
from tests.gpu_util import TOL_BF16, TOL_FP32, assert_bf16_rounding, assert_close, np64, oracle_gates

pytestmark = pytest.mark.gpu


def _step_inputs(inp, t):
    return {k: (None if v is None else v[:, t].contiguous()) for k, v in inp.items()
            if k in ("q", "k", "v", "alpha", "b", "w")}


@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
@pytest.mark.parametrize("qkv", ["f32", "bf16"])
def test_decode_steps_vs_oracle(d, gate_mode, qkv):
    w = replace(workload(0), B=3, T=5, H_qk=2, H_v=6, d=d, qkv_dtype=qkv, s0="normal")
    inp = make_inputs(w, seed=d + 1, gate_mode=gate_mode)
    S = inp["S0"].cuda().clone()
    outs = []
    for t in range(w.T):
        s = {k: (None if v is None else v.cuda()) for k, v in _step_inputs(inp, t).items()}
        outs.append(gdn2.decode_step(s["q"], s["k"], s["v"], s["alpha"], s["b"], s["w"], S,
                                     gate_mode=gate_mode, o_dtype=torch.float32))
    torch.cuda.synchronize()
    a, b, w_ = oracle_gates(gate_mode, inp["alpha"], inp["b"], inp["w"], d, d)
    o_ref, S_ref = oracle.gdn2_forward(np64(inp["q"]), np64(inp["k"]), np64(inp["v"]), a, b, w_,
                                       np64(inp["S0"]))
    assert_close(torch.stack(outs, 1), o_ref, TOL_FP32, "o")
    assert_close(S, S_ref, TOL_FP32, "S")


@pytest.mark.parametrize("d", [16, 128])
@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
def test_decode_gate_logits_vs_oracle(d, gate_mode):
    """Gates given as bf16 logits (the kernel applies the sigmoid): the oracle
    takes σ of the same logits in float64."""
    w = replace(workload(0), B=3, T=5, H_qk=2, H_v=6, d=d, qkv_dtype="bf16", s0="normal")
    inp = make_inputs(w, seed=d + 7, gate_mode=gate_mode, gate_logits=True)
    assert inp["alpha"].dtype == torch.bfloat16
    S = inp["S0"].cuda().clone()
    outs = []
    for t in range(w.T):
        s = {k: (None if v is None else v.cuda()) for k, v in _step_inputs(inp, t).items()}
        outs.append(gdn2.decode_step(s["q"], s["k"], s["v"], s["alpha"], s["b"], s["w"], S,
                                     gate_mode=gate_mode, o_dtype=torch.float32, gate_logits=True))
    torch.cuda.synchronize()
    a, b, w_ = oracle_gates(gate_mode, inp["alpha"], inp["b"], inp["w"], d, d, gate_logits=True)
    o_ref, S_ref = oracle.gdn2_forward(np64(inp["q"]), np64(inp["k"]), np64(inp["v"]), a, b, w_,
                                       np64(inp["S0"]))
    assert_close(torch.stack(outs, 1), o_ref, TOL_FP32, "o")
    assert_close(S, S_ref, TOL_FP32, "S")


def test_decode_l2norm_and_scale_bf16_out():
    w = replace(workload(0), B=4, T=3, H_qk=1, H_v=3, d=128, qkv_dtype="bf16", s0="normal", conv=True)
    inp = make_inputs(w, seed=3)   # conv=True: raw (unnormalised) q, k
    S = inp["S0"].cuda().clone()
    s = 128 ** -0.5
    outs = []
    for t in range(w.T):
        st = {k: (None if v is None else v.cuda()) for k, v in _step_inputs(inp, t).items()}
        S16 = S.clone()
        o16 = gdn2.decode_step(st["q"], st["k"], st["v"], st["alpha"], st["b"], st["w"], S16,
                               scale=s, l2norm_qk=True)
        outs.append(gdn2.decode_step(st["q"], st["k"], st["v"], st["alpha"], st["b"], st["w"], S,
                                     scale=s, l2norm_qk=True, o_dtype=torch.float32))
        torch.cuda.synchronize()
        assert_bf16_rounding(o16, outs[-1], f"o bf16 step {t}")
        torch.testing.assert_close(S16, S, rtol=0, atol=0)
    q, k, v = oracle.preprocess(np64(inp["q"]), np64(inp["k"]), np64(inp["v"]), None, True)
    o_ref, S_ref = oracle.gdn2_forward(q, k, v, np64(inp["alpha"]), np64(inp["b"]), np64(inp["w"]),
                                       np64(inp["S0"]), scale=s)
    assert_close(torch.stack(outs, 1), o_ref, TOL_FP32, "o")
    assert_close(S, S_ref, TOL_FP32, "S")


def test_decode_zero_batch_is_a_no_op():
    q = torch.empty((0, 1, 16), device="cuda")
    v = torch.empty((0, 1, 16), device="cuda")
    g = torch.empty((0, 1, 16), device="cuda")
    S = torch.empty((0, 1, 16, 16), device="cuda")
    o = gdn2.decode_step(q, q, v, g, g, g, S)
    assert o.shape == (0, 1, 16)


def test_full_size_decode_b256():
    """The decode workload in the bench's launch configuration: B=256, 16/48
    heads, d=128, bf16 q,k,v, fp32 state. Step 1 is checked on the whole
    tensor; all 1000 consecutive steps of the workload are checked on 8
    sequences (sequences are independent, so the subset check is exact)."""
    w = workload("decode_b256")
    pool = make_decode_pool(w, pool=16, device="cuda")
    S = pool["S0"].clone()
    S0 = np64(pool["S0"])
    steps = w.decode_steps
    seqs = [0, 1, 37, 100, 128, 200, 254, 255]
    sel = torch.tensor(seqs, device="cuda")
    outs = []
    o1 = None
    for t in range(steps):
        i = t % 16
        if t == 0:
            # the bench's launch (bf16 o) and the same step with fp32 o, from the same state
            S_copy = S.clone()
            o16 = gdn2.decode_step(pool["q"][i], pool["k"][i], pool["v"][i], pool["alpha"][i],
                                   pool["b"][i], pool["w"][i], S_copy)
        o = gdn2.decode_step(pool["q"][i], pool["k"][i], pool["v"][i], pool["alpha"][i],
                             pool["b"][i], pool["w"][i], S, o_dtype=torch.float32)
        outs.append(o.index_select(0, sel))
        if t == 0:
            torch.cuda.synchronize()
            S1 = np64(S)
            o1 = o.clone()
            assert_bf16_rounding(o16, o, "o bf16 step 1")
            torch.testing.assert_close(S_copy, S, rtol=0, atol=0)
            del S_copy
    torch.cuda.synchronize()
    # step 1 on the whole tensor
    x = {k: np64(pool[k][0])[:, None] for k in ("q", "k", "v", "alpha", "b", "w")}
    o1_ref, S1_ref = oracle.gdn2_forward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], S0)
    assert_close(o1, o1_ref[:, 0], TOL_FP32, "o step 1")
    assert_close(S1, S1_ref, TOL_FP32, "S step 1")
    # every step on a subset of sequences
    idx = [t % 16 for t in range(steps)]
    xs = {k: np.stack([np64(pool[k][i])[seqs] for i in idx], axis=1) for k in ("q", "k", "v", "alpha", "b", "w")}
    o_ref, S_ref = oracle.gdn2_forward(xs["q"], xs["k"], xs["v"], xs["alpha"], xs["b"], xs["w"], S0[seqs])
    got = torch.stack(outs, 1)
    assert_close(got, o_ref, TOL_FP32, f"o {steps} steps")
    assert_close(S[seqs], S_ref, TOL_FP32, f"S {steps} steps")
