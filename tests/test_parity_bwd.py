"""Backward pass (gdn2_chunk_bwd) against the float64 backward oracle, element
by element on seeded inputs: the gradients of <dO, o> + <dS_T, S_T> with
respect to q, k, v, the gates and S0 ("Resumo Técnico: Gated DeltaNet-2",
Metodologia §3). The kernel's arithmetic is fp32, so every gradient is held
to the fp32 bar, 1e-4 of its RMS, on the same (bf16-rounded where the inputs
are bf16) values the kernel reads."""

from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_gdn_b200 import gdn2
from delta_rule_linear_gdn_b200.inputs import make_inputs, workload
from tests.gpu_util import TOL_FP32, assert_close, np64, oracle_gates

pytestmark = pytest.mark.gpu


def upstream(inp, seed, o_dtype, with_dst=True, device="cuda"):
    """Seeded upstream gradients dO ~ N(0,1) (in o's dtype) and dS_T ~ N(0,1)."""
    g = torch.Generator(device="cpu").manual_seed(1000 + seed)
    B, T, H_v, d_v = inp["v"].shape
    d_k = inp["q"].shape[-1]
    dO = torch.randn((B, T, H_v, d_v), generator=g).to(o_dtype)
    dST = torch.randn((B, H_v, d_k, d_v), generator=g) if with_dst else None
    return dO.to(device), (None if dST is None else dST.to(device))


def oracle_grads(inp, dO, dST, gate_mode="full", gate_logits=False, gates_per_qk_head=False, scale=1.0,
                 seqs=None):
    """Expected gradients in the library's output forms (tied: dβ in "b";
    gates per QK head: sums over the group; logits: gradients of the logits).
    ``seqs`` restricts to a list of sequences (independent recurrences)."""
    pick = (lambda t: t) if seqs is None else (lambda t: None if t is None else t[seqs])
    q, k, v = (pick(np64(inp[n])) for n in ("q", "k", "v"))
    H_qk, H_v = q.shape[2], v.shape[2]
    d_k, d_v = q.shape[-1], v.shape[-1]
    a_raw, b_raw = pick(np64(inp["alpha"])), pick(np64(inp["b"]))
    w_raw = None if inp["w"] is None else pick(np64(inp["w"]))
    alpha, b, w = oracle_gates(gate_mode, a_raw, b_raw, w_raw, d_k, d_v, gate_logits,
                               H_v=H_v if gates_per_qk_head else None)
    S0 = None if inp["S0"] is None else pick(np64(inp["S0"]))
    g = oracle.gdn2_backward(q, k, v, alpha, b, w, S0, pick(np64(dO)), None if dST is None else pick(np64(dST)),
                             scale=scale)
    da, db, dw = g["alpha"], g["b"], g["w"]
    if gate_mode != "full":
        da, db = oracle.tied_gate_grads(gate_mode, da, db, dw)
        dw = None
    if gates_per_qk_head:
        da = oracle.grads_for_qk_heads(da, H_qk)
        db = oracle.grads_for_qk_heads(db, H_qk)
    if gate_logits:
        da = oracle.logit_grads(da, a_raw)
        db = oracle.logit_grads(db, b_raw)
        dw = None if dw is None else oracle.logit_grads(dw, w_raw)
    return {"q": g["q"], "k": g["k"], "v": g["v"], "alpha": da, "b": db, "w": dw, "S0": g["S0"]}


def check(got, ref, tol, what, seqs=None):
    for name, r in ref.items():
        if r is None:
            assert got[name] is None
            continue
        gg = got[name] if seqs is None else got[name][seqs]
        assert_close(gg, r, tol, f"{what}: d{name}")


def run_bwd(inp, dO, dST, **kw):
    c = {k_: (None if t is None else t.cuda()) for k_, t in inp.items()}
    g = gdn2.chunk_bwd(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], c["S0"], dO, dST, **kw)
    torch.cuda.synchronize()
    return g


def small(T=64, B=1, H_qk=1, H_v=1, d=16, qkv="f32", s0="normal"):
    return replace(workload(0), T=T, B=B, H_qk=H_qk, H_v=H_v, d=d, qkv_dtype=qkv, s0=s0)


def test_oracle_scale_workload():
    inp = make_inputs(small(), seed=0)
    dO, dST = upstream(inp, 0, torch.float32)
    check(run_bwd(inp, dO, dST), oracle_grads(inp, dO, dST), TOL_FP32, "d16 T64")


@pytest.mark.parametrize("T", [1, 15, 17, 61, 130])
@pytest.mark.parametrize("d", [16, 32, 64])
def test_ragged_lengths_grouped_heads(T, d):
    inp = make_inputs(small(T=T, B=2, H_qk=2, H_v=6, d=d), seed=T + d)
    dO, dST = upstream(inp, T + d, torch.float32)
    check(run_bwd(inp, dO, dST), oracle_grads(inp, dO, dST), TOL_FP32, f"T{T} d{d}")


@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
@pytest.mark.parametrize("gate_logits", [False, True])
@pytest.mark.parametrize("qk_gates", [False, True])
def test_gate_forms_bf16_d128(gate_mode, gate_logits, qk_gates):
    """The layer shape (bf16 q, k, v and dO, d = 128) on a short sequence with
    a ragged tail, every gate form: tied gates, logits, gates per QK head."""
    w = small(T=200, B=2, H_qk=2, H_v=6, d=128, qkv="bf16")
    inp = make_inputs(w, seed=81, gate_mode=gate_mode, gate_logits=gate_logits, gates_per_qk_head=qk_gates)
    dO, dST = upstream(inp, 81, torch.bfloat16)
    kw = dict(gate_mode=gate_mode, gate_logits=gate_logits, gates_per_qk_head=qk_gates)
    check(run_bwd(inp, dO, dST, **kw), oracle_grads(inp, dO, dST, **kw), TOL_FP32,
          f"{gate_mode} logits={gate_logits} qk={qk_gates}")


def test_scale_no_state_gradient_and_zero_entry_state():
    w = small(T=90, B=1, H_qk=1, H_v=3, d=64, qkv="bf16", s0="zeros")
    inp = make_inputs(w, seed=83)
    dO, _ = upstream(inp, 83, torch.float32, with_dst=False)
    s = 64 ** -0.5
    check(run_bwd(inp, dO, None, scale=s), oracle_grads(inp, dO, None, scale=s), TOL_FP32, "scale, dS_T=0")


def test_strong_decay_and_edges():
    """α = 1e-3 on some channels for 40 tokens, α = 1 elsewhere on one head,
    b = 0 on another: the running products of α take every α ∈ (0, 1]."""
    w = small(T=150, B=1, H_qk=2, H_v=6, d=128, qkv="bf16")
    inp = make_inputs(w, seed=85)
    a = inp["alpha"].clone()
    a[:, 30:70, :, 0:16] = 1e-3
    a[:, :, 1] = 1.0
    inp["alpha"] = a
    b = inp["b"].clone()
    b[:, :, 2] = 0.0
    inp["b"] = b
    dO, dST = upstream(inp, 85, torch.float32)
    check(run_bwd(inp, dO, dST), oracle_grads(inp, dO, dST), TOL_FP32, "strong decay")


def test_empty_sequence():
    inp = make_inputs(small(T=0), seed=87)
    dO, dST = upstream(inp, 87, torch.float32)
    g = run_bwd(inp, dO, dST)
    torch.testing.assert_close(g["S0"], dST, rtol=0, atol=0)


def test_full_size_prefill_t4096_all_heads():
    """The T = 4096, 48-V-head layer (bf16 q, k, v, dO), every head."""
    w = workload("prefill_t4096")
    inp = make_inputs(w, seed=1, device="cuda")
    dO, dST = upstream(inp, 1, torch.bfloat16)
    g = run_bwd(inp, dO, dST)
    check(g, oracle_grads(inp, dO, dST), TOL_FP32, "T4096")


def test_training_shape_b8_t8192_sampled_sequences():
    """B = 8, T = 8192, 48 V heads, nonzero entry state (the training-shape
    workload's recurrence inputs: q, k already unit length): all heads of two
    of the eight sequences (independent recurrences, so the subset is exact)."""
    w = replace(workload("conv_prefill_b8_t8192"), conv=False)
    inp = make_inputs(w, seed=4, device="cuda")
    dO, dST = upstream(inp, 4, torch.bfloat16)
    g = run_bwd(inp, dO, dST)
    seqs = [0, 5]
    check(g, oracle_grads(inp, dO, dST, seqs=seqs), TOL_FP32, "B8 T8192", seqs=seqs)
