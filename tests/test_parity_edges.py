"""The method's degenerate and extreme cases on every CUDA path: the
tensor-core prefill, the fp32 prefill and decode, each against the float64
oracle on the same inputs, and against a closed form where the pages give one.

Cases ("Uma análise das variantes de atenção linear da família DeltaNet",
sections "Da atenção de complexidade quadrática ao estado linear", "O problema
da escrita aditiva" and "DeltaNet: escrever o erro de previsão"; "Resumo
Técnico: Gated DeltaNet-2", Metodologia §1, the reductions):

* α ≡ 1: DeltaNet (no decay);
* α ≡ 1, b ≡ 0, w ≡ 1: additive linear attention, o_t = Σ_{i≤t} (k_iᵀ q_t) v_i;
* b ≡ 1 and q = k: the read after a full-erase write returns the write,
  o_t = S_tᵀ k_t = w_t ⊙ v_t for a unit key;
* w ≡ 0: nothing is written, the state only decays and is erased;
* strong decay: α = 1e-3 and 1e-6 on some channels for 16 or more tokens in a
  row (the tensor-core path takes such chunks through its exact kernel), and
  one head with α = 1e-3 on every channel for a whole chunk;
* bf16 gate logits of −100 (σ underflows to 0 in fp32);
* |v| = 1e5, beyond the 16-bit operand range of the tensor-core path, on the
  fp32 path."""

from dataclasses import replace

import numpy as np
import pytest
import torch

from delta_rule_linear_gdn_b200 import gdn2
from delta_rule_linear_gdn_b200.inputs import make_inputs, workload
from tests.gpu_util import TOL_BF16, TOL_FP32, assert_close, np64, oracle_chunk, to_cuda

pytestmark = pytest.mark.gpu

CASES = ["deltanet", "additive", "overwrite", "no_write", "strong_decay", "strong_decay_whole_chunk"]


def edge_inputs(case, seed=61):
    """Two sequences of 200 tokens (three full chunks and a ragged one), 2 QK /
    6 V heads, d = 128, bf16 q, k, v, nonzero entry state, per-channel gates."""
    w = replace(workload("prefill_t4096"), B=2, T=200, H_qk=2, H_v=6, s0="normal")
    inp = make_inputs(w, seed=seed)
    a, b, wg = inp["alpha"], inp["b"], inp["w"]
    if case == "deltanet":
        a = torch.ones_like(a)
    elif case == "additive":
        a, b, wg = torch.ones_like(a), torch.zeros_like(b), torch.ones_like(wg)
    elif case == "overwrite":
        b = torch.ones_like(b)
        inp["q"] = inp["k"].clone()
    elif case == "no_write":
        wg = torch.zeros_like(wg)
    elif case == "strong_decay":
        a = a.clone()
        a[:, 40:80, :, 0:16] = 1e-3        # 40 tokens across a chunk boundary
        a[:, 100:140, 1::2, 64:96] = 1e-6  # odd heads, 40 tokens
    elif case == "strong_decay_whole_chunk":
        a = a.clone()
        a[0, 64:128, 2, :] = 1e-3          # one head, every channel, chunk 1
    else:
        raise ValueError(case)
    inp.update(alpha=a.contiguous(), b=b.contiguous(), w=wg.contiguous())
    return inp


def _prefill(c, **kw):
    o, S = gdn2.chunk_fwd(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], c["S0"], chunk=64,
                          o_dtype=torch.float32, **kw)
    torch.cuda.synchronize()
    return o, S


def _closed_forms(case, inp, o, tol):
    if case == "overwrite":
        # o_t = S_tᵀ k_t = w_t ⊙ v_t (unit keys: the call normalises them, so
        # only the kernel's rounding of the unit key is left)
        z = np64(inp["w"]) * np64(inp["v"])
        assert_close(o, z, tol, "o = w ⊙ v after a full-erase write")
    if case == "additive":
        q, k, v = (np64(inp[n]) for n in ("q", "k", "v"))
        S0 = np64(inp["S0"])
        g = v.shape[2] // q.shape[2]
        qh = np.repeat(q, g, axis=2)
        kh = np.repeat(k, g, axis=2)
        # o_t = S0ᵀ q_t + Σ_{i≤t} (k_i · q_t) v_i
        scores = np.einsum("bthd,bshd->bhts", qh, kh)
        scores *= np.tril(np.ones(scores.shape[-2:]))[None, None]
        ref = np.einsum("bhts,bshd->bthd", scores, v) + np.einsum("bhkd,bthk->bthd", S0, qh)
        assert_close(o, ref, tol, "o = additive linear attention")


@pytest.mark.parametrize("case", CASES)
def test_tensor_core_prefill_edges(case):
    inp = edge_inputs(case)
    l2 = case == "overwrite"     # unit keys for the closed form
    o, S = _prefill(to_cuda(inp), l2norm_qk=l2)
    o_ref, S_ref = oracle_chunk(inp, l2norm_qk=l2)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    assert_close(o, o_ref, TOL_BF16, f"{case}: o")
    assert_close(S, S_ref, TOL_BF16, f"{case}: S_T")
    _closed_forms(case, inp, o, TOL_BF16)


@pytest.mark.parametrize("case", CASES)
def test_fp32_prefill_edges(case):
    inp = edge_inputs(case)
    l2 = case == "overwrite"
    o, S = _prefill(to_cuda(inp), precision="fp32", l2norm_qk=l2)
    o_ref, S_ref = oracle_chunk(inp, l2norm_qk=l2)
    assert_close(o, o_ref, TOL_FP32, f"{case}: o")
    assert_close(S, S_ref, TOL_FP32, f"{case}: S_T")
    _closed_forms(case, inp, o, TOL_FP32)


@pytest.mark.parametrize("case", CASES)
def test_decode_edges(case):
    """The first 70 tokens as 70 decode steps (fp32 arithmetic: the fp32 bar)."""
    inp = edge_inputs(case)
    T = 70
    inp = {k: (t[:, :T].contiguous() if t is not None and k not in ("S0", "conv_w") else t) for k, t in inp.items()}
    c = to_cuda(inp)
    S = c["S0"].clone()
    outs = []
    for t in range(T):
        outs.append(gdn2.decode_step(c["q"][:, t].contiguous(), c["k"][:, t].contiguous(), c["v"][:, t].contiguous(),
                                     c["alpha"][:, t].contiguous(), c["b"][:, t].contiguous(),
                                     c["w"][:, t].contiguous(), S, o_dtype=torch.float32))
    torch.cuda.synchronize()
    o = torch.stack(outs, 1)
    o_ref, S_ref = oracle_chunk(inp)
    assert_close(o, o_ref, TOL_FP32, f"{case}: o")
    assert_close(S, S_ref, TOL_FP32, f"{case}: S")


def test_strong_decay_long_sequence_pipelined():
    """Strong decay through the pipelined schedule (few heads, 80 chunks): the
    exact kernel runs between each segment's prep and its scan."""
    w = replace(workload("prefill_t4096"), T=64 * 80 + 21, H_qk=2, H_v=6, s0="normal")
    inp = make_inputs(w, seed=67)
    a = inp["alpha"].clone()
    a[:, 1000:1100, :, 0:32] = 1e-3
    a[:, 3000:3064, 4, :] = 1e-6
    a[:, 5000:, 5, 100:] = 1e-4
    inp["alpha"] = a
    o, S = _prefill(to_cuda(inp))
    o_ref, S_ref = oracle_chunk(inp)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(S, S_ref, TOL_BF16, "S_T")


@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
def test_logit_floor(gate_mode):
    """Logits of −100 (σ = 0 in fp32) on some channels / tokens: both prefill
    paths and decode stay finite and match the oracle on σ of the logits."""
    w = replace(workload("prefill_t4096"), B=1, T=150, H_qk=2, H_v=6, s0="normal")
    inp = make_inputs(w, seed=71, gate_mode=gate_mode, gate_logits=True)
    a = inp["alpha"].clone()
    if gate_mode == "gdn":
        a[:, 10:40, 0] = -100.0
    else:
        a[:, 10:40, :, 0:8] = -100.0
    inp["alpha"] = a
    c = to_cuda(inp)
    kw = dict(gate_mode=gate_mode, gate_logits=True)
    o, S = _prefill(c, **kw)
    o32, S32 = _prefill(c, precision="fp32", **kw)
    o_ref, S_ref = oracle_chunk(inp, gate_mode=gate_mode, gate_logits=True)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(S, S_ref, TOL_BF16, "S_T")
    assert_close(o32, o_ref, TOL_FP32, "o fp32 path")
    assert_close(S32, S_ref, TOL_FP32, "S_T fp32 path")


def test_large_values_fp32_path():
    """|v| = 1e5 is beyond the tensor-core path's fp16 operands (a stated
    precondition); the fp32 path takes it at the fp32 bar."""
    inp = edge_inputs("deltanet", seed=73)
    inp["v"] = (inp["v"].float() * 1e5).to(torch.bfloat16)
    inp["S0"] = inp["S0"] * 1e5
    o, S = _prefill(to_cuda(inp), precision="fp32")
    o_ref, S_ref = oracle_chunk(inp)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(S, S_ref, TOL_FP32, "S_T")


def test_device_status_reports_a_wait_that_gave_up():
    """The failure path without a fault: the test hook makes every scan of
    the tensor-core prefill wait on a barrier nothing signals, before it
    issues any product; the scan gives up, drains its copies, frees its
    tensor memory and sets the status word, which gdn2_chunk_fwd_status reads
    as GDN2_ERR_TIMEOUT. The context stays usable: the next call, with the
    hook off, is correct and reports GDN2_OK."""
    inp = edge_inputs("deltanet", seed=79)
    c = to_cuda(inp)
    args = (c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], c["S0"])
    p = gdn2.make_params(2, 200, 2, 6, 128, 128, chunk=64)
    ws = torch.empty(gdn2.chunk_fwd_workspace(p), dtype=torch.uint8, device="cuda")
    try:
        gdn2.debug_set_scan_stall(256)
        gdn2.chunk_fwd(*args, chunk=64, o_dtype=torch.float32, workspace=ws)
        assert gdn2.chunk_fwd_status(ws) == gdn2.ERR_TIMEOUT
        o_n = torch.empty((2, 200, 6, 128), device="cuda")
        gdn2.chunk_fwd_noalloc(*args, o=o_n, chunk=64)
        assert gdn2.chunk_fwd_noalloc_status() == gdn2.ERR_TIMEOUT
    finally:
        gdn2.debug_set_scan_stall(0)
    o, S = gdn2.chunk_fwd(*args, chunk=64, o_dtype=torch.float32, workspace=ws)
    assert gdn2.chunk_fwd_status(ws) == gdn2.OK
    o_ref, S_ref = oracle_chunk(inp)
    assert_close(o, o_ref, TOL_BF16, "o after the failure")
    assert_close(S, S_ref, TOL_BF16, "S_T after the failure")
    gdn2.chunk_fwd_noalloc(*args, o=o_n, chunk=64)
    assert gdn2.chunk_fwd_noalloc_status() == gdn2.OK
    assert_close(o_n, o_ref, TOL_BF16, "noalloc o after the failure")
    assert gdn2.chunk_fwd_status(None) == gdn2.OK
