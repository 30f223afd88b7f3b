"""Chunked prefill (gdn2_chunk_fwd) against the float64 oracle, element by
element, on seeded inputs; plus schedule-equivalence properties."""

from dataclasses import replace

import pytest
import torch

from delta_rule_linear_gdn_b200 import gdn2
from delta_rule_linear_gdn_b200.inputs import make_inputs, workload
from tests.gpu_util import TOL_BF16, TOL_FP32, assert_bf16_rounding, assert_close, np64, oracle_chunk, to_cuda

pytestmark = pytest.mark.gpu


def run(inp, **kw):
    c = to_cuda(inp)
    o, S = gdn2.chunk_fwd(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], c["S0"],
                          conv_w=c["conv_w"], **kw)
    torch.cuda.synchronize()
    return o, S


def small(T=64, B=1, H_qk=1, H_v=1, d=16, chunk=16, qkv="f32", s0="zeros", conv=False, **kw):
    return replace(workload(0), T=T, B=B, H_qk=H_qk, H_v=H_v, d=d, chunk=chunk, qkv_dtype=qkv, s0=s0,
                   conv=conv, **kw)


def test_oracle_scale_workload_fp32():
    """d=16, T=64, chunk 16, fp32: the 1e-4 bar."""
    w = workload("oracle_d16_t64")
    inp = make_inputs(w, seed=0)
    o, S = run(inp, chunk=w.chunk)
    o_ref, S_ref = oracle_chunk(inp)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(S, S_ref, TOL_FP32, "S_T")


@pytest.mark.parametrize("T", [1, 15, 17, 61, 130])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_ragged_lengths(T, chunk):
    inp = make_inputs(small(T=T, s0="normal"), seed=T)
    o, S = run(inp, chunk=chunk)
    o_ref, S_ref = oracle_chunk(inp)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(S, S_ref, TOL_FP32, "S_T")


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
def test_grouped_heads_all_dims_and_gate_modes(d, gate_mode):
    w = small(T=100, B=2, H_qk=2, H_v=6, d=d, chunk=32, s0="normal")
    inp = make_inputs(w, seed=d, gate_mode=gate_mode)
    o, S = run(inp, chunk=32, gate_mode=gate_mode, precision="fp32")
    o_ref, S_ref = oracle_chunk(inp, gate_mode=gate_mode)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(S, S_ref, TOL_FP32, "S_T")


def test_conv_and_l2norm_fused():
    w = small(T=77, B=2, H_qk=2, H_v=4, d=32, chunk=16, s0="normal", conv=True)
    inp = make_inputs(w, seed=5)
    o, S = run(inp, chunk=16, l2norm_qk=True)
    o_ref, S_ref = oracle_chunk(inp, l2norm_qk=True)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(S, S_ref, TOL_FP32, "S_T")


def test_scale_and_fp32_out_from_bf16_in():
    w = small(T=90, B=1, H_qk=1, H_v=3, d=64, chunk=64, qkv="bf16", s0="normal")
    inp = make_inputs(w, seed=6)
    s = 64 ** -0.5
    o, S = run(inp, chunk=64, scale=s, o_dtype=torch.float32, precision="fp32")
    o_ref, S_ref = oracle_chunk(inp, scale=s)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(S, S_ref, TOL_FP32, "S_T")


@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
def test_bf16_d128_chunk64(gate_mode):
    """The layer shape (bf16 in/out, d=128, chunk 64) on a short sequence with a
    ragged tail, through the default dispatch."""
    w = small(T=200, B=1, H_qk=2, H_v=6, d=128, chunk=64, qkv="bf16", s0="normal")
    inp = make_inputs(w, seed=7, gate_mode=gate_mode)
    o, S = run(inp, chunk=64, gate_mode=gate_mode, o_dtype=torch.float32)
    o_ref, S_ref = oracle_chunk(inp, gate_mode=gate_mode)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(S, S_ref, TOL_BF16, "S_T")
    o16, S16 = run(inp, chunk=64, gate_mode=gate_mode)
    assert_bf16_rounding(o16, o, "o bf16")
    torch.testing.assert_close(S16, S, rtol=0, atol=0)


@pytest.mark.parametrize("conv,gate_mode", [(True, "full"), (False, "full"), (True, "kda"), (True, "gdn")])
def test_bf16_d128_conv_and_l2norm_tensor_core(conv, gate_mode):
    """The depthwise causal conv and the L2 norm of q, k in the tensor-core
    prep's load: two sequences with a ragged tail, so the conv history
    crosses chunk boundaries but never sequence boundaries; all gate layouts."""
    w = small(T=200, B=2, H_qk=2, H_v=6, d=128, chunk=64, qkv="bf16", s0="normal", conv=True)
    inp = make_inputs(w, seed=31, gate_mode=gate_mode)
    if not conv:
        inp = dict(inp, conv_w=None)
    o, S = run(inp, chunk=64, gate_mode=gate_mode, l2norm_qk=True, o_dtype=torch.float32)
    o_ref, S_ref = oracle_chunk(inp, gate_mode=gate_mode, l2norm_qk=True)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(S, S_ref, TOL_BF16, "S_T")
    o16, S16 = run(inp, chunk=64, gate_mode=gate_mode, l2norm_qk=True)
    assert_bf16_rounding(o16, o, "o bf16")
    torch.testing.assert_close(S16, S, rtol=0, atol=0)


def test_empty_sequence_copies_state():
    inp = make_inputs(small(T=0, s0="normal"), seed=8)
    o, S = run(inp, chunk=16)
    assert o.shape[1] == 0
    torch.testing.assert_close(S.cpu(), inp["S0"], rtol=0, atol=0)
    inp0 = make_inputs(small(T=0), seed=8)
    _, S0z = run(inp0, chunk=16)
    assert torch.count_nonzero(S0z) == 0


def test_in_place_state():
    inp = make_inputs(small(T=40, B=2, H_qk=1, H_v=2, d=32, s0="normal"), seed=9)
    c = to_cuda(inp)
    S = c["S0"].clone()
    o, S_out = gdn2.chunk_fwd(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], S, chunk=16, S_T=S)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_chunk(inp)
    assert S_out.data_ptr() == S.data_ptr()
    assert_close(S, S_ref, TOL_FP32, "S_T in place")
    assert_close(o, o_ref, TOL_FP32, "o")


def test_chunk_size_invariance_and_split_sequence():
    """Schedules of the same recurrence agree: chunk 16/32/64, and [0,T) vs
    [0,t) then [t,T) carrying the state."""
    w = small(T=150, B=1, H_qk=1, H_v=2, d=64, s0="normal")
    inp = make_inputs(w, seed=10)
    outs = [run(inp, chunk=c) for c in (16, 32, 64)]
    for o, S in outs[1:]:
        torch.testing.assert_close(o, outs[0][0], rtol=1e-5, atol=1e-5)
        torch.testing.assert_close(S, outs[0][1], rtol=1e-5, atol=1e-5)
    c = to_cuda(inp)
    t = 70
    sl = lambda x: x[:, :t].contiguous()
    sr = lambda x: x[:, t:].contiguous()
    oa, Sa = gdn2.chunk_fwd(sl(c["q"]), sl(c["k"]), sl(c["v"]), sl(c["alpha"]), sl(c["b"]), sl(c["w"]),
                            c["S0"], chunk=32)
    ob, Sb = gdn2.chunk_fwd(sr(c["q"]), sr(c["k"]), sr(c["v"]), sr(c["alpha"]), sr(c["b"]), sr(c["w"]),
                            Sa, chunk=32)
    torch.testing.assert_close(torch.cat([oa, ob], 1), outs[1][0], rtol=1e-5, atol=1e-5)
    torch.testing.assert_close(Sb, outs[1][1], rtol=1e-5, atol=1e-5)


def test_overlapped_segments_match_one_pass_and_oracle():
    """Few heads and many chunks: the call pipelines its segments (each
    segment's scan beside the next segment's prep, the state carried through
    S_T). Same results, bit for bit, as the single-pass schedule (no S_T
    requested) and as the no-alloc call, whose fixed 32 MB scratch holds about
    half the chunks and so runs in plain segments; and the oracle's within the
    bf16-path bound. Ragged tail, nonzero entry state."""
    w = small(T=64 * 70 + 37, B=1, H_qk=4, H_v=12, d=128, chunk=64, qkv="bf16", s0="normal")
    inp = make_inputs(w, seed=41)
    c = to_cuda(inp)
    args = (c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], c["S0"])
    o, S = gdn2.chunk_fwd(*args, chunk=64, o_dtype=torch.float32)
    o1, _ = gdn2.chunk_fwd(*args, chunk=64, o_dtype=torch.float32, want_state=False)
    o2, S2 = torch.empty_like(o), torch.empty_like(S)
    gdn2.chunk_fwd_noalloc(*args, o=o2, S_T=S2, chunk=64)
    torch.cuda.synchronize()
    torch.testing.assert_close(o1, o, rtol=0, atol=0)
    torch.testing.assert_close(o2, o, rtol=0, atol=0)
    torch.testing.assert_close(S2, S, rtol=0, atol=0)
    ref = oracle_chunk(inp, heads=[(0, 0), (0, 11)])
    for (bi, h), (o_ref, S_ref) in ref.items():
        assert_close(o[bi:bi + 1, :, h:h + 1], o_ref, TOL_BF16, f"o[{bi},{h}]")
        assert_close(S[bi:bi + 1, h:h + 1], S_ref, TOL_BF16, f"S_T[{bi},{h}]")


@pytest.mark.parametrize("gate_mode", ["full", "gdn"])
def test_scan_two_sequences_many_heads(gate_mode):
    """Two sequences of the 48-V-head layer (96 scan CTAs, one per sequence
    and value head). Ragged tail, nonzero entry state; sampled heads of both
    sequences against the oracle."""
    w = small(T=150, B=2, H_qk=16, H_v=48, d=128, chunk=64, qkv="bf16", s0="normal")
    inp = make_inputs(w, seed=43, gate_mode=gate_mode)
    o, S = run(inp, chunk=64, gate_mode=gate_mode, o_dtype=torch.float32)
    ref = oracle_chunk(inp, gate_mode=gate_mode, heads=[(0, 0), (0, 47), (1, 1), (1, 30)])
    for (bi, h), (o_ref, S_ref) in ref.items():
        assert_close(o[bi:bi + 1, :, h:h + 1], o_ref, TOL_BF16, f"o[{bi},{h}]")
        assert_close(S[bi:bi + 1, h:h + 1], S_ref, TOL_BF16, f"S_T[{bi},{h}]")


@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
def test_gate_logits_tensor_core_and_fp32_paths(gate_mode):
    """Gates given as bf16 logits, σ applied in the kernels: the tensor-core
    prefill (with its TMA-loaded α tile in the per-channel modes) and the fp32
    path against the oracle on σ of the same logits; ragged tail, nonzero
    entry state, two sequences."""
    w = small(T=200, B=2, H_qk=2, H_v=6, d=128, chunk=64, qkv="bf16", s0="normal")
    inp = make_inputs(w, seed=47, gate_mode=gate_mode, gate_logits=True)
    o, S = run(inp, chunk=64, gate_mode=gate_mode, o_dtype=torch.float32, gate_logits=True)
    o32, S32 = run(inp, chunk=64, gate_mode=gate_mode, o_dtype=torch.float32, gate_logits=True, precision="fp32")
    o_ref, S_ref = oracle_chunk(inp, gate_mode=gate_mode, gate_logits=True)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(S, S_ref, TOL_BF16, "S_T")
    assert_close(o32, o_ref, TOL_FP32, "o fp32 path")
    assert_close(S32, S_ref, TOL_FP32, "S_T fp32 path")


def test_gate_logits_long_sequence_overlapped():
    """Logit gates through the pipelined schedule (few heads, 80 chunks): the
    same results as the gate values σ(logits) computed ahead on the host, to
    within the two sigmoids' rounding."""
    w = small(T=64 * 80, B=1, H_qk=2, H_v=6, d=128, chunk=64, qkv="bf16", s0="normal")
    inp = make_inputs(w, seed=53, gate_logits=True)
    o, S = run(inp, chunk=64, o_dtype=torch.float32, gate_logits=True)
    vals = dict(inp, alpha=torch.sigmoid(inp["alpha"].float()), b=torch.sigmoid(inp["b"].float()),
                w=torch.sigmoid(inp["w"].float()))
    o2, S2 = run(vals, chunk=64, o_dtype=torch.float32)
    ref = oracle_chunk(inp, gate_logits=True, heads=[(0, 0), (0, 5)])
    for (bi, h), (o_ref, S_ref) in ref.items():
        assert_close(o[bi:bi + 1, :, h:h + 1], o_ref, TOL_BF16, f"o[{bi},{h}]")
        assert_close(S[bi:bi + 1, h:h + 1], S_ref, TOL_BF16, f"S_T[{bi},{h}]")
    for got, want, name in ((o, o2, "o"), (S, S2, "S_T")):
        rel = ((got - want).abs().max() / want.pow(2).mean().sqrt()).item()
        assert rel <= 5e-3, (name, rel)


def test_decode_steps_equal_chunked_prefill():
    w = small(T=48, B=2, H_qk=2, H_v=4, d=32, s0="normal")
    inp = make_inputs(w, seed=11)
    o_ref, S_ref = run(inp, chunk=16)
    c = to_cuda(inp)
    S = c["S0"].clone()
    outs = []
    for t in range(w.T):
        outs.append(gdn2.decode_step(c["q"][:, t].contiguous(), c["k"][:, t].contiguous(),
                                     c["v"][:, t].contiguous(), c["alpha"][:, t].contiguous(),
                                     c["b"][:, t].contiguous(), c["w"][:, t].contiguous(), S))
    torch.cuda.synchronize()
    torch.testing.assert_close(torch.stack(outs, 1), o_ref, rtol=1e-4, atol=1e-5)
    torch.testing.assert_close(S, S_ref, rtol=1e-4, atol=1e-5)


def test_outputs_have_no_nan_and_no_stray_writes():
    """Canary: o and S_T sit inside larger buffers whose margins must stay untouched."""
    w = small(T=33, B=1, H_qk=1, H_v=2, d=32, s0="normal")
    inp = make_inputs(w, seed=12)
    c = to_cuda(inp)
    pad = 256
    o_buf = torch.full((pad * 2 + 33 * 2 * 32,), 7.0, device="cuda")
    s_buf = torch.full((pad * 2 + 2 * 32 * 32,), 7.0, device="cuda")
    o = o_buf[pad:pad + 33 * 2 * 32].view(1, 33, 2, 32)
    S = s_buf[pad:pad + 2 * 32 * 32].view(1, 2, 32, 32)
    gdn2.chunk_fwd(c["q"], c["k"], c["v"], c["alpha"], c["b"], c["w"], c["S0"], chunk=16, o=o, S_T=S)
    torch.cuda.synchronize()
    for buf, n in ((o_buf, o.numel()), (s_buf, S.numel())):
        assert torch.all(buf[:pad] == 7.0) and torch.all(buf[pad + n:] == 7.0)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()


# ------------------------------------------------------------ full-size workloads

def _full_size(name, gate_mode="full", **kw):
    """Full-size workload in the bench's launch configuration (bf16 o), plus the
    same launch with an fp32 o that the tolerance is applied to; every head of
    every sequence against the oracle (its threads take the (sequence, head)
    recurrences in parallel on the host's cores)."""
    w = workload(name)
    inp = make_inputs(w, device="cuda", gate_mode=gate_mode)
    call = lambda od: gdn2.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"],
                                     inp["S0"], chunk=w.chunk, gate_mode=gate_mode, conv_w=inp["conv_w"],
                                     l2norm_qk=w.conv, o_dtype=od, **kw)
    o16, S16 = call(torch.bfloat16)
    o, S = call(torch.float32)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    assert_bf16_rounding(o16, o, f"{name} o bf16")
    torch.testing.assert_close(S16, S, rtol=0, atol=0)
    del o16, S16
    o_ref, S_ref = oracle_chunk(inp, gate_mode=gate_mode, l2norm_qk=w.conv)
    # the bar on the whole tensors, and on every head alone
    assert_close(o, o_ref, TOL_BF16, f"{name} o")
    assert_close(S, S_ref, TOL_BF16, f"{name} S_T")
    o, S = np64(o), np64(S)
    for bi in range(w.B):
        for h in range(w.H_v):
            assert_close(o[bi, :, h], o_ref[bi, :, h], TOL_BF16, f"{name} o[{bi},{h}]")
            assert_close(S[bi, h], S_ref[bi, h], TOL_BF16, f"{name} S_T[{bi},{h}]")


def test_full_size_prefill_t4096_all_heads():
    _full_size("prefill_t4096")


@pytest.mark.parametrize("gate_mode", ["full", "kda", "gdn"])
def test_full_size_prefill_t32768_all_heads(gate_mode):
    _full_size("prefill_t32768", gate_mode=gate_mode)


def test_full_size_conv_prefill_b8_all_heads():
    _full_size("conv_prefill_b8_t8192")
