"""The conv history carried between calls (conv_state_in / conv_state_out):
chunked prefill on both paths and decode steps against the float64 oracle
run over the whole token stream, and the written history bit for bit."""

from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_gdn_b200 import gdn2
from delta_rule_linear_gdn_b200.inputs import make_conv_state, make_inputs, workload
from tests.gpu_util import TOL_BF16, TOL_FP32, assert_close, np64, oracle_chunk, to_cuda

pytestmark = pytest.mark.gpu


def small(T, path):
    """(workload, tolerance) of the tensor-core path (bf16, d=128, chunk 64) or
    the fp32 path (d=32, chunk 16), conv + L2 norm in the load, S0 given."""
    if path == "tensor_core":
        w = replace(workload(0), T=T, B=2, H_qk=2, H_v=6, d=128, chunk=64, qkv_dtype="bf16", s0="normal",
                    conv=True)
        return w, TOL_BF16
    w = replace(workload(0), T=T, B=2, H_qk=2, H_v=4, d=32, chunk=16, qkv_dtype="f32", s0="normal", conv=True)
    return w, TOL_FP32


def sl(x, t0, t1):
    return None if x is None else x[:, t0:t1].contiguous()


def prefill(c, t0, t1, S0, h_in, h_out, chunk):
    return gdn2.chunk_fwd(sl(c["q"], t0, t1), sl(c["k"], t0, t1), sl(c["v"], t0, t1), sl(c["alpha"], t0, t1),
                          sl(c["b"], t0, t1), sl(c["w"], t0, t1), S0, chunk=chunk, conv_w=c["conv_w"],
                          l2norm_qk=True, o_dtype=torch.float32, conv_state_in=h_in, conv_state_out=h_out)


def history_after(inp, t0, t1, hist):
    """The oracle's history after tokens [t0, t1), starting from ``hist``."""
    return oracle.conv_state_after(np64(inp["q"][:, t0:t1]), np64(inp["k"][:, t0:t1]), np64(inp["v"][:, t0:t1]),
                                   np64(hist))


def assert_history(got, want, what):
    """The history rows are copies of inputs: equal bit for bit."""
    g = got.detach().cpu().to(torch.float64).numpy()
    assert np.array_equal(g, want), f"{what}: written conv history differs"


@pytest.mark.parametrize("path", ["tensor_core", "fp32"])
@pytest.mark.parametrize("T", [1, 2, 3, 77, 200])
def test_chunk_conv_history_in_and_out(path, T):
    """A prefill that continues after three earlier tokens: the conv of its
    first tokens reads the given history, and the history after its last token
    is written (for T < 3 partly the incoming rows, shifted)."""
    w, tol = small(T, path)
    inp = make_inputs(w, seed=40 + T)
    hist = make_conv_state(w, seed=41 + T)
    c = to_cuda(inp)
    h_in = hist.cuda()
    h_out = torch.full_like(h_in, float("nan"))
    o, S = prefill(c, 0, T, c["S0"], h_in, h_out, w.chunk)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_chunk(inp, l2norm_qk=True, conv_state=hist)
    assert_close(o, o_ref, tol, "o")
    assert_close(S, S_ref, tol, "S_T")
    assert_history(h_out, history_after(inp, 0, T, hist), "conv_state_out")
    torch.testing.assert_close(h_in.cpu(), hist, rtol=0, atol=0)   # the input history is only read


def test_history_without_incoming_and_empty_call():
    """No incoming history means zeros (a sequence's start); a call with no
    tokens passes the incoming history through unchanged."""
    w, tol = small(2, "fp32")
    inp = make_inputs(w, seed=50)
    c = to_cuda(inp)
    h_out = torch.full(gdn2.conv_state_shape(w.B, w.H_qk, w.H_v, w.d, w.d), float("nan"), device="cuda")
    o, S = prefill(c, 0, 2, c["S0"], None, h_out, w.chunk)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_chunk(inp, l2norm_qk=True)
    assert_close(o, o_ref, tol, "o")
    assert_history(h_out, history_after(inp, 0, 2, None), "conv_state_out from zeros")
    assert torch.count_nonzero(h_out[:, 0]) == 0
    h_in = make_conv_state(w, seed=51).cuda()
    h_out2 = torch.full_like(h_in, float("nan"))
    o0, S0 = prefill(c, 0, 0, c["S0"], h_in, h_out2, w.chunk)
    torch.cuda.synchronize()
    assert o0.shape[1] == 0
    torch.testing.assert_close(h_out2, h_in, rtol=0, atol=0)
    torch.testing.assert_close(S0, c["S0"], rtol=0, atol=0)


@pytest.mark.parametrize("path", ["tensor_core", "fp32"])
def test_split_prefill_with_history_equals_whole(path):
    """[0,T) in one call equals [0,t) then [t,T), the second call starting
    from the first one's state and conv history: results within the path's
    tolerance of the oracle and of each other, the final history bit for bit."""
    T, t = 200, 67
    w, tol = small(T, path)
    inp = make_inputs(w, seed=52)
    hist = make_conv_state(w, seed=53)
    c = to_cuda(inp)
    h0 = hist.cuda()
    hw, ha, hb = (torch.full_like(h0, float("nan")) for _ in range(3))
    ow, Sw = prefill(c, 0, T, c["S0"], h0, hw, w.chunk)
    oa, Sa = prefill(c, 0, t, c["S0"], h0, ha, w.chunk)
    ob, Sb = prefill(c, t, T, Sa, ha, hb, w.chunk)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_chunk(inp, l2norm_qk=True, conv_state=hist)
    o_split = torch.cat([oa, ob], 1)
    assert_close(o_split, o_ref, tol, "o split")
    assert_close(Sb, S_ref, tol, "S_T split")
    assert_close(ow, o_ref, tol, "o whole")
    # The two schedules put the chunk boundaries in different places, so on the
    # bf16-operand path each carries its own rounding: they agree to the
    # path's bar, not bit for bit.
    rel = ((o_split - ow).abs().max() / ow.pow(2).mean().sqrt()).item()
    assert rel <= (TOL_BF16 if path == "tensor_core" else 1e-5), rel
    assert_history(ha, history_after(inp, 0, t, hist), "history after [0,t)")
    torch.testing.assert_close(hb, hw, rtol=0, atol=0)


@pytest.mark.parametrize("path", ["tensor_core", "fp32"])
@pytest.mark.parametrize("from_start", [False, True])
def test_decode_steps_with_conv_continue_a_prefill(path, from_start):
    """Prefill T0 tokens, then decode N tokens one step at a time with the conv
    (history ping-ponged between two buffers, L2 norm after the conv): every
    step's output, the final state and the final history agree with the
    oracle over all T0 + N tokens. With ``from_start`` there is no prefill and
    the first step has no incoming history."""
    T0 = 0 if from_start else 37
    N = 12
    w, tol = small(T0 + N, path)
    inp = make_inputs(w, seed=54)
    hist = None if from_start else make_conv_state(w, seed=55)
    c = to_cuda(inp)
    ping = torch.full(gdn2.conv_state_shape(w.B, w.H_qk, w.H_v, w.d, w.d), float("nan"), device="cuda",
                      dtype=c["q"].dtype)
    pong = torch.full_like(ping, float("nan"))
    if from_start:
        S = c["S0"].clone()
        h_in = None
        o_pre = None
    else:
        o_pre, S = prefill(c, 0, T0, c["S0"], hist.cuda(), ping, w.chunk)
        h_in = ping
    outs = []
    for i in range(N):
        t = T0 + i
        h_out = pong if h_in is ping else ping
        outs.append(gdn2.decode_step(c["q"][:, t].contiguous(), c["k"][:, t].contiguous(),
                                     c["v"][:, t].contiguous(), c["alpha"][:, t].contiguous(),
                                     c["b"][:, t].contiguous(), c["w"][:, t].contiguous(), S,
                                     l2norm_qk=True, o_dtype=torch.float32, conv_w=c["conv_w"],
                                     conv_state_in=h_in, conv_state_out=h_out))
        h_in = h_out
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_chunk(inp, l2norm_qk=True, conv_state=hist)
    assert_close(torch.stack(outs, 1), o_ref[:, T0:], tol, "decode o")
    if o_pre is not None:
        assert_close(o_pre, o_ref[:, :T0], tol, "prefill o")
    assert_close(S, S_ref, tol, "S after the decode steps")
    assert_history(h_in, history_after(inp, 0, T0 + N, hist), "history after the decode steps")
