"""The allocation-free prefill (gdn2_chunk_fwd_noalloc) against the regular
entry point (gdn2_chunk_fwd with a caller-provided workspace).

gdn2_chunk_fwd_noalloc serves callers that cannot allocate device memory at
call time (plugin hosts and serving runtimes that budget device memory up
front): the library takes the tensor-core kernel's scratch from a fixed array
of its own. This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process, where its first call performs the one-time scratch set-up."""

import ctypes
from dataclasses import replace

import pytest
import torch

from delta_rule_linear_gdn_b200 import gdn2
from delta_rule_linear_gdn_b200.inputs import make_inputs, workload
from tests.gpu_util import TOL_BF16, assert_close, np64

pytestmark = pytest.mark.gpu


def test_noalloc_matches_regular_entry_point_twice():
    w = replace(workload("prefill_t4096"), T=200, H_qk=2, H_v=6, s0="normal")
    inp = make_inputs(w, seed=21, device="cuda")
    args = (inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], inp["S0"])
    o_ref, S_ref = gdn2.chunk_fwd(*args, chunk=64, o_dtype=torch.float32)
    torch.cuda.synchronize()
    for call in range(2):   # two calls in a row share the library's scratch
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        gdn2.chunk_fwd_noalloc(*args, o=o, S_T=S, chunk=64)
        torch.cuda.synchronize()
        assert_close(o, np64(o_ref), TOL_BF16, f"o, call {call}")
        assert_close(S, np64(S_ref), TOL_BF16, f"S_T, call {call}")
        # same kernel, same inputs: the results are in fact identical
        assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


@pytest.mark.parametrize("with_state", [True, False])
def test_noalloc_long_sequence_runs_in_segments(with_state):
    """48 sequence-heads and 19 chunks: more than the fixed array holds at once,
    so the call runs in segments (carrying the state through S_T, or through
    the array itself when S_T is NULL)."""
    w = replace(workload("prefill_t4096"), T=1200, s0="normal")
    inp = make_inputs(w, seed=23, device="cuda")
    args = (inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], inp["S0"])
    o_ref, S_ref = gdn2.chunk_fwd(*args, chunk=64, o_dtype=torch.float32)
    o = torch.full_like(o_ref, float("nan"))
    S = torch.full_like(S_ref, float("nan")) if with_state else None
    gdn2.chunk_fwd_noalloc(*args, o=o, S_T=S, chunk=64)
    torch.cuda.synchronize()
    assert_close(o, np64(o_ref), TOL_BF16, "o")
    if with_state:
        assert_close(S, np64(S_ref), TOL_BF16, "S_T")
        assert torch.equal(S, S_ref)
    assert torch.equal(o, o_ref)


def test_noalloc_rejects_configurations_without_scratch():
    w = replace(workload("prefill_t4096"), T=64, H_qk=1, H_v=1, d=64)
    inp = make_inputs(w, seed=22, device="cuda")
    o = torch.empty((1, 64, 1, 64), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((1, 1, 64, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(gdn2.GDN2Error) as ei:
        gdn2.chunk_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], None,
                               o=o, S_T=S, chunk=64)
    assert ei.value.status == gdn2.ERR_UNSUPPORTED
    p = gdn2.make_params(1, 64, 1, 1, 128, 128, chunk=64)
    fn = gdn2.lib().gdn2_chunk_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(gdn2.Params)] + [ctypes.c_void_p] * 10
    assert fn(None, *[None] * 10) == gdn2.ERR_INVALID_ARG


def test_noalloc_conv_l2norm_segments_carry_conv_history():
    """The fixed array holds 37 chunks of this 12-sequence-head problem, so a
    2-sequence, 3000-token call (47 chunks) with the conv and L2 norm runs in
    two segments; the second segment's first tokens convolve with the last
    inputs of the first. Bit for bit the one-pass call."""
    w = replace(workload("conv_prefill_b8_t8192"), B=2, T=3000, H_qk=2, H_v=6)
    inp = make_inputs(w, seed=29, device="cuda")
    args = (inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], inp["S0"])
    o_ref, S_ref = gdn2.chunk_fwd(*args, chunk=64, o_dtype=torch.float32, conv_w=inp["conv_w"], l2norm_qk=True)
    o = torch.full_like(o_ref, float("nan"))
    S = torch.full_like(S_ref, float("nan"))
    gdn2.chunk_fwd_noalloc(*args, o=o, S_T=S, chunk=64, conv_w=inp["conv_w"], l2norm_qk=True)
    torch.cuda.synchronize()
    assert_close(o, np64(o_ref), TOL_BF16, "o")
    assert_close(S, np64(S_ref), TOL_BF16, "S_T")
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)
