"""Context-parallel prefill through the affine map of each segment.

CPU (gloo, world sizes 2 and 4): every rank runs the orchestration of
delta_rule_linear_gdn_b200.context_parallel on its own segment of one
sequence, with the float64 oracle as the forward pass and a plain matrix
product as the composition; the all-gather is real. The joined outputs and the
last rank's final state equal the oracle run over the whole sequence.

GPU: the single-GPU form (segments as a batch) against the oracle at the
bf16-path bar, and gdn2_state_affine against a float64 matrix product."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from delta_rule_linear_gdn_b200 import context_parallel as cp


class OracleBackend:
    """The orchestration's forward pass and composition on CPU tensors: the
    float64 oracle and numpy's matrix product (test infrastructure)."""

    def forward(self, q, k, v, alpha, b, w, S0):
        f = lambda t: None if t is None else t.double().numpy()
        o, S = oracle.gdn2_forward(f(q), f(k), f(v), f(alpha), f(b), f(w), f(S0))
        return torch.from_numpy(o), torch.from_numpy(S)

    def affine(self, M, N, S):
        if S is None:
            return N.double().clone()
        out = M.double().numpy() @ S.double().numpy() + N.double().numpy()
        return torch.from_numpy(np.ascontiguousarray(out))

    def eye(self, B, H, d, like):
        return torch.eye(d, dtype=torch.float64).expand(B, H, d, d).contiguous()

    def zeros_like(self, x):
        return torch.zeros_like(x)


def _inputs(seed, B=2, T=96, H_qk=1, H_v=2, d=16):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    x = dict(q=unit(rng.standard_normal((B, T, H_qk, d))), k=unit(rng.standard_normal((B, T, H_qk, d))),
             v=rng.standard_normal((B, T, H_v, d)), alpha=1 / (1 + np.exp(-rng.normal(3, 1, (B, T, H_v, d)))),
             b=rng.uniform(0, 1, (B, T, H_v, d)), w=rng.uniform(0, 1, (B, T, H_v, d)),
             S0=rng.standard_normal((B, H_v, d, d)) * 0.1)
    return {k_: torch.from_numpy(v_) for k_, v_ in x.items()}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x = _inputs(seed=5)
    T = x["q"].shape[1]
    L = T // world
    seg = {k_: (t[:, rank * L:(rank + 1) * L].contiguous() if k_ != "S0" else t) for k_, t in x.items()}
    o, S = cp.chunk_fwd_context_parallel(seg["q"], seg["k"], seg["v"], seg["alpha"], seg["b"], seg["w"],
                                         seg["S0"], backend=OracleBackend())
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, o.numpy(), S.numpy()))


@pytest.mark.parametrize("world", [2, 4])
def test_ranks_join_segments_into_the_whole_sequence(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = _inputs(seed=5)
    f = lambda t: t.numpy()
    o_ref, S_ref = oracle.gdn2_forward(f(x["q"]), f(x["k"]), f(x["v"]), f(x["alpha"]), f(x["b"]), f(x["w"]), f(x["S0"]))
    o = np.concatenate([o_ for _, o_, _ in out], axis=1)
    assert oracle.rel_err(o, o_ref) < 1e-10
    assert oracle.rel_err(out[-1][2], S_ref) < 1e-10


def test_segment_map_is_the_product_of_the_token_transitions():
    """M of a short segment (S0 = I, v = 0) against the explicit product of
    the d_k × d_k transitions A_t = (I − k_t e_tᵀ) Diag(α_t), and N against the
    state from S0 = 0 (the oracle's own run)."""
    x = _inputs(seed=7, B=1, T=6, d=8)
    M, N = cp.segment_maps(OracleBackend(), x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"])
    k, a, b = x["k"].numpy(), x["alpha"].numpy(), x["b"].numpy()
    for h in range(2):
        P = np.eye(8)
        for t in range(6):
            kt = k[0, t, 0]
            A = (np.eye(8) - np.outer(kt, b[0, t, h] * kt)) @ np.diag(a[0, t, h])
            P = A @ P
        np.testing.assert_allclose(M[0, h].numpy(), P, atol=1e-12)
    _, S = OracleBackend().forward(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], None)
    np.testing.assert_allclose(N.numpy(), S.numpy(), atol=1e-12)


# ------------------------------------------------------------------ GPU

@pytest.mark.gpu
@pytest.mark.parametrize("segments", [2, 4, 8])
def test_segments_on_one_gpu_match_the_oracle(segments):
    from dataclasses import replace
    from delta_rule_linear_gdn_b200 import gdn2
    from delta_rule_linear_gdn_b200.inputs import make_inputs, workload
    from tests.gpu_util import TOL_BF16, assert_close, oracle_chunk
    w = replace(workload("prefill_t4096"), T=64 * 24, H_qk=2, H_v=6, s0="normal")
    inp = make_inputs(w, seed=91, device="cuda")
    args = (inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], inp["S0"])
    o, S = cp.chunk_fwd_segments(*args, segments=segments, o_dtype=torch.float32)
    o1, S1 = gdn2.chunk_fwd(*args, o_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_chunk(inp)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(S, S_ref, TOL_BF16, "S_T")
    # and close to the one-pass call (the same arithmetic, in another order)
    assert (o - o1).abs().max() / o1.pow(2).mean().sqrt() < 2e-2


@pytest.mark.gpu
def test_state_affine_kernel():
    from delta_rule_linear_gdn_b200 import gdn2
    g = torch.Generator(device="cpu").manual_seed(3)
    for d in (32, 64, 128):
        M = torch.randn((2, 3, d, d), generator=g) / d ** 0.5
        N = torch.randn((2, 3, d, d), generator=g)
        S = torch.randn((2, 3, d, d), generator=g)
        ref = M.double() @ S.double() + N.double()
        Mc, Nc, Sc = M.cuda(), N.cuda(), S.cuda()
        out = gdn2.state_affine(Mc, Nc, Sc)
        torch.cuda.synchronize()
        assert (out.cpu().double() - ref).abs().max() / ref.pow(2).mean().sqrt() < 1e-5
        # in place, and with S_in / N omitted
        gdn2.state_affine(Mc, Nc, Sc, S_out=Sc)
        torch.cuda.synchronize()
        torch.testing.assert_close(Sc, out, rtol=0, atol=0)
        z = gdn2.state_affine(Mc, Nc, None)
        torch.cuda.synchronize()
        torch.testing.assert_close(z, Nc, rtol=0, atol=0)
