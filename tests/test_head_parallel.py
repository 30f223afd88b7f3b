"""Heads of one layer split across ranks (gloo, world sizes 2 and 4): every
rank runs the float64 oracle on its contiguous block of QK heads and the value
heads that read them; gathered along the head axis, the outputs and final
states equal one oracle run over the whole layer, bit for bit (the same loop
per head), for gates per value head and per QK head."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from delta_rule_linear_gdn_b200.head_parallel import head_shard, take_heads


def _inputs(seed, qk_gates):
    rng = np.random.default_rng(seed)
    B, T, H_qk, H_v, d = 2, 50, 4, 12, 16
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    Hg = H_qk if qk_gates else H_v
    x = dict(q=unit(rng.standard_normal((B, T, H_qk, d))), k=unit(rng.standard_normal((B, T, H_qk, d))),
             v=rng.standard_normal((B, T, H_v, d)), alpha=rng.uniform(0.5, 1.0, (B, T, Hg, d)),
             b=rng.uniform(0, 1, (B, T, Hg, d)), w=rng.uniform(0, 1, (B, T, H_v, d)),
             S0=rng.standard_normal((B, H_v, d, d)) * 0.1)
    return {k_: torch.from_numpy(v_) for k_, v_ in x.items()}, H_qk, H_v


def _run(x, H_v, qk_gates):
    f = lambda t: t.numpy()
    a, b = f(x["alpha"]), f(x["b"])
    if qk_gates:
        a, b = oracle.gates_for_value_heads(a, H_v), oracle.gates_for_value_heads(b, H_v)
    return oracle.gdn2_forward(f(x["q"]), f(x["k"]), f(x["v"]), a, b, f(x["w"]), f(x["S0"]))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, qk_gates, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x, H_qk, H_v = _inputs(11, qk_gates)
    mine = take_heads(x, H_qk, H_v, rank, world, gates_per_qk_head=qk_gates)
    o, S = _run(mine, H_v // world, qk_gates)
    o, S = torch.from_numpy(o), torch.from_numpy(S)
    os_ = [torch.empty_like(o) for _ in range(world)]
    Ss = [torch.empty_like(S) for _ in range(world)]
    dist.all_gather(os_, o)
    dist.all_gather(Ss, S)
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        q.put((torch.cat(os_, dim=2).numpy(), torch.cat(Ss, dim=1).numpy()))


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("qk_gates", [False, True])
def test_head_blocks_gather_into_the_whole_layer(world, qk_gates):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, qk_gates, q)) for r in range(world)]
    for p in procs:
        p.start()
    o, S = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, H_qk, H_v = _inputs(11, qk_gates)
    o_ref, S_ref = _run(x, H_v, qk_gates)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(S, S_ref)


def test_head_shard_rule():
    assert head_shard(16, 48, 0, 8) == (slice(0, 2), slice(0, 6))
    assert head_shard(16, 48, 7, 8) == (slice(14, 16), slice(42, 48))
    # within a block, local value head j reads local QK head j // 3, as the kernels do
    qs, vs = head_shard(16, 48, 3, 8)
    for h in range(vs.start, vs.stop):
        assert h // 3 - qs.start == (h - vs.start) // 3
    with pytest.raises(ValueError):
        head_shard(16, 48, 0, 3)
