"""Heads of one layer split across ranks.

Value head h reads query/key head h // (H_v / H_qk) ("Gated DeltaNet: o mixer
em 48 das 64 camadas", Conceito: each QK head serves a contiguous group of
value heads), so a contiguous block of H_qk / N query/key heads and the
H_v / N value heads that read them form a self-contained problem: within the
block, local value head j reads local QK head j // (H_v / H_qk), the same rule
the kernels apply. Every (sequence, value head) recurrence is independent, so
the ranks exchange nothing; in a tensor-parallel model each rank's
projections produce its block's q, k, v and gates directly (contiguous
[B, T, H_local, d] tensors, what the C calls take).
"""

from __future__ import annotations


def head_shard(H_qk: int, H_v: int, rank: int, world: int):
    """(qk_heads, v_heads): the slices of query/key heads and value heads that
    rank ``rank`` of ``world`` runs. H_qk must be a multiple of ``world``."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    if H_qk % world or H_v % H_qk:
        raise ValueError("H_qk must be a multiple of the rank count and H_v of H_qk")
    nq = H_qk // world
    g = H_v // H_qk
    return slice(rank * nq, (rank + 1) * nq), slice(rank * nq * g, (rank + 1) * nq * g)


def take_heads(inp: dict, H_qk: int, H_v: int, rank: int, world: int, gates_per_qk_head: bool = False,
               head_axis: int = 2):
    """The rank's block of an input dict of a layer (q, k [.., H_qk, d]; v,
    w [.., H_v, d]; alpha, b per value head or, with ``gates_per_qk_head``,
    per QK head; S0 [B, H_v, d, d]), as contiguous tensors. (A model computes
    these blocks directly; this stands in for that.)"""
    qs, vs = head_shard(H_qk, H_v, rank, world)
    gs = qs if gates_per_qk_head else vs

    def cut(t, s, axis):
        if t is None:
            return None
        idx = [slice(None)] * t.ndim
        idx[axis] = s
        return t[tuple(idx)].contiguous()

    out = dict(inp)
    out["q"], out["k"] = cut(inp["q"], qs, head_axis), cut(inp["k"], qs, head_axis)
    out["v"] = cut(inp["v"], vs, head_axis)
    out["w"] = cut(inp.get("w"), vs, head_axis)
    out["alpha"], out["b"] = cut(inp["alpha"], gs, head_axis), cut(inp["b"], gs, head_axis)
    if inp.get("S0") is not None:
        out["S0"] = cut(inp["S0"], vs, 1)
    return out
