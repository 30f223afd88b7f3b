"""Seeded synthetic inputs for the GDN-2 recurrence.

This module only draws random numbers with the value distributions of the
workloads; it holds none of the recurrence's arithmetic. It is the single
module shared by the CUDA path's tests/bench and the oracle's tests: both sides
receive the same tensors (the oracle a float64 copy of them).

Workloads (layer shape of "Gated DeltaNet: o mixer em 48 das 64 camadas",
Conceito: 16 QK heads serving 48 V heads, head dimension 128):

  index name                         shape
  0     oracle_d16_t64               B=1,T=64, 1 QK / 1 V head, d=16, chunk 16, fp32
  1     prefill_t4096                B=1,T=4096, 16/48 heads, d=128, chunk 64, bf16 q,k,v
  2     prefill_t32768               B=1,T=32768, 16/48, d=128, chunk 64, bf16, alpha mean 4
  3     decode_b256                  B=256 sequences, one token per step, 16/48, d=128
  4     conv_prefill_b8_t8192        B=8,T=8192, 16/48, d=128, conv k=4 + L2 fused, S0 != 0
  5     decode_b64                   B=64 sequences (profiler-sized decode), 16/48, d=128

Value distributions: q,k ~ N(0,1) rows scaled to unit length (raw N(0,1) when
the conv + L2 norm is fused into the kernel); v ~ N(0,1); alpha = sigmoid(N(mu,1))
per key channel (mu 3, or 4 for the T=32768 workload); b, w = sigmoid(N(0,1))
per channel; tied runs draw beta = sigmoid(N(0,1)) and a scalar alpha =
sigmoid(N(4,1)) per (sequence, token, V head); S0 = 0 or N(0, 0.02²) entries;
conv weights N(0, 0.5²). N(mu, s) names mean and standard deviation.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H_qk: int
    H_v: int
    d: int
    chunk: int
    qkv_dtype: str          # "f32" or "bf16"
    alpha_mu: float
    s0: str                 # "zeros" or "normal"
    conv: bool = False      # depthwise causal conv (k=4) + L2 norm fused into the kernel
    decode_steps: int = 0   # >0: a decode workload of that many consecutive steps


WORKLOADS = [
    Workload("oracle_d16_t64", 1, 64, 1, 1, 16, 16, "f32", 3.0, "zeros"),
    Workload("prefill_t4096", 1, 4096, 16, 48, 128, 64, "bf16", 3.0, "zeros"),
    Workload("prefill_t32768", 1, 32768, 16, 48, 128, 64, "bf16", 4.0, "zeros"),
    Workload("decode_b256", 256, 1, 16, 48, 128, 64, "bf16", 3.0, "normal", decode_steps=1000),
    Workload("conv_prefill_b8_t8192", 8, 8192, 16, 48, 128, 64, "bf16", 3.0, "normal", conv=True),
    # a quarter of the decode batch: the case profiler captures run on
    Workload("decode_b64", 64, 1, 16, 48, 128, 64, "bf16", 3.0, "normal", decode_steps=1000),
]

BY_NAME = {w.name: w for w in WORKLOADS}

S0_STD = 0.02
CONV_STD = 0.5
TIED_ALPHA_MU = 4.0


def workload(name_or_index, **overrides) -> Workload:
    w = WORKLOADS[name_or_index] if isinstance(name_or_index, int) else BY_NAME[name_or_index]
    return replace(w, **overrides) if overrides else w


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    return g


def _normal(shape, g, device, mean=0.0, std=1.0):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x


def _unit_rows(shape, g, device):
    # Uniform direction on the sphere: a Gaussian vector divided by its length.
    x = _normal(shape, g, device)
    x.div_(torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-30))
    return x


def _qkv_dtype(w: Workload):
    return torch.bfloat16 if w.qkv_dtype == "bf16" else torch.float32


def make_inputs(w: Workload, seed: int | None = None, device="cpu", gate_mode: str = "full",
                gate_logits: bool = False, gates_per_qk_head: bool = False):
    """Draw one batch of inputs for workload ``w``.

    gate_mode "full": alpha, b [B,T,Hv,dk], w [B,T,Hv,dv].
    gate_mode "kda":  alpha [B,T,Hv,dk] (mean alpha_mu), b = beta [B,T,Hv], w = None.
    gate_mode "gdn":  alpha [B,T,Hv] (mean 4), b = beta [B,T,Hv], w = None.
    Returns a dict of tensors on ``device`` (q,k,v in the workload's dtype;
    gates float32 sigmoids of normal draws, or with ``gate_logits`` those
    draws themselves rounded to bf16; S0 and conv weights float32). With
    ``gates_per_qk_head`` alpha and b (beta) have H_qk heads instead of H_v.
    """
    if seed is None:
        seed = WORKLOADS.index(BY_NAME[w.name]) if w.name in BY_NAME else 0
    dev = torch.device(device)
    B, T, Hqk, Hv, d = w.B, w.T, w.H_qk, w.H_v, w.d
    out = {}
    if w.conv:
        q = _normal((B, T, Hqk, d), _gen(seed, 1, dev), dev)
        k = _normal((B, T, Hqk, d), _gen(seed, 2, dev), dev)
    else:
        q = _unit_rows((B, T, Hqk, d), _gen(seed, 1, dev), dev)
        k = _unit_rows((B, T, Hqk, d), _gen(seed, 2, dev), dev)
    v = _normal((B, T, Hv, d), _gen(seed, 3, dev), dev)
    dt = _qkv_dtype(w)
    out["q"], out["k"], out["v"] = q.to(dt), k.to(dt), v.to(dt)
    gate = (lambda x: x.to(torch.bfloat16)) if gate_logits else torch.sigmoid
    Hg = Hqk if gates_per_qk_head else Hv     # heads of alpha and b
    if gate_mode == "full":
        out["alpha"] = gate(_normal((B, T, Hg, d), _gen(seed, 4, dev), dev, mean=w.alpha_mu))
        out["b"] = gate(_normal((B, T, Hg, d), _gen(seed, 5, dev), dev))
        out["w"] = gate(_normal((B, T, Hv, d), _gen(seed, 6, dev), dev))
    elif gate_mode == "kda":
        out["alpha"] = gate(_normal((B, T, Hg, d), _gen(seed, 4, dev), dev, mean=TIED_ALPHA_MU))
        out["b"] = gate(_normal((B, T, Hg), _gen(seed, 5, dev), dev))
        out["w"] = None
    elif gate_mode == "gdn":
        out["alpha"] = gate(_normal((B, T, Hg), _gen(seed, 4, dev), dev, mean=TIED_ALPHA_MU))
        out["b"] = gate(_normal((B, T, Hg), _gen(seed, 5, dev), dev))
        out["w"] = None
    else:
        raise ValueError(gate_mode)
    if w.s0 == "normal":
        out["S0"] = _normal((B, Hv, d, d), _gen(seed, 7, dev), dev, std=S0_STD)
    else:
        out["S0"] = None
    if w.conv:
        out["conv_w"] = _normal((2 * Hqk * d + Hv * d, 4), _gen(seed, 8, dev), dev, std=CONV_STD)
    else:
        out["conv_w"] = None
    return out


def make_conv_state(w: Workload, seed: int, device="cpu"):
    """A conv history [B, 3, 2·Hqk·d + Hv·d] in the workload's q,k,v dtype: the
    pre-conv inputs of three earlier tokens (standard normal draws, the
    distribution of the conv workload's q, k, v), channels q | k | v."""
    dev = torch.device(device)
    x = _normal((w.B, 3, (2 * w.H_qk + w.H_v) * w.d), _gen(seed, 9, dev), dev)
    return x.to(_qkv_dtype(w))


def make_decode_pool(w: Workload, pool: int = 16, seed: int | None = None, device="cpu",
                     gate_mode: str = "full", gate_logits: bool = False, gates_per_qk_head: bool = False):
    """Per-step decode inputs: ``pool`` independent one-token step sets, cycled by
    the caller, plus the initial state. Tensors carry a leading pool axis."""
    if seed is None:
        seed = 3
    steps = make_inputs(replace(w, T=pool, s0="zeros"), seed=seed, device=device, gate_mode=gate_mode,
                        gate_logits=gate_logits, gates_per_qk_head=gates_per_qk_head)
    # [B, pool, ...] -> [pool, B, ...]
    for key in ("q", "k", "v", "alpha", "b", "w"):
        if steps[key] is not None:
            steps[key] = steps[key].transpose(0, 1).contiguous()
    dev = torch.device(device)
    steps["S0"] = _normal((w.B, w.H_v, w.d, w.d), _gen(seed, 7, dev), dev, std=S0_STD)
    return steps
