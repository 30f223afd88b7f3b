"""Context-parallel prefill: one sequence split into segments that run at the
same time, joined through the affine map of each segment.

Over a segment of tokens the recurrence maps its entry state affinely to its
exit state: every step S ↦ (I − k eᵀ) Diag(α) S + k zᵀ is affine ("Resumo
Técnico: Gated DeltaNet-2", Metodologia §1), and so is their composition,

    S_out = M · S_in + N,

and the chunked form's only sequential step is this state sweep ("Uma análise
das variantes de atenção linear da família DeltaNet", "Pipeline Triton da
versão por chunks"). M is the segment's final state from S0 = I with v = 0
(no writes), N its final state from S0 = 0. With every segment's (M, N)
known, the entry state of segment g is the composition of the maps of the
segments before it applied to the sequence's S0; each segment then runs once
more from its entry state, giving its outputs and (for the last) S_T.

Two forms:

* :func:`chunk_fwd_context_parallel` -- one segment per rank of a
  ``torch.distributed`` group (NCCL between GPUs): the ranks all-gather their
  (M, N) -- the one exchange step -- and each composes the maps before it.
* :func:`chunk_fwd_segments` -- the same algebra on one GPU, the segments of
  a sequence run as a batch (worth it when the heads alone leave most SMs
  idle, e.g. one or two value heads over a long sequence).

The arithmetic runs in the CUDA library (``gdn2_chunk_fwd`` for the three
passes, ``gdn2_state_affine`` for the composition); this module only
arranges the calls. The algorithm itself, :func:`affine_join`, takes its
forward pass and composition as arguments.
"""

from __future__ import annotations

import torch

from . import gdn2


class CudaBackend:
    """The library's calls on torch CUDA tensors (``kw``: chunk_fwd's gate and
    scale options)."""

    def __init__(self, **kw):
        if kw.get("conv_w") is not None or kw.get("l2norm_qk"):
            raise ValueError("context-parallel prefill takes the recurrence's inputs (no fused conv / L2 norm)")
        self.kw = kw

    def forward(self, q, k, v, alpha, b, w, S0):
        return gdn2.chunk_fwd(q, k, v, alpha, b, w, S0, **self.kw)

    def affine(self, M, N, S):
        return gdn2.state_affine(M, N, S)

    def eye(self, B, H, d, like):
        return torch.eye(d, dtype=torch.float32, device=like.device).expand(B, H, d, d).contiguous()

    def zeros_like(self, x):
        return torch.zeros_like(x)


def segment_maps(backend, q, k, v, alpha, b, w):
    """(M, N) of a segment (per sequence and value head): S_T from S0 = I with
    v = 0, and S_T from S0 = 0."""
    B, H_v, d = v.shape[0], v.shape[2], v.shape[3]
    _, M = backend.forward(q, k, backend.zeros_like(v), alpha, b, w, backend.eye(B, H_v, d, v))
    _, N = backend.forward(q, k, v, alpha, b, w, None)
    return M, N


def affine_join(backend, maps, S0, upto):
    """Entry state of segment ``upto``: the maps of segments 0 .. upto−1
    (a list of (M, N)) applied in order to S0 (None = zeros)."""
    S = S0
    for M, N in maps[:upto]:
        S = backend.affine(M, N, S)
    return S


def chunk_fwd_context_parallel(q, k, v, alpha, b, w, S0=None, *, group=None, backend=None, **kw):
    """This rank's segment of a sequence split across the ranks of ``group``
    (rank r holds tokens [r·L, (r+1)·L) of every sequence, in order of rank;
    the tensors are that segment, [B, L, ...]). ``S0`` is the sequences'
    initial state, the same on every rank (None = zeros). Returns (o, S_T) of
    the segment: its outputs, and its exit state (the sequences' final state
    on the last rank). Collectives: one all-gather of every rank's (M, N)."""
    import torch.distributed as dist
    backend = backend or CudaBackend(**kw)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    M, N = segment_maps(backend, q, k, v, alpha, b, w)
    Ms = [torch.empty_like(M) for _ in range(world)]
    Ns = [torch.empty_like(N) for _ in range(world)]
    dist.all_gather(Ms, M.contiguous(), group=group)
    dist.all_gather(Ns, N.contiguous(), group=group)
    S_in = affine_join(backend, list(zip(Ms, Ns)), S0, rank)
    return backend.forward(q, k, v, alpha, b, w, S_in)


def chunk_fwd_segments(q, k, v, alpha, b, w, S0=None, *, segments, **kw):
    """One sequence (B = 1) of T tokens as ``segments`` equal pieces run as a
    batch on one GPU (T a multiple of ``segments``): the segments' maps in one
    batched pass each, the composition, and a final batched pass from every
    segment's entry state. Same results as gdn2_chunk_fwd up to rounding.
    Returns (o [1,T,H_v,d_v], S_T [1,H_v,d_k,d_v])."""
    backend = CudaBackend(**kw)
    B, T = q.shape[0], q.shape[1]
    if B != 1 or segments < 1 or T % segments:
        raise ValueError("one sequence whose length is a multiple of the segment count")
    L = T // segments

    def seg(x):
        return None if x is None else x.reshape((segments, L) + tuple(x.shape[2:]))

    qs, ks, vs, as_, bs, ws = (seg(x) for x in (q, k, v, alpha, b, w))
    M, N = segment_maps(backend, qs, ks, vs, as_, bs, ws)
    S_in = torch.empty_like(N)
    S = S0
    for g in range(segments):
        # entry state of segment g, then carried across it
        S_in[g:g + 1].copy_(S if S is not None else torch.zeros_like(N[:1]))
        S = backend.affine(M[g:g + 1], N[g:g + 1], S_in[g:g + 1])
    o, S_T = backend.forward(qs, ks, vs, as_, bs, ws, S_in)
    return o.reshape((1, T) + tuple(o.shape[2:])), S_T[segments - 1:]
