"""ctypes binding of libgdn2 (declared in include/gdn2.h).

Argument marshalling only: shapes are read from the tensors, outputs are
allocated with PyTorch (device memory), and every step of the recurrence runs
in the CUDA library. There is no CPU or PyTorch fallback: if the library is
missing or fails to load, every call raises.

Entry points mirror the C ABI:

* :func:`chunk_fwd` -> ``gdn2_chunk_fwd`` (chunked prefill)
* :func:`chunk_fwd_workspace` -> ``gdn2_chunk_fwd_workspace``
* :func:`decode_step` -> ``gdn2_decode_step`` (one recurrent step, state in place)
* :func:`chunk_fwd_noalloc` -> ``gdn2_chunk_fwd_noalloc`` (prefill with the library's
  own fixed scratch, for callers that cannot allocate device memory)
* :func:`chunk_bwd` -> ``gdn2_chunk_bwd`` (gradients of the prefill), with
  :func:`chunk_bwd_workspace` -> ``gdn2_chunk_bwd_workspace``
* :func:`state_affine` -> ``gdn2_state_affine`` (S_out = M S_in + N per head: the
  affine map of a segment, for context-parallel prefill)
* :func:`chunk_fwd_status` -> ``gdn2_chunk_fwd_status`` (device status of the last
  call on a workspace), :func:`chunk_fwd_noalloc_status` -> ``gdn2_chunk_fwd_noalloc_status``
* :func:`debug_set_scan_stall` -> ``gdn2_debug_set_scan_stall`` (failure-path test hook)
* :func:`status_str`, :func:`version`
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn2.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(6)
MAX_SEQS = 384   # GDN2_MAX_SEQS: sequences per packed (cu_seqlens) call
F32, BF16 = 0, 1
GATES = {"full": 0, "kda": 1, "gdn": 2}
PRECISION = {"default": 0, "fp32": 1}

EXPORTS = ("gdn2_status_str", "gdn2_version", "gdn2_chunk_fwd_workspace", "gdn2_chunk_fwd",
           "gdn2_decode_step", "gdn2_chunk_fwd_status", "gdn2_debug_set_scan_stall",
           "gdn2_chunk_fwd_noalloc", "gdn2_chunk_fwd_noalloc_status", "gdn2_chunk_bwd",
           "gdn2_chunk_bwd_workspace", "gdn2_state_affine")


class Params(ctypes.Structure):
    """Mirror of ``gdn2_params``."""
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("H_qk", ctypes.c_int), ("H_v", ctypes.c_int),
        ("d_k", ctypes.c_int), ("d_v", ctypes.c_int), ("chunk", ctypes.c_int),
        ("scale", ctypes.c_float), ("qkv_dtype", ctypes.c_int), ("o_dtype", ctypes.c_int),
        ("gate_mode", ctypes.c_int), ("precision", ctypes.c_int), ("l2norm_qk", ctypes.c_int),
        ("conv_w", ctypes.c_void_p), ("gate_logits", ctypes.c_int),
        ("conv_state_in", ctypes.c_void_p), ("conv_state_out", ctypes.c_void_p),
        ("gate_heads", ctypes.c_int), ("n_seqs", ctypes.c_int), ("cu_seqlens", ctypes.c_void_p),
    ]


class GDN2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)}")


_lib = None


def lib():
    """Load libgdn2.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m delta_rule_linear_gdn_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp = ctypes.c_void_p
        pp = ctypes.POINTER(Params)
        L.gdn2_status_str.argtypes = [ctypes.c_int]
        L.gdn2_status_str.restype = ctypes.c_char_p
        L.gdn2_version.argtypes = []
        L.gdn2_version.restype = ctypes.c_int
        L.gdn2_chunk_fwd_workspace.argtypes = [pp]
        L.gdn2_chunk_fwd_workspace.restype = ctypes.c_size_t
        L.gdn2_chunk_fwd.argtypes = [pp] + [vp] * 10 + [ctypes.c_size_t, vp]
        L.gdn2_chunk_fwd.restype = ctypes.c_int
        L.gdn2_decode_step.argtypes = [pp] + [vp] * 9
        L.gdn2_decode_step.restype = ctypes.c_int
        L.gdn2_chunk_bwd_workspace.argtypes = [pp]
        L.gdn2_chunk_bwd_workspace.restype = ctypes.c_size_t
        L.gdn2_chunk_bwd.argtypes = [pp] + [vp] * 17 + [ctypes.c_size_t, vp]
        L.gdn2_chunk_bwd.restype = ctypes.c_int
        L.gdn2_state_affine.argtypes = [pp] + [vp] * 5
        L.gdn2_state_affine.restype = ctypes.c_int
        L.gdn2_chunk_fwd_status.argtypes = [vp, vp]
        L.gdn2_chunk_fwd_status.restype = ctypes.c_int
        L.gdn2_chunk_fwd_noalloc_status.argtypes = [vp]
        L.gdn2_chunk_fwd_noalloc_status.restype = ctypes.c_int
        L.gdn2_debug_set_scan_stall.argtypes = [ctypes.c_uint]
        L.gdn2_debug_set_scan_stall.restype = None
        _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().gdn2_status_str(int(status)).decode()


def version() -> int:
    return lib().gdn2_version()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype_code(dt) -> int:
    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {dt} (bf16 or fp32)")


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_params(B, T, H_qk, H_v, d_k, d_v, *, chunk=64, scale=1.0, qkv_dtype=BF16, o_dtype=BF16,
                gate_mode="full", precision="default", l2norm_qk=False, conv_w=None, gate_logits=False,
                conv_state_in=None, conv_state_out=None, gates_per_qk_head=False, cu_seqlens=None) -> Params:
    """``cu_seqlens``: None, or a ctypes c_int array of N + 1 token offsets
    (see :func:`cu_seqlens_array`), which must stay alive while the Params are
    used."""
    return Params(int(B), int(T), int(H_qk), int(H_v), int(d_k), int(d_v), int(chunk), float(scale),
                  int(qkv_dtype), int(o_dtype), GATES[gate_mode] if isinstance(gate_mode, str) else int(gate_mode),
                  PRECISION[precision] if isinstance(precision, str) else int(precision),
                  1 if l2norm_qk else 0, _ptr(conv_w), 1 if gate_logits else 0,
                  _ptr(conv_state_in), _ptr(conv_state_out), 1 if gates_per_qk_head else 0,
                  0 if cu_seqlens is None else len(cu_seqlens) - 1,
                  None if cu_seqlens is None else ctypes.cast(cu_seqlens, ctypes.c_void_p).value)


def cu_seqlens_array(cu_seqlens):
    """Host int32 offsets (list, tuple, numpy or CPU tensor) as the ctypes array
    the C call reads."""
    vals = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    return (ctypes.c_int * len(vals))(*vals)


def conv_state_shape(B, H_qk, H_v, d_k, d_v):
    """Shape of a conv history buffer: [B, 3, 2·H_qk·d_k + H_v·d_v] (q | k | v channels)."""
    return (B, 3, 2 * H_qk * d_k + H_v * d_v)


def _check_shapes(lead, H_qk, H_v, d_k, d_v, k, v, alpha, b, w, gate_mode, gates_per_qk_head, states=(),
                  conv_w=None, n_states=None):
    """Shapes of everything the call reads or writes, so that no kernel indexes
    past a tensor: ``lead`` is (B, T) or (B,); ``states`` are
    [n_states (default B),H_v,d_k,d_v]."""
    ns = lead[0] if n_states is None else n_states
    mode = GATES[gate_mode] if isinstance(gate_mode, str) else int(gate_mode)
    Hg = H_qk if gates_per_qk_head else H_v
    want = {"k": lead + (H_qk, d_k), "v": lead + (H_v, d_v)}
    if mode == GATES["full"]:
        want.update(alpha=lead + (Hg, d_k), b=lead + (Hg, d_k), w=lead + (H_v, d_v))
    elif mode == GATES["kda"]:
        want.update(alpha=lead + (Hg, d_k), b=lead + (Hg,))
    else:
        want.update(alpha=lead + (Hg,), b=lead + (Hg,))
    got = {"k": k, "v": v, "alpha": alpha, "b": b, "w": w}
    for name, shape in want.items():
        t = got[name]
        if t is not None and tuple(t.shape) != shape:
            raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
    for name, t in states:
        if t is not None and tuple(t.shape) != (ns, H_v, d_k, d_v):
            raise ValueError(f"{name} must have shape {(ns, H_v, d_k, d_v)}, got {tuple(t.shape)}")
    if conv_w is not None and tuple(conv_w.shape) != (2 * H_qk * d_k + H_v * d_v, 4):
        raise ValueError(f"conv_w must have shape {(2 * H_qk * d_k + H_v * d_v, 4)}, got {tuple(conv_w.shape)}")


def _check_conv_state(t, name, qkv_dtype, shape):
    if t is None:
        return
    _check(t, name, qkv_dtype)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check(t, name, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def chunk_fwd_workspace(params: Params) -> int:
    return int(lib().gdn2_chunk_fwd_workspace(ctypes.byref(params)))


def chunk_fwd(q, k, v, alpha, b, w=None, S0=None, *, chunk=64, scale=1.0, gate_mode="full",
              precision="default", l2norm_qk=False, conv_w=None, o_dtype=None, o=None, S_T=None,
              workspace=None, stream=None, want_state=True, gate_logits=False, conv_state_in=None,
              conv_state_out=None, gates_per_qk_head=False, cu_seqlens=None):
    """Chunked prefill. q,k [B,T,H_qk,d_k]; v [B,T,H_v,d_v]; gates per
    ``gate_mode``: fp32 values, or bf16 logits with ``gate_logits`` (the kernels
    apply the sigmoid); S0 [B,H_v,d_k,d_v] fp32 or None. With ``conv_w``, the
    conv history before token 0 comes from ``conv_state_in`` (None: zeros) and
    the history after the last token is written to ``conv_state_out`` (both
    :func:`conv_state_shape`, q's dtype, distinct buffers). With
    ``gates_per_qk_head`` alpha and b have H_qk heads, shared by the value
    heads of each QK head. With ``cu_seqlens`` (host offsets, N + 1 of them)
    the tensors hold N sequences of different lengths packed along T (B = 1),
    and S0, S_T and the conv histories have N rows. Returns (o, S_T)."""
    B, T, H_qk, d_k = q.shape
    H_v, d_v = v.shape[2], v.shape[3]
    cu = None if cu_seqlens is None else cu_seqlens_array(cu_seqlens)
    NS = B if cu is None else len(cu) - 1    # sequences that own a state
    o_dtype = q.dtype if o_dtype is None else o_dtype
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, q.dtype)
    gdt = torch.bfloat16 if gate_logits else torch.float32
    for name, t in (("alpha", alpha), ("b", b), ("w", w)):
        _check(t, name, gdt)
    for name, t in (("S0", S0), ("conv_w", conv_w)):
        _check(t, name, torch.float32)
    _check_shapes((B, T), H_qk, H_v, d_k, d_v, k, v, alpha, b, w, gate_mode, gates_per_qk_head,
                  states=(("S0", S0), ("S_T", S_T)), conv_w=conv_w, n_states=NS)
    hshape = conv_state_shape(NS, H_qk, H_v, d_k, d_v)
    _check_conv_state(conv_state_in, "conv_state_in", q.dtype, hshape)
    _check_conv_state(conv_state_out, "conv_state_out", q.dtype, hshape)
    p = make_params(B, T, H_qk, H_v, d_k, d_v, chunk=chunk, scale=scale, qkv_dtype=_dtype_code(q.dtype),
                    o_dtype=_dtype_code(o_dtype), gate_mode=gate_mode, precision=precision,
                    l2norm_qk=l2norm_qk, conv_w=conv_w, gate_logits=gate_logits,
                    conv_state_in=conv_state_in, conv_state_out=conv_state_out,
                    gates_per_qk_head=gates_per_qk_head, cu_seqlens=cu)
    if o is None:
        o = torch.empty((B, T, H_v, d_v), dtype=o_dtype, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((NS, H_v, d_k, d_v), dtype=torch.float32, device=q.device)
    _check(o, "o", o_dtype)
    if tuple(o.shape) != (B, T, H_v, d_v):
        raise ValueError(f"o must have shape {(B, T, H_v, d_v)}, got {tuple(o.shape)}")
    _check(S_T, "S_T", torch.float32)
    need = chunk_fwd_workspace(p)   # (reads the offsets too)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().gdn2_chunk_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                              _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace), ws_bytes,
                              _stream_handle(stream))
    if st != OK:
        raise GDN2Error(st, "gdn2_chunk_fwd")
    return o, S_T


def decode_step(q, k, v, alpha, b, w, S, *, scale=1.0, gate_mode="full", l2norm_qk=False, o_dtype=None,
                o=None, stream=None, gate_logits=False, conv_w=None, conv_state_in=None, conv_state_out=None,
                gates_per_qk_head=False):
    """One decode step. q,k [B,H_qk,d_k]; v [B,H_v,d_v]; gates without the T
    axis (fp32 values, or bf16 logits with ``gate_logits``); S [B,H_v,d_k,d_v]
    fp32 updated in place. With ``conv_w`` the step's conv reads
    ``conv_state_in`` (None: zeros) and writes the shifted history to
    ``conv_state_out`` (a second buffer: swap the two between steps). With
    ``gates_per_qk_head`` alpha and b have H_qk heads. Returns o [B,H_v,d_v]."""
    B, H_qk, d_k = q.shape
    H_v, d_v = v.shape[1], v.shape[2]
    o_dtype = q.dtype if o_dtype is None else o_dtype
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, q.dtype)
    gdt = torch.bfloat16 if gate_logits else torch.float32
    for name, t in (("alpha", alpha), ("b", b), ("w", w)):
        _check(t, name, gdt)
    _check(S, "S", torch.float32)
    _check(conv_w, "conv_w", torch.float32)
    _check_shapes((B,), H_qk, H_v, d_k, d_v, k, v, alpha, b, w, gate_mode, gates_per_qk_head,
                  states=(("S", S),), conv_w=conv_w)
    hshape = conv_state_shape(B, H_qk, H_v, d_k, d_v)
    _check_conv_state(conv_state_in, "conv_state_in", q.dtype, hshape)
    _check_conv_state(conv_state_out, "conv_state_out", q.dtype, hshape)
    p = make_params(B, 1, H_qk, H_v, d_k, d_v, scale=scale, qkv_dtype=_dtype_code(q.dtype),
                    o_dtype=_dtype_code(o_dtype), gate_mode=gate_mode, l2norm_qk=l2norm_qk,
                    gate_logits=gate_logits, conv_w=conv_w, conv_state_in=conv_state_in,
                    conv_state_out=conv_state_out, gates_per_qk_head=gates_per_qk_head)
    if o is None:
        o = torch.empty((B, H_v, d_v), dtype=o_dtype, device=q.device)
    _check(o, "o", o_dtype)
    if tuple(o.shape) != (B, H_v, d_v):
        raise ValueError(f"o must have shape {(B, H_v, d_v)}, got {tuple(o.shape)}")
    st = lib().gdn2_decode_step(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                                _ptr(S), _ptr(o), _stream_handle(stream))
    if st != OK:
        raise GDN2Error(st, "gdn2_decode_step")
    return o


def chunk_fwd_noalloc(q, k, v, alpha, b, w=None, S0=None, *, o, S_T=None, chunk=64, scale=1.0,
                      gate_mode="full", l2norm_qk=False, conv_w=None, stream=None, gate_logits=False,
                      gates_per_qk_head=False):
    """Chunked prefill through ``gdn2_chunk_fwd_noalloc``: the library takes the
    kernel's scratch from its own fixed device array, so nothing is allocated
    for the call. ``o`` and ``S_T`` (or None) are caller-provided outputs (the
    caller owns all device memory). Returns (o, S_T)."""
    L = lib()
    fn = L.gdn2_chunk_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(Params)] + [ctypes.c_void_p] * 10
    fn.restype = ctypes.c_int
    B, T, H_qk, d_k = q.shape
    H_v, d_v = v.shape[2], v.shape[3]
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, q.dtype)
    gdt = torch.bfloat16 if gate_logits else torch.float32
    for name, t in (("alpha", alpha), ("b", b), ("w", w)):
        _check(t, name, gdt)
    for name, t in (("S0", S0), ("S_T", S_T), ("conv_w", conv_w)):
        _check(t, name, torch.float32)
    _check(o, "o")
    _check_shapes((B, T), H_qk, H_v, d_k, d_v, k, v, alpha, b, w, gate_mode, gates_per_qk_head,
                  states=(("S0", S0), ("S_T", S_T)), conv_w=conv_w)
    if tuple(o.shape) != (B, T, H_v, d_v):
        raise ValueError(f"o must have shape {(B, T, H_v, d_v)}, got {tuple(o.shape)}")
    p = make_params(B, T, H_qk, H_v, d_k, d_v, chunk=chunk, scale=scale, qkv_dtype=_dtype_code(q.dtype),
                    o_dtype=_dtype_code(o.dtype), gate_mode=gate_mode, l2norm_qk=l2norm_qk, conv_w=conv_w,
                    gate_logits=gate_logits, gates_per_qk_head=gates_per_qk_head)
    st = fn(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
            _ptr(S_T), _stream_handle(stream))
    if st != OK:
        raise GDN2Error(st, "gdn2_chunk_fwd_noalloc")
    return o, S_T


def chunk_fwd_status(workspace, stream=None) -> int:
    """Status code of the device-side waits of the last :func:`chunk_fwd` that
    ran with ``workspace`` (OK or ERR_TIMEOUT); synchronises the stream first."""
    return int(lib().gdn2_chunk_fwd_status(_ptr(workspace), _stream_handle(stream)))


def chunk_fwd_noalloc_status(stream=None) -> int:
    """Status code of the last :func:`chunk_fwd_noalloc` on the current device."""
    return int(lib().gdn2_chunk_fwd_noalloc_status(_stream_handle(stream)))


def debug_set_scan_stall(polls: int) -> None:
    """Failure-path test hook: polls > 0 makes every later tensor-core prefill's
    scan give up on a wait before it issues any product; 0 turns it off."""
    lib().gdn2_debug_set_scan_stall(int(polls))


def chunk_bwd_workspace(params: Params) -> int:
    return int(lib().gdn2_chunk_bwd_workspace(ctypes.byref(params)))


def chunk_bwd(q, k, v, alpha, b, w, S0, dO, dS_T=None, *, scale=1.0, gate_mode="full", gate_logits=False,
              gates_per_qk_head=False, precision="default", workspace=None, stream=None, want_dS0=True):
    """Gradients of <dO, o> + <dS_T, S_T> for :func:`chunk_fwd`'s inputs (same
    argument forms; dO in o's dtype, dS_T fp32 or None). Returns a dict of fp32
    tensors q, k, v, alpha, b, w (None in the tied modes, where b holds dβ), S0
    (None without ``want_dS0``)."""
    B, T, H_qk, d_k = q.shape
    H_v, d_v = v.shape[2], v.shape[3]
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, q.dtype)
    gdt = torch.bfloat16 if gate_logits else torch.float32
    for name, t in (("alpha", alpha), ("b", b), ("w", w)):
        _check(t, name, gdt)
    _check(dO, "dO")
    for name, t in (("S0", S0), ("dS_T", dS_T)):
        _check(t, name, torch.float32)
    _check_shapes((B, T), H_qk, H_v, d_k, d_v, k, v, alpha, b, w, gate_mode, gates_per_qk_head,
                  states=(("S0", S0), ("dS_T", dS_T)))
    if tuple(dO.shape) != (B, T, H_v, d_v):
        raise ValueError(f"dO must have shape {(B, T, H_v, d_v)}, got {tuple(dO.shape)}")
    p = make_params(B, T, H_qk, H_v, d_k, d_v, scale=scale, qkv_dtype=_dtype_code(q.dtype),
                    o_dtype=_dtype_code(dO.dtype), gate_mode=gate_mode, precision=precision,
                    gate_logits=gate_logits, gates_per_qk_head=gates_per_qk_head)
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"q": torch.empty(q.shape, **f32), "k": torch.empty(k.shape, **f32), "v": torch.empty(v.shape, **f32),
         "alpha": torch.empty(alpha.shape, **f32), "b": torch.empty(b.shape, **f32),
         "w": None if w is None else torch.empty(w.shape, **f32),
         "S0": torch.empty((B, H_v, d_k, d_v), **f32) if want_dS0 else None}
    need = chunk_bwd_workspace(p)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().gdn2_chunk_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                              _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]),
                              _ptr(g["alpha"]), _ptr(g["b"]), _ptr(g["w"]), _ptr(g["S0"]), _ptr(workspace),
                              ws_bytes, _stream_handle(stream))
    if st != OK:
        raise GDN2Error(st, "gdn2_chunk_bwd")
    return g


def state_affine(M, N, S_in, S_out=None, stream=None):
    """S_out = M · S_in + N per (sequence, value head): M [B,H_v,d_k,d_k]; N,
    S_in [B,H_v,d_k,d_v] (either may be None = zeros). S_out may be S_in (in
    place); a new tensor when None. Returns S_out."""
    B, H_v, d_k, _ = M.shape
    ref = N if N is not None else S_in
    d_v = ref.shape[-1] if ref is not None else d_k
    for name, t in (("M", M), ("N", N), ("S_in", S_in)):
        _check(t, name, torch.float32)
    if S_out is None:
        S_out = torch.empty((B, H_v, d_k, d_v), dtype=torch.float32, device=M.device)
    _check(S_out, "S_out", torch.float32)
    for name, t in (("N", N), ("S_in", S_in), ("S_out", S_out)):
        if t is not None and tuple(t.shape) != (B, H_v, d_k, d_v):
            raise ValueError(f"{name} must have shape {(B, H_v, d_k, d_v)}, got {tuple(t.shape)}")
    p = make_params(B, 0, 1, H_v, d_k, d_v)
    st = lib().gdn2_state_affine(ctypes.byref(p), _ptr(M), _ptr(N), _ptr(S_in), _ptr(S_out), _stream_handle(stream))
    if st != OK:
        raise GDN2Error(st, "gdn2_state_affine")
    return S_out
