"""The C ABI library loads and exports every symbol include/gdn2.h declares, and
host-side validation rejects bad arguments before any CUDA call (so these run
without a GPU)."""

import ctypes
import os
import re

import pytest

from delta_rule_linear_gdn_b200 import gdn2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn2.h")


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(gdn2.LIB_PATH):
        from delta_rule_linear_gdn_b200 import build
        build.build()
    return gdn2.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN2_API\s+[\w\s\*]+?\b(gdn2_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    assert set(gdn2.EXPORTS) <= set(syms), syms
    assert "gdn2_chunk_fwd" in syms and "gdn2_decode_step" in syms


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    for s in range(6):
        assert gdn2.status_str(s).startswith("GDN2_")
    assert "unknown" in gdn2.status_str(99)
    assert gdn2.version() == 200


def _params(**kw):
    base = dict(B=1, T=64, H_qk=1, H_v=1, d_k=16, d_v=16, chunk=16, qkv_dtype=gdn2.F32, o_dtype=gdn2.F32)
    raw = {f: kw.pop(f) for f in ("gate_logits", "gate_heads") if f in kw}
    base.update(kw)
    p = gdn2.make_params(**base)
    for f, val in raw.items():
        setattr(p, f, int(val))           # raw field value, including invalid ones
    return p


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def _call_chunk(L, p, **ptrs):
    names = ["q", "k", "v", "alpha", "b", "w", "S0", "o", "S_T", "ws"]
    vals = {n: FAKE * (i + 1) for i, n in enumerate(names)}
    vals["ws"] = None
    vals.update(ptrs)
    return L.gdn2_chunk_fwd(ctypes.byref(p), *[vals[n] for n in names], 0, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(B=-1), gdn2.ERR_INVALID_ARG),
    (dict(T=-5), gdn2.ERR_INVALID_ARG),
    (dict(H_qk=2, H_v=3), gdn2.ERR_INVALID_ARG),
    (dict(H_qk=0), gdn2.ERR_INVALID_ARG),
    (dict(d_k=24, d_v=24), gdn2.ERR_UNSUPPORTED),
    (dict(d_k=16, d_v=32), gdn2.ERR_UNSUPPORTED),
    (dict(chunk=48), gdn2.ERR_UNSUPPORTED),
    (dict(qkv_dtype=7), gdn2.ERR_INVALID_ARG),
    (dict(gate_mode=5), gdn2.ERR_INVALID_ARG),
    (dict(precision=3), gdn2.ERR_INVALID_ARG),
    (dict(scale=float("nan")), gdn2.ERR_INVALID_ARG),
    (dict(gate_logits=2), gdn2.ERR_INVALID_ARG),
    (dict(gate_heads=2), gdn2.ERR_INVALID_ARG),
])
def test_chunk_rejects_bad_params(L, kw, expect):
    assert _call_chunk(L, _params(**kw)) == expect


def test_chunk_rejects_null_and_misaligned_pointers(L):
    p = _params()
    assert _call_chunk(L, p, q=None) == gdn2.ERR_INVALID_ARG
    assert _call_chunk(L, p, o=None) == gdn2.ERR_INVALID_ARG
    assert _call_chunk(L, p, alpha=None) == gdn2.ERR_INVALID_ARG
    assert _call_chunk(L, p, k=FAKE * 2 + 4) == gdn2.ERR_INVALID_ARG
    # full gates need w; tied gates forbid it
    assert _call_chunk(L, p, w=None) == gdn2.ERR_INVALID_ARG
    assert _call_chunk(L, _params(gate_mode=1)) == gdn2.ERR_INVALID_ARG


def test_chunk_rejects_aliased_output(L):
    p = _params()
    # o on top of q
    assert _call_chunk(L, p, o=FAKE) == gdn2.ERR_INVALID_ARG
    # S_T overlapping o
    assert _call_chunk(L, p, S_T=FAKE * 8 + 64) == gdn2.ERR_INVALID_ARG


def test_decode_rejects_bad_args(L):
    p = _params()
    args = [FAKE * (i + 1) for i in range(8)]
    args[6] = None  # S
    assert L.gdn2_decode_step(ctypes.byref(p), *args, None) == gdn2.ERR_INVALID_ARG
    assert L.gdn2_decode_step(None, *[FAKE] * 8, None) == gdn2.ERR_INVALID_ARG


def _call_decode(L, p, **ptrs):
    names = ["q", "k", "v", "alpha", "b", "w", "S", "o"]
    vals = {n: FAKE * (i + 1) for i, n in enumerate(names)}
    vals.update(ptrs)
    return L.gdn2_decode_step(ctypes.byref(p), *[vals[n] for n in names], None)


def test_conv_state_validation(L):
    # history buffers at 64 KiB multiples past the other arguments (576 bytes each here)
    hin, hout, conv_w = FAKE * 30, FAKE * 31, FAKE * 20
    for call in (_call_chunk, _call_decode):
        # history without a conv
        assert call(L, _params(conv_state_in=hin)) == gdn2.ERR_INVALID_ARG
        assert call(L, _params(conv_state_out=hout)) == gdn2.ERR_INVALID_ARG
        # misaligned
        assert call(L, _params(conv_w=conv_w, conv_state_out=hout + 8)) == gdn2.ERR_INVALID_ARG
        # outgoing history on the incoming one (also in place), or on an input
        assert call(L, _params(conv_w=conv_w, conv_state_in=hin, conv_state_out=hin)) == gdn2.ERR_INVALID_ARG
        assert call(L, _params(conv_w=conv_w, conv_state_in=hin, conv_state_out=hin + 512)) == gdn2.ERR_INVALID_ARG
        assert call(L, _params(conv_w=conv_w, conv_state_out=FAKE * 2)) == gdn2.ERR_INVALID_ARG
        assert call(L, _params(conv_w=conv_w, conv_state_out=conv_w)) == gdn2.ERR_INVALID_ARG
    # the output o written over the incoming history
    assert _call_chunk(L, _params(conv_w=conv_w, conv_state_in=hin), o=hin) == gdn2.ERR_INVALID_ARG
    assert _call_decode(L, _params(conv_w=conv_w, conv_state_in=hin), o=hin) == gdn2.ERR_INVALID_ARG
    assert _call_decode(L, _params(conv_w=conv_w, conv_state_in=hin), S=hin - 256) == gdn2.ERR_INVALID_ARG


def test_varlen_validation_and_workspace(L):
    """Packed sequences (cu_seqlens, host offsets): every malformed table is
    refused before any launch; the workspace of the tensor-core path holds a
    slot per chunk of every sequence."""
    def vp(cu, **kw):
        arr = gdn2.cu_seqlens_array(cu)
        base = dict(B=1, T=int(cu[-1]), H_qk=1, H_v=2, d_k=16, d_v=16, chunk=16, qkv_dtype=gdn2.F32,
                    o_dtype=gdn2.F32, cu_seqlens=arr)
        base.update(kw)
        return gdn2.make_params(**base), arr
    for cu, kw in (([1, 5], {}), ([0, 5, 3, 9], {}), ([0, 4, 9], dict(T=10)), ([0, 4, 9], dict(B=2))):
        p, keep = vp(cu, **kw)
        assert _call_chunk(L, p) == gdn2.ERR_INVALID_ARG, (cu, kw)
    p, keep = vp(list(range(gdn2.MAX_SEQS + 2)))            # one sequence too many
    assert _call_chunk(L, p) == gdn2.ERR_INVALID_ARG
    p = _params()
    p.n_seqs = 2                                            # a count without offsets
    assert _call_chunk(L, p) == gdn2.ERR_INVALID_ARG
    p, keep = vp([0, 3, 7])
    assert _call_decode(L, p) == gdn2.ERR_INVALID_ARG       # decode has no packed form
    fn = L.gdn2_chunk_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(gdn2.Params)] + [ctypes.c_void_p] * 10
    fn.restype = ctypes.c_int
    assert fn(ctypes.byref(p), *[FAKE * (i + 1) for i in range(9)], None) == gdn2.ERR_UNSUPPORTED
    # S0 sized for B = 1 rather than for the 3 sequences overlaps o placed right after it
    p, keep = vp([0, 3, 7, 7], H_v=1)
    s0_one = 16 * 16 * 4
    assert _call_chunk(L, p, S0=FAKE * 7, o=FAKE * 7 + s0_one) == gdn2.ERR_INVALID_ARG
    # tensor-core workspace: 256-byte header + one 74,752-byte slot per (chunk, value head)
    cu = [0, 130, 130, 131, 331]                            # chunks of 64: 3, 0, 1, 4
    arr = gdn2.cu_seqlens_array(cu)
    p = gdn2.make_params(1, 331, 2, 6, 128, 128, chunk=64, cu_seqlens=arr)
    assert gdn2.chunk_fwd_workspace(p) == 256 + 8 * 6 * 74752
    # the conv / L2 norm run in the prep's own load: no extra workspace
    p = gdn2.make_params(1, 331, 2, 6, 128, 128, chunk=64, cu_seqlens=arr, l2norm_qk=True)
    assert gdn2.chunk_fwd_workspace(p) == 256 + 8 * 6 * 74752


def _header_param_fields():
    text = open(HEADER).read()
    body = text[text.index("typedef struct {"):text.index("} gdn2_params;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    return re.findall(r"(\w+)\s*;", body)


def test_params_mirror_matches_header_field_order():
    names = [f[0] for f in gdn2.Params._fields_]
    assert names == _header_param_fields()
    assert names[-7:] == ["conv_w", "gate_logits", "conv_state_in", "conv_state_out", "gate_heads", "n_seqs",
                          "cu_seqlens"]
    assert gdn2.make_params(1, 1, 1, 1, 16, 16, gate_logits=True).gate_logits == 1
    assert gdn2.conv_state_shape(2, 16, 48, 128, 128) == (2, 3, 10240)


def test_workspace_query_is_host_only(L):
    assert L.gdn2_chunk_fwd_workspace(None) == 0
    assert gdn2.chunk_fwd_workspace(_params(B=-1)) == 0
    # the precise path needs no workspace
    assert gdn2.chunk_fwd_workspace(_params(precision=1)) == 0


def test_noalloc_validates_like_chunk_fwd(L):
    """gdn2_chunk_fwd_noalloc runs the shared validation first: invalid
    parameters get the statuses of gdn2_chunk_fwd (not UNSUPPORTED), before
    any CUDA call, and the status queries refuse a misaligned workspace."""
    fn = L.gdn2_chunk_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(gdn2.Params)] + [ctypes.c_void_p] * 10
    fn.restype = ctypes.c_int
    ptrs = [FAKE * (i + 1) for i in range(9)]
    for kw, expect in ((dict(B=-1), gdn2.ERR_INVALID_ARG), (dict(H_qk=2, H_v=3), gdn2.ERR_INVALID_ARG),
                       (dict(gate_mode=5), gdn2.ERR_INVALID_ARG), (dict(chunk=48), gdn2.ERR_UNSUPPORTED),
                       (dict(d_k=24, d_v=24), gdn2.ERR_UNSUPPORTED)):
        assert fn(ctypes.byref(_params(**kw)), *ptrs, None) == expect, kw
    # valid, but the fp32 path needs no scratch
    assert fn(ctypes.byref(_params()), *ptrs, None) == gdn2.ERR_UNSUPPORTED
    assert L.gdn2_chunk_fwd_status(FAKE + 16, None) == gdn2.ERR_INVALID_ARG
    assert L.gdn2_chunk_fwd_status(None, None) == gdn2.OK
