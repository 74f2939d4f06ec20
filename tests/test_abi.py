"""The C-ABI library loads and exports every symbol include/gdn.h declares; host-side validation
rejects bad arguments before anything is launched (CPU only: no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

import linear_attention_sequence_rule_b200 as gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 1 << 20  # a 16-byte-aligned, never-dereferenced address: every call below fails first


def declared_symbols():
    names = set()
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if hdr.endswith(".h"):
            text = open(os.path.join(ROOT, "include", hdr)).read()
            names |= set(re.findall(r"GDN_API[^;(]*?\b(gdn_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert {"gdn_chunk_fwd", "gdn_decode_step", "gdn_chunk_fwd_workspace_bytes",
            "gdn_status_string", "gdn_last_error", "gdn_version"} <= names
    lib = ctypes.CDLL(gdn.LIB_PATH)
    for n in sorted(names):
        assert hasattr(lib, n), f"{n} declared in include/ but not exported by libgdn.so"


def test_status_strings_and_version():
    assert gdn.gdn_status_string(0) == "GDN_OK"
    assert gdn.gdn_status_string(-2) == "GDN_ERR_UNSUPPORTED"
    assert gdn.gdn_status_string(-99) == "GDN_ERR_UNKNOWN"
    assert gdn.gdn_version().startswith("gdn-b200")


def chunk(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, log_alpha=FAKE, beta=FAKE, S0=None, out=FAKE, S_final=None,
             B=1, T=64, H=1, dk=64, dv=64, chunk=64, cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16,
             workspace=None, workspace_bytes=0, stream=None)
    a.update(kw)
    return gdn.gdn_chunk_fwd(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dv=192), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=512), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dv=512), gdn.GDN_ERR_UNSUPPORTED),
    (dict(chunk=32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(chunk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(chunk=128, workspace=None), gdn.GDN_ERR_WORKSPACE),   # the general path needs its scratch
    (dict(dk=256, workspace=None), gdn.GDN_ERR_WORKSPACE),
    (dict(B=0), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(H=0), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(T=0), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(T=-5, cu_seqlens=FAKE), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(q=None), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(out=None), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(beta=None), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(k=FAKE + 4), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(cu_seqlens=FAKE + 8), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(S0=FAKE, S_final=FAKE + 16), gdn.GDN_ERR_INVALID_ARGUMENT),
])
def test_chunk_fwd_rejects_bad_arguments(kw, code):
    assert chunk(**kw) == code
    assert gdn.gdn_last_error() != ""


def fused(**kw):
    a = dict(q_raw=FAKE, k_raw=FAKE, v=FAKE, a_raw=FAKE, b_raw=FAKE, S0=None, out=FAKE, S_final=None,
             B=1, T=64, H=1, dk=64, dv=64, chunk=64, cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16,
             a_scale=1.0, b_scale=1.0, workspace=None, workspace_bytes=0, stream=None)
    a.update(kw)
    return gdn.gdn_chunk_fwd_fused(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=gdn.GDN_DTYPE_F32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=256), gdn.GDN_ERR_UNSUPPORTED),
    (dict(chunk=128), gdn.GDN_ERR_UNSUPPORTED),
    (dict(a_scale=-1.0), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(a_scale=float("inf")), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(a_scale=float("nan")), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(b_scale=2.5), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(b_scale=-0.1), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(b_raw=None), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(k_raw=FAKE + 4), gdn.GDN_ERR_INVALID_ARGUMENT),
])
def test_fused_chunk_fwd_rejects_bad_arguments(kw, code):
    assert fused(**kw) == code
    assert "gdn_chunk_fwd" in gdn.gdn_last_error()


def test_grouped_entries_reject_bad_head_counts():
    base = dict(q=FAKE, k=FAKE, v=FAKE, log_alpha=FAKE, beta=FAKE, S0=None, out=FAKE, S_final=None,
                B=1, T=64, dk=64, dv=64, chunk=64, cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16,
                workspace=None, workspace_bytes=0, stream=None)
    for Hk, Hv in ((2, 3), (0, 4), (4, 2), (2, 0)):
        assert gdn.gdn_chunk_fwd_gva(Hk=Hk, Hv=Hv, **base) == gdn.GDN_ERR_INVALID_ARGUMENT
        assert "gdn_chunk_fwd_gva" in gdn.gdn_last_error()
        assert gdn.gdn_decode_step_gva(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, Hk, Hv, 64, 64,
                                       gdn.GDN_DTYPE_BF16, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    # a valid grouping still meets the ordinary checks
    assert gdn.gdn_chunk_fwd_gva(Hk=2, Hv=4, **(base | dict(dk=96))) == gdn.GDN_ERR_UNSUPPORTED
    assert gdn.gdn_decode_step_gva(FAKE, FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 4, 64, 64,
                                   gdn.GDN_DTYPE_BF16, None) == gdn.GDN_ERR_INVALID_ARGUMENT


def test_workspace_query():
    assert gdn.gdn_chunk_fwd_workspace_bytes(1, 64, 1, 64, 64, 64, 0, 1) >= 0
    bad = ctypes.c_size_t(-1).value
    assert gdn.gdn_chunk_fwd_workspace_bytes(1, 64, 1, 96, 64, 64, 0, 1) == bad
    assert gdn.gdn_chunk_fwd_workspace_bytes(0, 64, 1, 64, 64, 64, 0, 1) == bad
    assert gdn.gdn_chunk_fwd_workspace_bytes(1, 64, 1, 64, 64, 96, 0, 1) == bad
    # value head size 256 with bf16: column blocks of the fused kernel (no segment scan, so no
    # workspace)
    assert gdn.gdn_chunk_fwd_workspace_bytes(1, 4096, 1, 128, 256, 64, 0, 1) == 0
    # the general path (chunk 128, key head size 256, fp32 at dv 256) passes its per-chunk factors
    # through the workspace: W, U~ (C x dk, C x dv), P (C x C) and two decay vectors per chunk and
    # head, plus the chunk table
    for B, T, H, dk, dv, C, varlen, dt in ((1, 64, 1, 64, 64, 128, 0, 1), (2, 300, 3, 256, 128, 64, 0, 1),
                                           (3, 1000, 2, 128, 256, 128, 1, 0), (1, 64, 1, 128, 256, 64, 0, 0)):
        n = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, dk, dv, C, varlen, dt)
        chunks = (T // C + B) if varlen else B * ((T + C - 1) // C)
        assert n >= chunks * H * C * (dk + dv + C + 2) * 4, (B, T, H, dk, dv, C)


def decode(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, log_alpha=FAKE, beta=FAKE, S_inout=FAKE, out=FAKE, N=1, H=1,
             dk=128, dv=128, dtype=gdn.GDN_DTYPE_BF16, stream=None)
    a.update(kw)
    return gdn.gdn_decode_step(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=3), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=512), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dv=192), gdn.GDN_ERR_UNSUPPORTED),
    (dict(N=0), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(H=-1), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(S_inout=None), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(out=FAKE + 2), gdn.GDN_ERR_INVALID_ARGUMENT),
])
def test_decode_rejects_bad_arguments(kw, code):
    assert decode(**kw) == code
    assert gdn.gdn_last_error() != ""


def test_fused_decode_rejects_bad_arguments():
    a = dict(q_raw=FAKE, k_raw=FAKE, v=FAKE, a_raw=FAKE, b_raw=FAKE, S_inout=FAKE, out=FAKE, N=1, H=1, dk=128,
             dv=128, dtype=gdn.GDN_DTYPE_BF16, a_scale=1.0, b_scale=1.0, stream=None)
    assert gdn.gdn_decode_step_fused(**(a | dict(dk=96))) == gdn.GDN_ERR_UNSUPPORTED
    assert gdn.gdn_decode_step_fused(**(a | dict(b_scale=2.5))) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert gdn.gdn_decode_step_fused(**(a | dict(a_scale=-1.0))) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert gdn.gdn_decode_step_fused(**(a | dict(a_scale=float("inf")))) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert gdn.gdn_decode_step_fused(**(a | dict(out=FAKE + 2))) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert "gdn_decode_step_fused" in gdn.gdn_last_error()


def test_torch_layer_checks_shapes_without_launching():
    import torch
    q = torch.zeros(1, 64, 1, 64)
    with pytest.raises(ValueError):
        gdn.chunk_fwd(q, q, q[..., :32], torch.zeros(1, 64, 1), torch.zeros(1, 64, 2))


def test_backward_entry_validation():
    a = dict(q=FAKE, k=FAKE, v=FAKE, log_alpha=FAKE, beta=FAKE, S0=None, dout=FAKE, dS_final=None, dq=FAKE,
             dk=FAKE, dv=FAKE, dlog_alpha=FAKE, dbeta=FAKE, dS0=None, B=1, T=64, H=1, dk_=64, dv_=64, chunk=64,
             cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16, workspace=None, workspace_bytes=0, stream=None)
    assert gdn.gdn_chunk_bwd(**(a | dict(dk_=96, dv_=128))) == gdn.GDN_ERR_UNSUPPORTED
    assert gdn.gdn_chunk_bwd(**(a | dict(dk_=256, dv_=64))) == gdn.GDN_ERR_UNSUPPORTED
    assert gdn.gdn_chunk_bwd(**(a | dict(dq=None))) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert gdn.gdn_chunk_bwd(**(a | dict(dbeta=FAKE + 4))) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert gdn.gdn_chunk_bwd(**a) == gdn.GDN_ERR_WORKSPACE
    assert "gdn_chunk_bwd" in gdn.gdn_last_error()
    assert gdn.gdn_chunk_bwd_workspace_bytes(1, 64, 1, 256, 128, 64, 0) == (1 << 64) - 1
    assert gdn.gdn_chunk_bwd_workspace_bytes(2, 128, 3, 64, 64, 64, 0) > 5 * 2 * 2 * 3 * 64 * 64 * 4 - 1
    # value head sizes 128 and 256 (64-column value splits): more workspace; other sizes rejected
    w64 = gdn.gdn_chunk_bwd_workspace_bytes(2, 128, 3, 64, 64, 64, 0)
    assert gdn.gdn_chunk_bwd_workspace_bytes(2, 128, 3, 64, 128, 64, 0) > 2 * w64 - 4096
    assert gdn.gdn_chunk_bwd_workspace_bytes(2, 128, 3, 64, 256, 64, 1) > 4 * w64 - 4096
    assert gdn.gdn_chunk_bwd_workspace_bytes(2, 128, 3, 64, 96, 64, 0) == (1 << 64) - 1
    # key head size 128 (two key blocks): sixteen matrices per unit instead of eight
    assert gdn.gdn_chunk_bwd_workspace_bytes(2, 128, 3, 128, 64, 64, 0) > 2 * w64 - 4096
    assert gdn.gdn_chunk_bwd(**(a | dict(dv_=128))) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_chunk_bwd(**(a | dict(dv_=512))) == gdn.GDN_ERR_UNSUPPORTED


def host_chunk(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, log_alpha=FAKE, beta=FAKE, S0=None, out=FAKE, S_final=None,
             B=2, T=64, H=1, dk=64, dv=64, chunk=64, cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16,
             workspace=FAKE * 256, workspace_bytes=1 << 40, stream=None)
    a.update(kw)
    return gdn.gdn_chunk_fwd_host(**a)


def _cu(*vals):
    arr = (ctypes.c_int32 * len(vals))(*vals)
    return ctypes.cast(arr, ctypes.c_void_p).value, arr


def test_host_entry_workspace_covers_every_input_and_output():
    # bf16 dense, no segment scan needed for one-sequence parts this short
    n = gdn.gdn_chunk_fwd_host_workspace_bytes(2, 64, 1, 64, 64, 64, 0, gdn.GDN_DTYPE_BF16)
    tokens = 2 * 64
    assert n >= 3 * tokens * 64 * 2 + 2 * tokens * 4 + 2 * 2 * 64 * 64 * 4 + tokens * 64 * 2
    assert gdn.gdn_chunk_fwd_host_workspace_bytes(2, 64, 1, 96, 64, 64, 0, gdn.GDN_DTYPE_BF16) == \
        ctypes.c_size_t(-1).value


def test_host_entry_rejects_before_any_copy():
    assert host_chunk(dk=96) == gdn.GDN_ERR_UNSUPPORTED
    assert host_chunk(B=0) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert host_chunk(out=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert host_chunk(q=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert host_chunk(workspace=None) == gdn.GDN_ERR_WORKSPACE
    assert host_chunk(workspace_bytes=16) == gdn.GDN_ERR_WORKSPACE
    assert host_chunk(workspace=FAKE * 256 + 16) == gdn.GDN_ERR_INVALID_ARGUMENT
    p, keep = _cu(0, 10, 5)  # decreasing
    assert host_chunk(T=5, cu_seqlens=p) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert "decreases" in gdn.gdn_last_error()
    p, keep = _cu(1, 3, 5)  # does not start at 0
    assert host_chunk(T=5, cu_seqlens=p) == gdn.GDN_ERR_INVALID_ARGUMENT
    p, keep = _cu(0, 3, 5)  # does not end at T
    assert host_chunk(T=6, cu_seqlens=p) == gdn.GDN_ERR_INVALID_ARGUMENT


def phase_call(**kw):
    a = dict(K=FAKE, Q=FAKE, v=FAKE, log_lam=FAKE, beta=FAKE, M0=None, out=FAKE, M_final=None, B=1, T=64, H=1,
             dk=32, dv=64, cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16, workspace=FAKE * 256, workspace_bytes=1 << 40,
             stream=None)
    a.update(kw)
    return gdn.gdn_phase_fwd(**a)


def test_phase_entry_rejects_before_any_launch():
    assert phase_call(dk=48) == gdn.GDN_ERR_UNSUPPORTED
    assert phase_call(dk=128) == gdn.GDN_ERR_UNSUPPORTED   # 2 dk = 256 real columns
    assert phase_call(dv=96) == gdn.GDN_ERR_UNSUPPORTED
    assert phase_call(dv=256, dtype=gdn.GDN_DTYPE_F32) == gdn.GDN_ERR_UNSUPPORTED  # 256 with bf16 only
    assert gdn.gdn_phase_fwd_workspace_bytes(1, 64, 1, 32, 256, 0, gdn.GDN_DTYPE_BF16) != ctypes.c_size_t(-1).value
    assert phase_call(B=0) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert phase_call(K=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert phase_call(out=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert phase_call(Q=FAKE + 8) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert phase_call(workspace=None) == gdn.GDN_ERR_WORKSPACE
    assert phase_call(workspace_bytes=1024) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_phase_fwd_workspace_bytes(1, 64, 1, 48, 64, 0, gdn.GDN_DTYPE_BF16) == ctypes.c_size_t(-1).value
    n = gdn.gdn_phase_fwd_workspace_bytes(2, 64, 3, 32, 64, 0, gdn.GDN_DTYPE_BF16)
    token_heads = 2 * 64 * 3
    assert n >= token_heads * (2 * 64 * 2 + 2 * 64 * 2 + 64 * 2 + 4)


def test_fused_backward_rejects_before_any_launch():
    a = dict(q_raw=FAKE, k_raw=FAKE, v=FAKE, a_raw=FAKE, b_raw=FAKE, S0=None, dout=FAKE, dS_final=None, dq_raw=FAKE,
             dk_raw=FAKE, dv=FAKE, da_raw=FAKE, db_raw=FAKE, dS0=None, B=1, T=64, H=1, dk=64, dv_=64, chunk=64,
             cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16, a_scale=1.0, b_scale=1.0, workspace=FAKE * 256,
             workspace_bytes=1 << 40, stream=None)

    def call(**kw):
        return gdn.gdn_chunk_bwd_fused(**dict(a, **kw))
    assert call(dk=128) == gdn.GDN_ERR_UNSUPPORTED
    assert call(dtype=9) == gdn.GDN_ERR_UNSUPPORTED
    assert call(b_scale=2.5) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert call(a_scale=-1.0) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert call(db_raw=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert call(dout=FAKE + 4) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert call(workspace=None) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_chunk_bwd_fused_workspace_bytes(1, 64, 1, 128, 64, 64, 0) == ctypes.c_size_t(-1).value
    assert call(dv_=96) == gdn.GDN_ERR_UNSUPPORTED
    assert gdn.gdn_chunk_bwd_fused_workspace_bytes(1, 64, 1, 64, 256, 64, 0) > \
        gdn.gdn_chunk_bwd_fused_workspace_bytes(1, 64, 1, 64, 64, 64, 0)


def test_grouped_backward_rejects_bad_groups():
    a = dict(q=FAKE, k=FAKE, v=FAKE, log_alpha=FAKE, beta=FAKE, S0=None, dout=FAKE, dS_final=None, dq=FAKE, dk=FAKE,
             dv=FAKE, dlog_alpha=FAKE, dbeta=FAKE, dS0=None, B=1, T=64, Hk=2, Hv=5, dk_=64, dv_=64, chunk=64,
             cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16, workspace=FAKE * 256, workspace_bytes=1 << 40, stream=None)
    assert gdn.gdn_chunk_bwd_gva(**a) == gdn.GDN_ERR_INVALID_ARGUMENT        # 5 value heads on 2 q/k heads
    assert gdn.gdn_chunk_bwd_gva(**dict(a, Hv=4, dk_=96)) == gdn.GDN_ERR_UNSUPPORTED
    assert gdn.gdn_chunk_bwd_gva(**dict(a, Hv=4, workspace=None)) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_chunk_bwd_gva_workspace_bytes(1, 64, 2, 5, 64, 64, 64, 0) == ctypes.c_size_t(-1).value
    plain = gdn.gdn_chunk_bwd_workspace_bytes(1, 64, 4, 64, 64, 64, 0)
    assert gdn.gdn_chunk_bwd_gva_workspace_bytes(1, 64, 2, 4, 64, 64, 64, 0) >= plain + 2 * 64 * 4 * 64 * 4


def test_phase_backward_rejects_before_any_launch():
    a = dict(K=FAKE, Q=FAKE, v=FAKE, log_lam=FAKE, beta=FAKE, M0=None, dout=FAKE, dM_final=None, dK=FAKE, dQ=FAKE,
             dv_out=FAKE, dlog_lam=FAKE, dbeta=FAKE, dM0=None, B=1, T=64, H=1, dk=32, dv=64, cu_seqlens=None,
             dtype=gdn.GDN_DTYPE_BF16, workspace=FAKE * 256, workspace_bytes=1 << 40, stream=None)
    assert gdn.gdn_phase_bwd(**dict(a, dk=64)) == gdn.GDN_ERR_UNSUPPORTED   # the backward takes 64 real columns
    assert gdn.gdn_phase_bwd(**dict(a, dv=512)) == gdn.GDN_ERR_UNSUPPORTED
    assert gdn.gdn_phase_bwd_workspace_bytes(1, 64, 1, 32, 128, 0) > gdn.gdn_phase_bwd_workspace_bytes(1, 64, 1, 32, 64, 0)
    assert gdn.gdn_phase_bwd(**dict(a, dQ=None)) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert gdn.gdn_phase_bwd(**dict(a, K=FAKE + 4)) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert gdn.gdn_phase_bwd(**dict(a, workspace=None)) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_phase_bwd_workspace_bytes(1, 64, 1, 64, 64, 0) == ctypes.c_size_t(-1).value


def declared_prototypes():
    """name -> (return type, [parameter types]) for every GDN_API declaration in include/."""
    protos = {}
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if not hdr.endswith(".h"):
            continue
        text = re.sub(r"/\*.*?\*/", " ", open(os.path.join(ROOT, "include", hdr)).read(), flags=re.S)
        for ret, name, params in re.findall(r"GDN_API\s+([^;(]*?)\b(gdn_\w+)\s*\(([^)]*)\)\s*;", text):
            plist = [p.strip() for p in params.split(",") if p.strip() and p.strip() != "void"]
            protos[name] = (" ".join(ret.split()), plist)
    return protos


def ctype_of(decl):
    """The ctypes type a C parameter or return type must be marshalled as."""
    if "*" in decl:
        return ctypes.c_char_p if decl.replace(" ", "").startswith("constchar*") else ctypes.c_void_p
    words = decl.replace("const", "").split()
    base = words[0]
    return {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "float": ctypes.c_float}[base]


def test_binding_signatures_match_the_header():
    # every entry's ctypes argtypes and restype agree with its C prototype, parameter by parameter
    # (a shifted or mistyped argument would reach a kernel as a wrong pointer or size)
    protos = declared_prototypes()
    assert len(protos) >= 20
    for name, (ret, params) in sorted(protos.items()):
        fn = getattr(gdn._lib, name)
        assert fn.argtypes is not None, f"{name}: no argtypes"
        got = list(fn.argtypes)
        want = [ctype_of(p) for p in params]
        assert got == want, f"{name}: argtypes {got} != header {want}"
        assert fn.restype == ctype_of(ret), f"{name}: restype {fn.restype} != header {ret}"


def rowdecay_call(**kw):
    a = dict(K=FAKE, Q=FAKE, v=FAKE, log_r=FAKE, beta=FAKE, M0=None, out=FAKE, M_final=None, B=1, T=64, H=1,
             dk=32, dv=64, cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16, stream=None)
    a.update(kw)
    return gdn.gdn_phase_rowdecay_fwd(**a)


def test_rowdecay_entry_rejects_before_any_launch():
    assert rowdecay_call(dk=48) == gdn.GDN_ERR_UNSUPPORTED
    assert rowdecay_call(dk=128) == gdn.GDN_ERR_UNSUPPORTED
    assert rowdecay_call(dv=0) == gdn.GDN_ERR_UNSUPPORTED
    assert rowdecay_call(dv=5000) == gdn.GDN_ERR_UNSUPPORTED
    assert rowdecay_call(dtype=7) == gdn.GDN_ERR_UNSUPPORTED
    assert rowdecay_call(B=0) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert rowdecay_call(T=0) == gdn.GDN_ERR_INVALID_ARGUMENT          # dense needs T >= 1
    assert rowdecay_call(log_r=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert rowdecay_call(out=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert rowdecay_call(K=FAKE + 8) == gdn.GDN_ERR_INVALID_ARGUMENT   # not 16-byte aligned
    # M0 and M_final overlapping partially
    assert rowdecay_call(M0=FAKE, M_final=FAKE + 256) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert "rowdecay" in gdn.gdn_last_error()


def noalloc(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, log_alpha=FAKE, beta=FAKE, S0=None, out=FAKE, S_final=None,
             B=1, T=64, H=1, dk=64, dv=64, chunk=64, cu_seqlens=None, dtype=gdn.GDN_DTYPE_BF16,
             stream=None)
    a.update(kw)
    return gdn.gdn_chunk_fwd_noalloc(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(chunk=32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(B=0), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(q=None), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(out=None), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(k=FAKE + 4), gdn.GDN_ERR_INVALID_ARGUMENT),
    (dict(S0=FAKE, S_final=FAKE + 16), gdn.GDN_ERR_INVALID_ARGUMENT),
    # one long sequence (a segmented plan on a device) with a bad pointer
    (dict(T=65536, q=None), gdn.GDN_ERR_INVALID_ARGUMENT),
])
def test_noalloc_entry_rejects_before_touching_the_device(kw, code):
    """Every argument is checked on the host before the library's scratch array is looked up: on
    this machine, without a device, a lookup would fail with GDN_ERR_CUDA instead."""
    assert noalloc(**kw) == code
    assert "gdn_chunk_fwd" in gdn.gdn_last_error()  # the shape checks are gdn_chunk_fwd's own


def test_noalloc_entry_rejects_oversized_scratch_on_the_host():
    # chunk 128 runs on the general path, whose workspace grows with the token count: far beyond
    # the 32 MiB array for a long sequence
    B, T, H, dk, dv = 1, 65536, 16, 128, 128
    need = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, dk, dv, 128, 0, gdn.GDN_DTYPE_BF16)
    assert need > 32 * 2 ** 20
    assert noalloc(B=B, T=T, H=H, dk=dk, dv=dv, chunk=128) == gdn.GDN_ERR_WORKSPACE
    assert "32 MiB" in gdn.gdn_last_error() or str(32 * 2 ** 20) in gdn.gdn_last_error()
