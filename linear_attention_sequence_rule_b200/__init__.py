"""Python binding of libgdn, the B200 (sm_100a) gated delta-rule library.

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
PyTorch provides device memory and streams.  The binding has two layers:

* ``gdn_chunk_fwd``, ``gdn_chunk_fwd_noalloc``, ``gdn_chunk_fwd_host``, ``gdn_phase_fwd``,
  ``gdn_phase_rowdecay_fwd``, ``gdn_decode_step``,
  ``gdn_chunk_fwd_workspace_bytes``, ``gdn_chunk_fwd_host_workspace_bytes``,
  ``gdn_status_string``, ``gdn_last_error``, ``gdn_version`` -- the C-ABI entry points of
  ``include/gdn.h`` with the same names and arguments (pointers as Python ints);
* ``chunk_fwd``, ``chunk_fwd_host``, ``chunk_fwd_fused``, ``chunk_fwd_gva``, ``chunk_bwd``,
  ``chunk_bwd_fused``, ``chunk_bwd_gva``, ``phase_fwd``, ``phase_rowdecay_fwd``, ``phase_bwd``, ``decode_step``,
  ``decode_step_fused`` and ``decode_step_gva`` --
  the same calls taking torch tensors; they check shapes,
  devices and dtypes, allocate outputs with torch when none are given, and raise ``GdnError``
  on a non-zero status.

If ``libgdn.so`` has not been built, importing this package raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "GdnError", "GDN_OK", "GDN_ERR_INVALID_ARGUMENT", "GDN_ERR_UNSUPPORTED", "GDN_ERR_WORKSPACE",
    "GDN_ERR_CUDA", "GDN_ERR_TIMEOUT", "GDN_DTYPE_F32", "GDN_DTYPE_BF16", "LIB_PATH",
    "gdn_chunk_fwd", "gdn_chunk_fwd_noalloc", "gdn_chunk_fwd_fused", "gdn_chunk_fwd_gva",
    "gdn_chunk_fwd_host", "gdn_chunk_fwd_host_workspace_bytes", "chunk_fwd_host",
    "gdn_phase_fwd", "gdn_phase_fwd_workspace_bytes", "phase_fwd",
    "gdn_phase_rowdecay_fwd", "phase_rowdecay_fwd",
    "gdn_phase_bwd", "gdn_phase_bwd_workspace_bytes", "phase_bwd",
    "gdn_chunk_bwd_fused", "gdn_chunk_bwd_fused_workspace_bytes", "chunk_bwd_fused",
    "gdn_chunk_bwd_gva", "gdn_chunk_bwd_gva_workspace_bytes", "chunk_bwd_gva",
    "gdn_decode_step", "gdn_decode_step_fused", "decode_step_fused", "gdn_decode_step_gva", "gdn_chunk_bwd", "gdn_chunk_bwd_workspace_bytes", "gdn_chunk_fwd_workspace_bytes", "gdn_status_string",
    "gdn_last_error", "gdn_version", "gdn_device_status", "gdn_selftest_wait_timeout", "device_status", "chunk_fwd", "chunk_fwd_fused",
    "chunk_fwd_gva", "chunk_bwd", "decode_step", "decode_step_gva", "workspace_bytes",
]

GDN_OK = 0
GDN_ERR_INVALID_ARGUMENT = -1
GDN_ERR_UNSUPPORTED = -2
GDN_ERR_WORKSPACE = -3
GDN_ERR_CUDA = -4
GDN_ERR_TIMEOUT = -5
GDN_DTYPE_F32 = 0
GDN_DTYPE_BF16 = 1

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python linear_attention_sequence_rule_b200/build.py`"
        " (there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

_vp, _sz, _i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
_lib.gdn_chunk_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                               _vp, _i, _vp, _sz, _vp]
_lib.gdn_chunk_fwd.restype = _i
_lib.gdn_chunk_fwd_fused.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                     _vp, _i, ctypes.c_float, ctypes.c_float, _vp, _sz, _vp]
_lib.gdn_chunk_fwd_fused.restype = _i
_lib.gdn_chunk_fwd_gva.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                   _vp, _i, _vp, _sz, _vp]
_lib.gdn_chunk_fwd_gva.restype = _i
_lib.gdn_decode_step_gva.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
_lib.gdn_decode_step_gva.restype = _i
_lib.gdn_chunk_bwd.argtypes = [_vp] * 14 + [_i] * 6 + [_vp, _i, _vp, _sz, _vp]
_lib.gdn_chunk_bwd.restype = _i
_lib.gdn_chunk_bwd_fused.argtypes = [_vp] * 14 + [_i] * 6 + [_vp, _i, ctypes.c_float, ctypes.c_float, _vp, _sz, _vp]
_lib.gdn_chunk_bwd_fused.restype = _i
_lib.gdn_chunk_bwd_fused_workspace_bytes.argtypes = [_i] * 7
_lib.gdn_chunk_bwd_fused_workspace_bytes.restype = _sz
_lib.gdn_chunk_bwd_gva.argtypes = [_vp] * 14 + [_i] * 7 + [_vp, _i, _vp, _sz, _vp]
_lib.gdn_chunk_bwd_gva.restype = _i
_lib.gdn_chunk_bwd_gva_workspace_bytes.argtypes = [_i] * 8
_lib.gdn_chunk_bwd_gva_workspace_bytes.restype = _sz
_lib.gdn_chunk_bwd_workspace_bytes.argtypes = [_i] * 7
_lib.gdn_chunk_bwd_workspace_bytes.restype = _sz
_lib.gdn_chunk_fwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                       _i, _vp, _i, _vp]
_lib.gdn_chunk_fwd_noalloc.restype = _i
_lib.gdn_chunk_fwd_host.argtypes = list(_lib.gdn_chunk_fwd.argtypes)
_lib.gdn_chunk_fwd_host.restype = _i
_lib.gdn_chunk_fwd_host_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i]
_lib.gdn_chunk_fwd_host_workspace_bytes.restype = _sz
_lib.gdn_phase_fwd.argtypes = [_vp] * 8 + [_i] * 5 + [_vp, _i, _vp, _sz, _vp]
_lib.gdn_phase_fwd.restype = _i
_lib.gdn_phase_fwd_workspace_bytes.argtypes = [_i] * 7
_lib.gdn_phase_rowdecay_fwd.argtypes = [_vp] * 8 + [_i] * 5 + [_vp, _i, _vp]
_lib.gdn_phase_rowdecay_fwd.restype = _i
_lib.gdn_phase_bwd.argtypes = [_vp] * 14 + [_i] * 5 + [_vp, _i, _vp, _sz, _vp]
_lib.gdn_phase_bwd.restype = _i
_lib.gdn_phase_bwd_workspace_bytes.argtypes = [_i] * 6
_lib.gdn_phase_bwd_workspace_bytes.restype = _sz
_lib.gdn_phase_fwd_workspace_bytes.restype = _sz
_lib.gdn_chunk_fwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i]
_lib.gdn_chunk_fwd_workspace_bytes.restype = _sz
_lib.gdn_decode_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
_lib.gdn_decode_step.restype = _i
_lib.gdn_decode_step_fused.argtypes = [_vp] * 7 + [_i] * 5 + [ctypes.c_float, ctypes.c_float, _vp]
_lib.gdn_decode_step_fused.restype = _i
_lib.gdn_selftest_wait_timeout.argtypes = [_i, _vp]
_lib.gdn_selftest_wait_timeout.restype = _i
_lib.gdn_device_status.argtypes = [_vp]
_lib.gdn_device_status.restype = _i
_lib.gdn_status_string.argtypes = [_i]
_lib.gdn_status_string.restype = ctypes.c_char_p
_lib.gdn_last_error.argtypes = []
_lib.gdn_last_error.restype = ctypes.c_char_p
_lib.gdn_version.argtypes = []
_lib.gdn_version.restype = ctypes.c_char_p


class GdnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{gdn_status_string(status)}: {message}")
        self.status = status


# ---- C-ABI mirrors ---------------------------------------------------------------------------

def gdn_chunk_fwd(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk, cu_seqlens,
                  dtype, workspace, workspace_bytes, stream) -> int:
    return _lib.gdn_chunk_fwd(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk,
                              cu_seqlens, dtype, workspace, workspace_bytes, stream)


def gdn_chunk_fwd_fused(q_raw, k_raw, v, a_raw, b_raw, S0, out, S_final, B, T, H, dk, dv, chunk,
                        cu_seqlens, dtype, a_scale, b_scale, workspace, workspace_bytes, stream) -> int:
    return _lib.gdn_chunk_fwd_fused(q_raw, k_raw, v, a_raw, b_raw, S0, out, S_final, B, T, H, dk, dv,
                                    chunk, cu_seqlens, dtype, a_scale, b_scale, workspace,
                                    workspace_bytes, stream)


def gdn_chunk_fwd_gva(q, k, v, log_alpha, beta, S0, out, S_final, B, T, Hk, Hv, dk, dv, chunk,
                      cu_seqlens, dtype, workspace, workspace_bytes, stream) -> int:
    return _lib.gdn_chunk_fwd_gva(q, k, v, log_alpha, beta, S0, out, S_final, B, T, Hk, Hv, dk, dv, chunk,
                                  cu_seqlens, dtype, workspace, workspace_bytes, stream)


def gdn_decode_step_gva(q, k, v, log_alpha, beta, S_inout, out, N, Hk, Hv, dk, dv, dtype,
                        stream) -> int:
    return _lib.gdn_decode_step_gva(q, k, v, log_alpha, beta, S_inout, out, N, Hk, Hv, dk, dv, dtype,
                                    stream)


def gdn_chunk_bwd(q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk, dv, dlog_alpha, dbeta, dS0, B, T,
                  H, dk_, dv_, chunk, cu_seqlens, dtype, workspace, workspace_bytes, stream) -> int:
    return _lib.gdn_chunk_bwd(q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk, dv, dlog_alpha, dbeta,
                              dS0, B, T, H, dk_, dv_, chunk, cu_seqlens, dtype, workspace, workspace_bytes,
                              stream)


def gdn_chunk_bwd_workspace_bytes(B, T, H, dk, dv, chunk, varlen) -> int:
    return _lib.gdn_chunk_bwd_workspace_bytes(B, T, H, dk, dv, chunk, varlen)


def gdn_chunk_fwd_noalloc(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk,
                          cu_seqlens, dtype, stream) -> int:
    return _lib.gdn_chunk_fwd_noalloc(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv,
                                      chunk, cu_seqlens, dtype, stream)


def gdn_chunk_fwd_host(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk, cu_seqlens,
                       dtype, workspace, workspace_bytes, stream) -> int:
    return _lib.gdn_chunk_fwd_host(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk,
                                   cu_seqlens, dtype, workspace, workspace_bytes, stream)


def gdn_chunk_fwd_host_workspace_bytes(B, T, H, dk, dv, chunk, varlen, dtype) -> int:
    return _lib.gdn_chunk_fwd_host_workspace_bytes(B, T, H, dk, dv, chunk, varlen, dtype)


def gdn_phase_fwd(K, Q, v, log_lam, beta, M0, out, M_final, B, T, H, dk, dv, cu_seqlens, dtype, workspace,
                  workspace_bytes, stream) -> int:
    return _lib.gdn_phase_fwd(K, Q, v, log_lam, beta, M0, out, M_final, B, T, H, dk, dv, cu_seqlens, dtype,
                              workspace, workspace_bytes, stream)


def gdn_phase_rowdecay_fwd(K, Q, v, log_r, beta, M0, out, M_final, B, T, H, dk, dv, cu_seqlens, dtype,
                           stream) -> int:
    return _lib.gdn_phase_rowdecay_fwd(K, Q, v, log_r, beta, M0, out, M_final, B, T, H, dk, dv, cu_seqlens, dtype,
                                       stream)


def gdn_phase_fwd_workspace_bytes(B, T, H, dk, dv, varlen, dtype) -> int:
    return _lib.gdn_phase_fwd_workspace_bytes(B, T, H, dk, dv, varlen, dtype)


def gdn_phase_bwd(K, Q, v, log_lam, beta, M0, dout, dM_final, dK, dQ, dv_out, dlog_lam, dbeta, dM0, B, T, H, dk,
                  dv, cu_seqlens, dtype, workspace, workspace_bytes, stream) -> int:
    return _lib.gdn_phase_bwd(K, Q, v, log_lam, beta, M0, dout, dM_final, dK, dQ, dv_out, dlog_lam, dbeta, dM0, B,
                              T, H, dk, dv, cu_seqlens, dtype, workspace, workspace_bytes, stream)


def gdn_phase_bwd_workspace_bytes(B, T, H, dk, dv, varlen) -> int:
    return _lib.gdn_phase_bwd_workspace_bytes(B, T, H, dk, dv, varlen)


def gdn_chunk_fwd_workspace_bytes(B, T, H, dk, dv, chunk, varlen, dtype) -> int:
    return _lib.gdn_chunk_fwd_workspace_bytes(B, T, H, dk, dv, chunk, varlen, dtype)


def gdn_decode_step(q, k, v, log_alpha, beta, S_inout, out, N, H, dk, dv, dtype, stream) -> int:
    return _lib.gdn_decode_step(q, k, v, log_alpha, beta, S_inout, out, N, H, dk, dv, dtype, stream)


def gdn_decode_step_fused(q_raw, k_raw, v, a_raw, b_raw, S_inout, out, N, H, dk, dv, dtype, a_scale, b_scale,
                          stream) -> int:
    return _lib.gdn_decode_step_fused(q_raw, k_raw, v, a_raw, b_raw, S_inout, out, N, H, dk, dv, dtype, a_scale,
                                      b_scale, stream)


def gdn_selftest_wait_timeout(limit_ms, stream) -> int:
    return _lib.gdn_selftest_wait_timeout(limit_ms, stream)


def gdn_device_status(stream) -> int:
    return _lib.gdn_device_status(stream)


def device_status(stream=None) -> None:
    """Synchronise and raise GdnError if a kernel recorded a device-side timeout."""
    rc = gdn_device_status(_stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())


def gdn_status_string(status: int) -> str:
    return _lib.gdn_status_string(status).decode()


def gdn_last_error() -> str:
    return _lib.gdn_last_error().decode()


def gdn_version() -> str:
    return _lib.gdn_version().decode()


# ---- torch-level calls ------------------------------------------------------------------------

_DT = {torch.bfloat16: GDN_DTYPE_BF16, torch.float32: GDN_DTYPE_F32}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t, name, dtype=None, shape=None, device=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def workspace_bytes(B, T, H, dk, dv, varlen=False, dtype=torch.bfloat16, chunk=64) -> int:
    n = gdn_chunk_fwd_workspace_bytes(B, T, H, dk, dv, chunk, int(bool(varlen)), _DT[dtype])
    if n == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_INVALID_ARGUMENT, gdn_last_error())
    return n


def _chunk_prepare(q, k, v, ga, gb, S0, cu_seqlens, out, S_final, output_final_state, workspace,
                   chunk, names, grouped=False):
    """Shape/device/dtype checks and output/workspace allocation shared by the chunk entries."""
    dt = q.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = q.device
    if cu_seqlens is not None:
        T, Hk, dk = q.shape
        B = cu_seqlens.shape[0] - 1
        lead = (T,)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    else:
        B, T, Hk, dk = q.shape
        lead = (B, T)
    dv = v.shape[-1]
    H = v.shape[-2] if grouped else Hk  # value heads
    _need(q, names[0], dt, (*lead, Hk, dk), dev)
    _need(k, names[1], dt, (*lead, Hk, dk), dev)
    _need(v, "v", dt, (*lead, H, dv), dev)
    _need(ga, names[2], torch.float32, (*lead, H), dev)
    _need(gb, names[3], torch.float32, (*lead, H), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    if out is None:
        out = torch.empty((*lead, H, dv), dtype=dt, device=dev)
    _need(out, "out", dt, (*lead, H, dv), dev)
    if S_final is None and output_final_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _need(S_final, "S_final", torch.float32, (B, H, dk, dv), dev)
    need = workspace_bytes(B, T, H, dk, dv, cu_seqlens is not None, dt, chunk)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return dict(B=B, T=T, H=H, Hk=Hk, dk=dk, dv=dv, dt=dt, out=out, S_final=S_final,
                workspace=workspace, wbytes=wbytes)


def chunk_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, out=None, S_final=None,
              output_final_state=True, workspace=None, chunk=64, stream=None):
    """Chunkwise forward.  Dense q,k [B,T,H,dk], v [B,T,H,dv]; varlen (cu_seqlens int32 [B+1] on
    the device) packs q,k [T,H,dk] ...  Returns (out, S_final or None)."""
    p = _chunk_prepare(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, output_final_state,
                       workspace, chunk, ("q", "k", "log_alpha", "beta"))
    rc = gdn_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(p["out"]),
                       _ptr(p["S_final"]), p["B"], p["T"], p["H"], p["dk"], p["dv"], chunk,
                       _ptr(cu_seqlens), _DT[p["dt"]], _ptr(p["workspace"]), p["wbytes"],
                       _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return p["out"], p["S_final"]


def chunk_fwd_host(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, out=None, S_final=None,
                   output_final_state=True, workspace=None, chunk=64, stream=None):
    """``chunk_fwd`` from and to host memory (``gdn_chunk_fwd_host``): q, k, v, gates, S0 and
    cu_seqlens are CPU tensors (page-locked ones let the copies overlap), out and S_final are
    written to CPU tensors (allocated page-locked when not given), workspace is a CUDA uint8
    tensor of ``gdn_chunk_fwd_host_workspace_bytes`` bytes (allocated on the current device when
    not given).  Asynchronous: the outputs are complete once ``stream`` has completed."""
    dt = q.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    cpu = torch.device("cpu")
    if cu_seqlens is not None:
        T, H, dk = q.shape
        B = cu_seqlens.shape[0] - 1
        lead = (T,)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), cpu)
    else:
        B, T, H, dk = q.shape
        lead = (B, T)
    dv = v.shape[-1]
    _need(q, "q", dt, (*lead, H, dk), cpu)
    _need(k, "k", dt, (*lead, H, dk), cpu)
    _need(v, "v", dt, (*lead, H, dv), cpu)
    _need(log_alpha, "log_alpha", torch.float32, (*lead, H), cpu)
    _need(beta, "beta", torch.float32, (*lead, H), cpu)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dk, dv), cpu)
    if out is None:
        out = torch.empty((*lead, H, dv), dtype=dt).pin_memory()
    _need(out, "out", dt, (*lead, H, dv), cpu)
    if S_final is None and output_final_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32).pin_memory()
    if S_final is not None:
        _need(S_final, "S_final", torch.float32, (B, H, dk, dv), cpu)
    need = gdn_chunk_fwd_host_workspace_bytes(B, T, H, dk, dv, chunk, int(cu_seqlens is not None), _DT[dt])
    if need == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_INVALID_ARGUMENT, gdn_last_error())
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    if not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    rc = gdn_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(out),
                            _ptr(S_final), B, T, H, dk, dv, chunk, _ptr(cu_seqlens), _DT[dt], _ptr(workspace),
                            workspace.numel(), _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return out, S_final


def _as_pairs(x, name):
    """A complex tensor as contiguous fp32 (re, im) pairs; real tensors must already end in 2."""
    if x is None:
        return None
    if x.is_complex():
        x = torch.view_as_real(x.to(torch.complex64).contiguous())
    if x.dtype != torch.float32 or x.shape[-1] != 2:
        raise ValueError(f"{name} must be complex64 or float32 [..., 2]")
    return x.contiguous()


def phase_fwd(K, Q, v, log_lam, beta, M0=None, cu_seqlens=None, out=None, M_final=None,
              output_final_state=True, workspace=None, stream=None):
    """Complex-phase delta memory (``gdn_phase_fwd``).  K, Q complex [B,T,H,dk] (or packed [T,H,dk]
    with cu_seqlens), complex64 or float32 [..., 2]; v [.., H, dv] bf16 (tensor-core path) or fp32;
    log_lam, beta [.., H] fp32; M0 complex [B, H, dv, dk] or None.  Returns (out, M_final complex64
    or None)."""
    Kp, Qp = _as_pairs(K, "K"), _as_pairs(Q, "Q")
    dt = v.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = v.device
    if cu_seqlens is not None:
        T, H, dk = Kp.shape[:3]
        B = cu_seqlens.shape[0] - 1
        lead = (T,)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    else:
        B, T, H, dk = Kp.shape[:4]
        lead = (B, T)
    dv = v.shape[-1]
    _need(Kp, "K", torch.float32, (*lead, H, dk, 2), dev)
    _need(Qp, "Q", torch.float32, (*lead, H, dk, 2), dev)
    _need(v, "v", dt, (*lead, H, dv), dev)
    _need(log_lam, "log_lam", torch.float32, (*lead, H), dev)
    _need(beta, "beta", torch.float32, (*lead, H), dev)
    M0p = _as_pairs(M0, "M0")
    if M0p is not None:
        _need(M0p, "M0", torch.float32, (B, H, dv, dk, 2), dev)
    if out is None:
        out = torch.empty((*lead, H, dv), dtype=dt, device=dev)
    _need(out, "out", dt, (*lead, H, dv), dev)
    Mf = None
    if M_final is not None:
        Mf = torch.view_as_real(M_final) if M_final.is_complex() else M_final
    elif output_final_state:
        Mf = torch.empty((B, H, dv, dk, 2), dtype=torch.float32, device=dev)
    if Mf is not None:
        _need(Mf, "M_final", torch.float32, (B, H, dv, dk, 2), dev)
    need = gdn_phase_fwd_workspace_bytes(B, T, H, dk, dv, int(cu_seqlens is not None), _DT[dt])
    if need == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_UNSUPPORTED, f"gdn_phase_fwd: unsupported sizes dk={dk} dv={dv}")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    rc = gdn_phase_fwd(_ptr(Kp), _ptr(Qp), _ptr(v), _ptr(log_lam), _ptr(beta), _ptr(M0p), _ptr(out), _ptr(Mf),
                       B, T, H, dk, dv, _ptr(cu_seqlens), _DT[dt], _ptr(workspace), workspace.numel(),
                       _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return out, (None if Mf is None else torch.view_as_complex(Mf))


def phase_rowdecay_fwd(K, Q, v, log_r, beta, M0=None, cu_seqlens=None, out=None, M_final=None,
                       output_final_state=True, stream=None):
    """Complex-phase delta memory with one decay per value channel (``gdn_phase_rowdecay_fwd``):
    as ``phase_fwd`` with log_r [.., H, dv] fp32 in place of log_lam.  Returns (out, M_final
    complex64 or None)."""
    Kp, Qp = _as_pairs(K, "K"), _as_pairs(Q, "Q")
    dt = v.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = v.device
    if cu_seqlens is not None:
        T, H, dk = Kp.shape[:3]
        B = cu_seqlens.shape[0] - 1
        lead = (T,)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    else:
        B, T, H, dk = Kp.shape[:4]
        lead = (B, T)
    dv = v.shape[-1]
    _need(Kp, "K", torch.float32, (*lead, H, dk, 2), dev)
    _need(Qp, "Q", torch.float32, (*lead, H, dk, 2), dev)
    _need(v, "v", dt, (*lead, H, dv), dev)
    _need(log_r, "log_r", torch.float32, (*lead, H, dv), dev)
    _need(beta, "beta", torch.float32, (*lead, H), dev)
    M0p = _as_pairs(M0, "M0")
    if M0p is not None:
        _need(M0p, "M0", torch.float32, (B, H, dv, dk, 2), dev)
    if out is None:
        out = torch.empty((*lead, H, dv), dtype=dt, device=dev)
    _need(out, "out", dt, (*lead, H, dv), dev)
    Mf = None
    if M_final is not None:
        Mf = torch.view_as_real(M_final) if M_final.is_complex() else M_final
    elif output_final_state:
        Mf = torch.empty((B, H, dv, dk, 2), dtype=torch.float32, device=dev)
    if Mf is not None:
        _need(Mf, "M_final", torch.float32, (B, H, dv, dk, 2), dev)
    rc = gdn_phase_rowdecay_fwd(_ptr(Kp), _ptr(Qp), _ptr(v), _ptr(log_r), _ptr(beta), _ptr(M0p), _ptr(out),
                                _ptr(Mf), B, T, H, dk, dv, _ptr(cu_seqlens), _DT[dt], _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return out, (None if Mf is None else torch.view_as_complex(Mf))


def phase_bwd(K, Q, v, log_lam, beta, dout, M0=None, dM_final=None, cu_seqlens=None, want_dM0=True,
              workspace=None, stream=None):
    """Gradients of ``phase_fwd`` (dk = 32 complex, dv 64, 128 or 256): returns (dK, dQ complex64, dv fp32,
    dlog_lam, dbeta fp32, dM0 complex64 or None); complex gradients as d/dRe + i d/dIm."""
    Kp, Qp = _as_pairs(K, "K"), _as_pairs(Q, "Q")
    dt = v.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = v.device
    if cu_seqlens is not None:
        T, H, dk = Kp.shape[:3]
        B = cu_seqlens.shape[0] - 1
        lead = (T,)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    else:
        B, T, H, dk = Kp.shape[:4]
        lead = (B, T)
    dv = v.shape[-1]
    _need(Kp, "K", torch.float32, (*lead, H, dk, 2), dev)
    _need(Qp, "Q", torch.float32, (*lead, H, dk, 2), dev)
    _need(v, "v", dt, (*lead, H, dv), dev)
    _need(dout, "dout", dt, (*lead, H, dv), dev)
    _need(log_lam, "log_lam", torch.float32, (*lead, H), dev)
    _need(beta, "beta", torch.float32, (*lead, H), dev)
    M0p, dMp = _as_pairs(M0, "M0"), _as_pairs(dM_final, "dM_final")
    for name, x in (("M0", M0p), ("dM_final", dMp)):
        if x is not None:
            _need(x, name, torch.float32, (B, H, dv, dk, 2), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dK, dQ = torch.empty((*lead, H, dk, 2), **f32), torch.empty((*lead, H, dk, 2), **f32)
    dV = torch.empty((*lead, H, dv), **f32)
    dla, dbe = torch.empty((*lead, H), **f32), torch.empty((*lead, H), **f32)
    dM0 = torch.empty((B, H, dv, dk, 2), **f32) if want_dM0 else None
    need = gdn_phase_bwd_workspace_bytes(B, T, H, dk, dv, int(cu_seqlens is not None))
    if need == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_UNSUPPORTED, f"gdn_phase_bwd: unsupported sizes dk={dk} dv={dv}")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    rc = gdn_phase_bwd(_ptr(Kp), _ptr(Qp), _ptr(v), _ptr(log_lam), _ptr(beta), _ptr(M0p), _ptr(dout), _ptr(dMp),
                       _ptr(dK), _ptr(dQ), _ptr(dV), _ptr(dla), _ptr(dbe), _ptr(dM0), B, T, H, dk, dv,
                       _ptr(cu_seqlens), _DT[dt], _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return (torch.view_as_complex(dK), torch.view_as_complex(dQ), dV, dla, dbe,
            None if dM0 is None else torch.view_as_complex(dM0))


def chunk_fwd_fused(q_raw, k_raw, v, a_raw, b_raw, a_scale, b_scale, S0=None, cu_seqlens=None,
                    out=None, S_final=None, output_final_state=True, workspace=None, chunk=64,
                    stream=None):
    """Chunkwise forward with the input prologue in the kernel (bf16): q_raw, k_raw are
    normalised per row, log_alpha = -a_scale softplus(a_raw), beta = b_scale sigmoid(b_raw).
    Layouts as ``chunk_fwd``.  Returns (out, S_final or None)."""
    p = _chunk_prepare(q_raw, k_raw, v, a_raw, b_raw, S0, cu_seqlens, out, S_final,
                       output_final_state, workspace, chunk, ("q_raw", "k_raw", "a_raw", "b_raw"))
    rc = gdn_chunk_fwd_fused(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a_raw), _ptr(b_raw), _ptr(S0),
                             _ptr(p["out"]), _ptr(p["S_final"]), p["B"], p["T"], p["H"], p["dk"],
                             p["dv"], chunk, _ptr(cu_seqlens), _DT[p["dt"]], float(a_scale),
                             float(b_scale), _ptr(p["workspace"]), p["wbytes"], _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return p["out"], p["S_final"]


def chunk_fwd_gva(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, out=None, S_final=None,
                  output_final_state=True, workspace=None, chunk=64, stream=None):
    """Chunkwise forward with grouped value heads: q,k [B,T,Hk,dk], v [B,T,Hv,dv], gates
    [B,T,Hv], states [B,Hv,dk,dv]; value head h reads q/k head h // (Hv // Hk).  Returns
    (out [B,T,Hv,dv], S_final or None)."""
    p = _chunk_prepare(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, output_final_state,
                       workspace, chunk, ("q", "k", "log_alpha", "beta"), grouped=True)
    rc = gdn_chunk_fwd_gva(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                           _ptr(p["out"]), _ptr(p["S_final"]), p["B"], p["T"], p["Hk"], p["H"], p["dk"],
                           p["dv"], chunk, _ptr(cu_seqlens), _DT[p["dt"]], _ptr(p["workspace"]),
                           p["wbytes"], _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return p["out"], p["S_final"]


def chunk_bwd(q, k, v, log_alpha, beta, dout, S0=None, dS_final=None, cu_seqlens=None, want_dS0=True,
              workspace=None, chunk=64, stream=None):
    """Gradients of ``chunk_fwd`` (dk in {64, 128}, dv in {64, 128, 256}): returns fp32 (dq, dk, dv, dlog_alpha, dbeta,
    dS0 or None) for dout = dL/dout and dS_final = dL/dS_final (None: zero)."""
    dt = q.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = q.device
    if cu_seqlens is not None:
        T, H, dk = q.shape
        B = cu_seqlens.shape[0] - 1
        lead = (T,)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    else:
        B, T, H, dk = q.shape
        lead = (B, T)
    dv = v.shape[-1]
    for name, x, shp in (("q", q, (*lead, H, dk)), ("k", k, (*lead, H, dk)), ("v", v, (*lead, H, dv)),
                         ("dout", dout, (*lead, H, dv))):
        _need(x, name, dt, shp, dev)
    _need(log_alpha, "log_alpha", torch.float32, (*lead, H), dev)
    _need(beta, "beta", torch.float32, (*lead, H), dev)
    for name, x in (("S0", S0), ("dS_final", dS_final)):
        if x is not None:
            _need(x, name, torch.float32, (B, H, dk, dv), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dkk, dvv = torch.empty((*lead, H, dk), **f32), torch.empty((*lead, H, dk), **f32), torch.empty((*lead, H, dv), **f32)
    dla, dbe = torch.empty((*lead, H), **f32), torch.empty((*lead, H), **f32)
    dS0 = torch.empty((B, H, dk, dv), **f32) if want_dS0 else None
    need = gdn_chunk_bwd_workspace_bytes(B, T, H, dk, dv, chunk, int(cu_seqlens is not None))
    if need == (1 << 64) - 1:
        raise GdnError(GDN_ERR_UNSUPPORTED, f"gdn_chunk_bwd does not take dk={dk} dv={dv} chunk={chunk}")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    rc = gdn_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(dout),
                       _ptr(dS_final), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dla), _ptr(dbe), _ptr(dS0), B, T,
                       H, dk, dv, chunk, _ptr(cu_seqlens), _DT[dt], _ptr(workspace),
                       workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return dq, dkk, dvv, dla, dbe, dS0


def gdn_chunk_bwd_gva(q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk, dv, dlog_alpha, dbeta, dS0, B, T, Hk,
                      Hv, dk_, dv_, chunk, cu_seqlens, dtype, workspace, workspace_bytes, stream) -> int:
    return _lib.gdn_chunk_bwd_gva(q, k, v, log_alpha, beta, S0, dout, dS_final, dq, dk, dv, dlog_alpha, dbeta, dS0,
                                  B, T, Hk, Hv, dk_, dv_, chunk, cu_seqlens, dtype, workspace, workspace_bytes,
                                  stream)


def gdn_chunk_bwd_gva_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, varlen) -> int:
    return _lib.gdn_chunk_bwd_gva_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, varlen)


def chunk_bwd_gva(q, k, v, log_alpha, beta, dout, S0=None, dS_final=None, cu_seqlens=None, want_dS0=True,
                  workspace=None, chunk=64, stream=None):
    """Gradients of ``chunk_fwd_gva`` (dk = dv = 64): q, k [.., Hk, 64]; v, dout [.., Hv, 64]; returns
    fp32 (dq, dk [.., Hk, 64], dv, dlog_alpha, dbeta, dS0 or None), dq and dk summed over each q/k
    head's value heads."""
    dt = q.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = q.device
    if cu_seqlens is not None:
        T, Hk, dk = q.shape
        B = cu_seqlens.shape[0] - 1
        lead = (T,)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    else:
        B, T, Hk, dk = q.shape
        lead = (B, T)
    Hv, dv = v.shape[-2], v.shape[-1]
    for name, x, shp in (("q", q, (*lead, Hk, dk)), ("k", k, (*lead, Hk, dk)), ("v", v, (*lead, Hv, dv)),
                         ("dout", dout, (*lead, Hv, dv))):
        _need(x, name, dt, shp, dev)
    _need(log_alpha, "log_alpha", torch.float32, (*lead, Hv), dev)
    _need(beta, "beta", torch.float32, (*lead, Hv), dev)
    for name, x in (("S0", S0), ("dS_final", dS_final)):
        if x is not None:
            _need(x, name, torch.float32, (B, Hv, dk, dv), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dkk, dvv = torch.empty((*lead, Hk, dk), **f32), torch.empty((*lead, Hk, dk), **f32), torch.empty((*lead, Hv, dv), **f32)
    dla, dbe = torch.empty((*lead, Hv), **f32), torch.empty((*lead, Hv), **f32)
    dS0 = torch.empty((B, Hv, dk, dv), **f32) if want_dS0 else None
    need = gdn_chunk_bwd_gva_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, int(cu_seqlens is not None))
    if need == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_UNSUPPORTED, f"gdn_chunk_bwd_gva does not take Hk={Hk} Hv={Hv} dk={dk} dv={dv}")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    rc = gdn_chunk_bwd_gva(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(dout),
                           _ptr(dS_final), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dla), _ptr(dbe), _ptr(dS0), B, T,
                           Hk, Hv, dk, dv, chunk, _ptr(cu_seqlens), _DT[dt], _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return dq, dkk, dvv, dla, dbe, dS0


def gdn_chunk_bwd_fused(q_raw, k_raw, v, a_raw, b_raw, S0, dout, dS_final, dq_raw, dk_raw, dv, da_raw, db_raw,
                        dS0, B, T, H, dk, dv_, chunk, cu_seqlens, dtype, a_scale, b_scale, workspace,
                        workspace_bytes, stream) -> int:
    return _lib.gdn_chunk_bwd_fused(q_raw, k_raw, v, a_raw, b_raw, S0, dout, dS_final, dq_raw, dk_raw, dv, da_raw,
                                    db_raw, dS0, B, T, H, dk, dv_, chunk, cu_seqlens, dtype, a_scale, b_scale,
                                    workspace, workspace_bytes, stream)


def gdn_chunk_bwd_fused_workspace_bytes(B, T, H, dk, dv, chunk, varlen) -> int:
    return _lib.gdn_chunk_bwd_fused_workspace_bytes(B, T, H, dk, dv, chunk, varlen)


def chunk_bwd_fused(q_raw, k_raw, v, a_raw, b_raw, dout, a_scale, b_scale, S0=None, dS_final=None,
                    cu_seqlens=None, want_dS0=True, workspace=None, chunk=64, stream=None):
    """Gradients of ``chunk_fwd_fused`` with respect to its raw inputs (dk = 64, dv in {64, 128, 256}): returns fp32
    (dq_raw, dk_raw, dv, da_raw, db_raw, dS0 or None)."""
    dt = q_raw.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = q_raw.device
    if cu_seqlens is not None:
        T, H, dk = q_raw.shape
        B = cu_seqlens.shape[0] - 1
        lead = (T,)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    else:
        B, T, H, dk = q_raw.shape
        lead = (B, T)
    dv = v.shape[-1]
    for name, x, shp in (("q_raw", q_raw, (*lead, H, dk)), ("k_raw", k_raw, (*lead, H, dk)),
                         ("v", v, (*lead, H, dv)), ("dout", dout, (*lead, H, dv))):
        _need(x, name, dt, shp, dev)
    _need(a_raw, "a_raw", torch.float32, (*lead, H), dev)
    _need(b_raw, "b_raw", torch.float32, (*lead, H), dev)
    for name, x in (("S0", S0), ("dS_final", dS_final)):
        if x is not None:
            _need(x, name, torch.float32, (B, H, dk, dv), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dkk, dvv = torch.empty((*lead, H, dk), **f32), torch.empty((*lead, H, dk), **f32), torch.empty((*lead, H, dv), **f32)
    da, db = torch.empty((*lead, H), **f32), torch.empty((*lead, H), **f32)
    dS0 = torch.empty((B, H, dk, dv), **f32) if want_dS0 else None
    need = gdn_chunk_bwd_fused_workspace_bytes(B, T, H, dk, dv, chunk, int(cu_seqlens is not None))
    if need == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_UNSUPPORTED, f"gdn_chunk_bwd_fused does not take dk={dk} dv={dv} chunk={chunk}")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    rc = gdn_chunk_bwd_fused(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a_raw), _ptr(b_raw), _ptr(S0), _ptr(dout),
                             _ptr(dS_final), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(da), _ptr(db), _ptr(dS0), B, T, H,
                             dk, dv, chunk, _ptr(cu_seqlens), _DT[dt], float(a_scale), float(b_scale),
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return dq, dkk, dvv, da, db, dS0


def decode_step_gva(q, k, v, log_alpha, beta, S, out=None, stream=None):
    """One decode step with grouped value heads: q,k [N,Hk,dk], v [N,Hv,dv], gates [N,Hv],
    S [N,Hv,dk,dv] fp32 updated in place.  Returns out [N,Hv,dv]."""
    dt = q.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = q.device
    N, Hk, dk = q.shape
    Hv, dv = v.shape[-2], v.shape[-1]
    _need(q, "q", dt, (N, Hk, dk), dev)
    _need(k, "k", dt, (N, Hk, dk), dev)
    _need(v, "v", dt, (N, Hv, dv), dev)
    _need(log_alpha, "log_alpha", torch.float32, (N, Hv), dev)
    _need(beta, "beta", torch.float32, (N, Hv), dev)
    _need(S, "S", torch.float32, (N, Hv, dk, dv), dev)
    if out is None:
        out = torch.empty((N, Hv, dv), dtype=dt, device=dev)
    _need(out, "out", dt, (N, Hv, dv), dev)
    rc = gdn_decode_step_gva(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S), _ptr(out),
                             N, Hk, Hv, dk, dv, _DT[dt], _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return out


def decode_step(q, k, v, log_alpha, beta, S, out=None, stream=None):
    """One decode step, S [N,H,dk,dv] fp32 updated in place.  Returns out [N,H,dv]."""
    dt = q.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = q.device
    N, H, dk = q.shape
    dv = v.shape[-1]
    _need(q, "q", dt, (N, H, dk), dev)
    _need(k, "k", dt, (N, H, dk), dev)
    _need(v, "v", dt, (N, H, dv), dev)
    _need(log_alpha, "log_alpha", torch.float32, (N, H), dev)
    _need(beta, "beta", torch.float32, (N, H), dev)
    _need(S, "S", torch.float32, (N, H, dk, dv), dev)
    if out is None:
        out = torch.empty((N, H, dv), dtype=dt, device=dev)
    _need(out, "out", dt, (N, H, dv), dev)
    rc = gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S), _ptr(out),
                         N, H, dk, dv, _DT[dt], _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return out


def decode_step_fused(q_raw, k_raw, v, a_raw, b_raw, a_scale, b_scale, S, out=None, stream=None):
    """One decode step from raw projections (``gdn_decode_step_fused``): q_raw, k_raw [N,H,dk]
    unnormalised, a_raw, b_raw [N,H] fp32 raw gate projections; S [N,H,dk,dv] fp32 updated in
    place.  Returns out [N,H,dv]."""
    dt = q_raw.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    dev = q_raw.device
    N, H, dk = q_raw.shape
    dv = v.shape[-1]
    _need(q_raw, "q_raw", dt, (N, H, dk), dev)
    _need(k_raw, "k_raw", dt, (N, H, dk), dev)
    _need(v, "v", dt, (N, H, dv), dev)
    _need(a_raw, "a_raw", torch.float32, (N, H), dev)
    _need(b_raw, "b_raw", torch.float32, (N, H), dev)
    _need(S, "S", torch.float32, (N, H, dk, dv), dev)
    if out is None:
        out = torch.empty((N, H, dv), dtype=dt, device=dev)
    _need(out, "out", dt, (N, H, dv), dev)
    rc = gdn_decode_step_fused(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a_raw), _ptr(b_raw), _ptr(S), _ptr(out),
                               N, H, dk, dv, _DT[dt], float(a_scale), float(b_scale), _stream_ptr(stream))
    if rc != GDN_OK:
        raise GdnError(rc, gdn_last_error())
    return out
