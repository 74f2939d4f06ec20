"""fp64 CPU oracle for the gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library and never imports
it; the only thing both sides use is the seeded input generator in ``workloads.py``.

Two independent computations live here:

* ``forward`` / ``decode_step`` -- the sequential definition (plain C, fp64, OpenMP over
  independent (sequence, head) chains), ``gdn_oracle.c``; ``backward`` -- its gradients by
  reverse mode over the same loop.
* ``chunkwise.forward_chunkwise`` -- the chunkwise WY / UT-transform form in numpy fp64, written
  separately from the algebra, used only to pin the sequential oracle (and vice versa).

Every function returns fp64 numpy arrays.  Inputs may be torch tensors or numpy arrays of any
float dtype; they are upcast exactly to fp64 (bf16 and fp32 values are representable in fp64).

Parity of every function here is pinned by the CPU tests in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``libgdn_oracle.so`` (gcc, -O2, OpenMP, strict IEEE)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math", "-std=c11",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            lib.gdn_oracle_forward.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ip, ip, ctypes.c_int,
                                               ctypes.c_int]
            lib.gdn_oracle_forward.restype = ctypes.c_int
            lib.gdn_oracle_decode_step.argtypes = [dp, dp, dp, dp, dp, dp, dp,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_int]
            lib.gdn_oracle_decode_step.restype = ctypes.c_int
            lib.gdn_oracle_backward.argtypes = [dp] * 14 + [ctypes.c_int] * 5 + [ip, ctypes.c_int]
            lib.gdn_oracle_backward.restype = ctypes.c_int
            lib.gdn_oracle_max_threads.argtypes = []
            lib.gdn_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> exact fp64 copy on the CPU
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _dp(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def max_threads() -> int:
    """Threads the oracle's OpenMP runtime uses by default."""
    return int(_load().gdn_oracle_max_threads())


def forward(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, units=None, nthreads=0,
            want_out=True):
    """Sequential fp64 forward of the recurrence.

    Dense layout: q,k [B,T,H,dk]; v [B,T,H,dv]; log_alpha, beta [B,T,H]; S0 [B,H,dk,dv] or None.
    Varlen (``cu_seqlens`` given, int [B+1]): q,k [T,H,dk] ... packed; B = len(cu_seqlens) - 1.
    ``units``: optional iterable of (sequence * H + head) indices to compute; the other entries
    of the returned arrays are NaN.
    Returns (out, S_final) as fp64 arrays shaped like v and [B,H,dk,dv].
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be = _f64(log_alpha), _f64(beta)
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int32))
        B = cu.shape[0] - 1
        T = int(cu[-1])
        H, dk = q.shape[-2], q.shape[-1]
        assert q.shape[0] == T
    else:
        cu = None
        B, T, H, dk = q.shape
    dv = v.shape[-1]
    S0 = _f64(S0)
    if S0 is not None:
        assert S0.shape == (B, H, dk, dv)
    out = np.full(v.shape, np.nan) if want_out else None
    S_final = np.full((B, H, dk, dv), np.nan)
    if units is not None:
        u = np.ascontiguousarray(np.asarray(list(units), dtype=np.int32))
        n_units = int(u.shape[0])
    else:
        u, n_units = None, 0
    rc = lib.gdn_oracle_forward(_dp(q), _dp(k), _dp(v), _dp(la), _dp(be), _dp(S0), _dp(out),
                                _dp(S_final), B, T, H, dk, dv, _ip(cu), _ip(u), n_units,
                                int(nthreads))
    if rc != 0:
        raise ValueError("gdn_oracle_forward rejected its arguments")
    return out, S_final


def backward(q, k, v, log_alpha, beta, S0, dout, dS_final=None, cu_seqlens=None, nthreads=0):
    """fp64 gradients of ``forward`` by reverse mode over the sequential definition.

    ``dout`` is dL/dout (shaped like v), ``dS_final`` dL/dS_final or None.  Returns
    (dq, dk, dv, dlog_alpha, dbeta, dS0) shaped like the inputs (dS0 [B,H,dk,dv] even when S0 is
    None).  Keeps every state of a sequence in memory: for test-sized inputs.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be = _f64(log_alpha), _f64(beta)
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int32))
        B = cu.shape[0] - 1
        T = int(cu[-1])
        H, dk = q.shape[-2], q.shape[-1]
    else:
        cu = None
        B, T, H, dk = q.shape
    dv = v.shape[-1]
    S0 = _f64(S0)
    dout = _f64(dout)
    dS_final = _f64(dS_final)
    dq, dkk, dvv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dla, dbe = np.zeros(la.shape), np.zeros(be.shape)
    dS0 = np.zeros((B, H, dk, dv))
    rc = lib.gdn_oracle_backward(_dp(q), _dp(k), _dp(v), _dp(la), _dp(be), _dp(S0), _dp(dout),
                                 _dp(dS_final), _dp(dq), _dp(dkk), _dp(dvv), _dp(dla), _dp(dbe),
                                 _dp(dS0), B, T, H, dk, dv, _ip(cu), int(nthreads))
    if rc != 0:
        raise ValueError("gdn_oracle_backward rejected its arguments")
    return dq, dkk, dvv, dla, dbe, dS0


def decode_step(q, k, v, log_alpha, beta, S, nthreads=0):
    """One fp64 decode step.  q,k [N,H,dk]; v [N,H,dv]; gates [N,H]; S [N,H,dk,dv].

    Returns (out [N,H,dv], S_new); the input state is not modified.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be = _f64(log_alpha), _f64(beta)
    S_new = _f64(S).copy()
    N, H, dk = q.shape
    dv = v.shape[-1]
    out = np.empty((N, H, dv))
    rc = lib.gdn_oracle_decode_step(_dp(q), _dp(k), _dp(v), _dp(la), _dp(be), _dp(S_new),
                                    _dp(out), N, H, dk, dv, int(nthreads))
    if rc != 0:
        raise ValueError("gdn_oracle_decode_step rejected its arguments")
    return out, S_new
