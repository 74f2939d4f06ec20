"""fp64 oracle for grouped value heads: Hv value heads share Hk q/k heads, value head h reading
q/k head h // (Hv // Hk) (the sharing grouped-query attention uses, Sykra README, "Architectural
Highlights").

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  The definition written out: each value
head runs the plain recurrence with its group's q/k, so the q/k heads are repeated and the
sequential oracle runs on Hv heads.
"""
from __future__ import annotations

import numpy as np

import oracle


def _expand(x, G):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.repeat(np.asarray(x, dtype=np.float64), G, axis=-2)


def forward_gva(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, units=None):
    """q,k [..., Hk, dk]; v [..., Hv, dv]; gates [..., Hv]; S0 [B, Hv, dk, dv] or None."""
    Hk, Hv = q.shape[-2], v.shape[-2]
    assert Hv % Hk == 0
    G = Hv // Hk
    return oracle.forward(_expand(q, G), _expand(k, G), v, log_alpha, beta, S0, cu_seqlens=cu_seqlens,
                          units=units)


def decode_step_gva(q, k, v, log_alpha, beta, S):
    """q,k [N, Hk, dk]; v [N, Hv, dv]; gates [N, Hv]; S [N, Hv, dk, dv] (fp64, not modified)."""
    G = v.shape[-2] // q.shape[-2]
    return oracle.decode_step(_expand(q, G), _expand(k, G), v, log_alpha, beta, S)


def backward_gva(q, k, v, log_alpha, beta, S0, dout, dS_final=None, cu_seqlens=None):
    """fp64 gradients of ``forward_gva``: the backward oracle on the Hv heads with q/k repeated,
    then dq, dk of each q/k head summed over the G value heads that read it (the chain rule of
    the repeat).  Returns (dq, dk [.., Hk, dk], dv, dlog_alpha, dbeta [.., Hv], dS0)."""
    Hk, Hv = q.shape[-2], v.shape[-2]
    G = Hv // Hk
    dq, dk, dv, dla, dbe, dS0 = oracle.backward(_expand(q, G), _expand(k, G), v, log_alpha, beta, S0, dout,
                                                dS_final, cu_seqlens=cu_seqlens)
    lead = dq.shape[:-2]
    dq = dq.reshape(*lead, Hk, G, dq.shape[-1]).sum(axis=-2)
    dk = dk.reshape(*lead, Hk, G, dk.shape[-1]).sum(axis=-2)
    return dq, dk, dv, dla, dbe, dS0
