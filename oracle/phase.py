"""fp64 oracle of the complex-phase delta memory (DeltaPhase README, section 2 "Complex Phase Matrix
Delta Memory", with its gated-decay form; section 5 "Delta-Laplace Phase Memory Core" for keys
e^{s dt}, Re s <= 0).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): only tests/, the package's smoke check and
bench.py's CPU baseline may import this module.

Per (sequence, head) a complex state M in C^{dv x dk}; per token t, with complex key K_t and query
Q_t (dk), real value V_t (dv), and scalars lam_t = exp(log_lam_t) in (0, 1] and beta_t:

    v_old = (1/dk) Re(M_{t-1} conj(K_t))       read-out of the key from the previous state
    e_t   = V_t - v_old                         error signal
    M_t   = lam_t M_{t-1} + beta_t e_t K_t^T    decayed state plus the rank-one correction
    o_t   = (1/dk) Re(M_t conj(Q_t))            read-out of the query

The first three lines are the section's three steps with the gated decay; the read-out of the
query (post-update state, the key's 1/dk scale) and lam_t as one scalar per (token, head) are
readings (the section prints no query read-out).

``forward_rowdecay`` is the Laplace core's per-row form (section 5, "Exact Chunkwise-Parallel
Scan"): the decay is diag(r_t), one factor r_t,j = exp(log_r_t,j) per output row j of M (value
channel), M_t = diag(r_t) M_{t-1} + beta_t e_t K_t^T with e_t and o_t as above.  Reading: r_t is
an input per (token, head, channel), as lam_t is in the scalar form, and finite in log (r > 0).  ``forward_rowdecay_chunkwise``
is its chunk form, with the per-channel triangular solve the section describes.

``forward`` is that definition token by token in complex128.  ``forward_chunkwise`` is the chunk
form derived separately (a unit-lower triangular solve per chunk for the errors), used as a pin.

Inputs: K, Q complex arrays [..., H, dk] or real arrays [..., H, dk, 2] (re, im); V [..., H, dv];
log_lam, beta [..., H]; M0 [B, H, dv, dk] complex (or [..., 2] real) or None (zero).  Dense
tensors have leading [B, T]; with cu_seqlens they are packed [T_total, ...].
Returns (out [..., H, dv] float64, M_final [B, H, dv, dk] complex128).
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _np(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        x = x.double() if not x.is_complex() else x.to(dtype=__import__("torch").complex128)
        x = x.numpy()
    return np.asarray(x)


def as_complex(x):
    """Complex128 view of a complex array or of a real array whose last axis is (re, im)."""
    x = _np(x)
    if x is None:
        return None
    if np.iscomplexobj(x):
        return x.astype(np.complex128)
    assert x.shape[-1] == 2, x.shape
    x = x.astype(np.float64)
    return x[..., 0] + 1j * x[..., 1]


def _real(x):
    x = _np(x)
    return None if x is None else x.astype(np.float64)


def _sequences(n_lead, cu_seqlens, T_dense):
    """(sequence index, token slice) for dense [B, T] or packed inputs."""
    if cu_seqlens is None:
        return [(b, None) for b in range(n_lead)]
    cu = np.asarray(_np(cu_seqlens), dtype=np.int64)
    return [(s, slice(int(cu[s]), int(cu[s + 1]))) for s in range(len(cu) - 1)]


def forward(K, Q, V, log_lam, beta, M0=None, cu_seqlens=None):
    """The definition, token by token (all (sequence, head) chains of a dense batch at once)."""
    K, Q, M0 = as_complex(K), as_complex(Q), as_complex(M0)
    V, la, be = _real(V), _real(log_lam), _real(beta)
    dk, dv = K.shape[-1], V.shape[-1]
    H = V.shape[-2]
    out = np.zeros(V.shape)
    if cu_seqlens is None:
        B, T = V.shape[:2]
        M = np.zeros((B, H, dv, dk), np.complex128) if M0 is None else M0.copy()
        for t in range(T):
            k, q = K[:, t], Q[:, t]                      # [B, H, dk]
            v_old = np.einsum("bhji,bhi->bhj", M, np.conj(k)).real / dk
            e = V[:, t] - v_old                          # [B, H, dv]
            lam = np.exp(la[:, t])[..., None, None]
            M = lam * M + (be[:, t, :, None] * e)[..., :, None] * k[..., None, :]
            out[:, t] = np.einsum("bhji,bhi->bhj", M, np.conj(q)).real / dk
        return out, M
    seqs = _sequences(None, cu_seqlens, None)
    Mf = np.zeros((len(seqs), H, dv, dk), np.complex128)
    for s, sl in seqs:
        M = np.zeros((H, dv, dk), np.complex128) if M0 is None else M0[s].copy()
        for t in range(sl.start, sl.stop):
            v_old = np.einsum("hji,hi->hj", M, np.conj(K[t])).real / dk
            e = V[t] - v_old
            M = np.exp(la[t])[:, None, None] * M + (be[t][:, None] * e)[:, :, None] * K[t][:, None, :]
            out[t] = np.einsum("hji,hi->hj", M, np.conj(Q[t])).real / dk
        Mf[s] = M
    return out, Mf


def _chunk(M0, K, Q, V, la, be):
    """One chunk of one (sequence, head): M0 [dv, dk]; K, Q [C, dk]; V [C, dv]; la, be [C].

    With g_t the sum of log_lam over the chunk's tokens up to t (g_{-1} = 0), the state before
    token t is M_{t-1} = e^{g_{t-1}} M0 + sum_{s<t} e^{g_{t-1} - g_s} beta_s e_s K_s^T, so the errors
    solve (I + A) E = V - (1/dk) diag(e^{g_{t-1}}) Re(conj(K) M0^T) with
    A_ts = (1/dk) e^{g_{t-1} - g_s} beta_s Re(K_s . conj K_t) for s < t; then the outputs and the
    exit state follow from E in closed form.
    """
    C, dk = K.shape
    g = np.cumsum(la)
    g_prev = np.concatenate([[0.0], g[:-1]])
    gram_k = (K @ np.conj(K).T).real               # [s, t] -> Re(K_s . conj K_t)
    gram_q = (K @ np.conj(Q).T).real               # [s, t] -> Re(K_s . conj Q_t)
    t_idx, s_idx = np.meshgrid(np.arange(C), np.arange(C), indexing="ij")
    A = np.where(s_idx < t_idx, np.exp(g_prev[:, None] - g[None, :]) * be[None, :] * gram_k.T, 0.0) / dk
    rhs = V - np.exp(g_prev)[:, None] * (np.conj(K) @ M0.T).real / dk
    E = solve_triangular(np.eye(C) + A, rhs, lower=True, unit_diagonal=True)
    P = np.where(s_idx <= t_idx, np.exp(g[:, None] - g[None, :]) * be[None, :] * gram_q.T, 0.0)
    O = (np.exp(g)[:, None] * (np.conj(Q) @ M0.T).real + P @ E) / dk
    w = be * np.exp(g[-1] - g)
    M_end = np.exp(g[-1]) * M0 + (E * w[:, None]).T @ K
    return O, M_end


def forward_chunkwise(K, Q, V, log_lam, beta, M0=None, chunk=64, cu_seqlens=None):
    """The chunk form: the same results as ``forward`` up to rounding."""
    K, Q, M0 = as_complex(K), as_complex(Q), as_complex(M0)
    V, la, be = _real(V), _real(log_lam), _real(beta)
    dk, dv = K.shape[-1], V.shape[-1]
    H = V.shape[-2]
    out = np.zeros(V.shape)
    if cu_seqlens is None:
        B, T = V.shape[:2]
        runs = [(b, (b, slice(0, T))) for b in range(B)]
    else:
        runs = [(s, (sl,)) for s, sl in _sequences(None, cu_seqlens, None)]
    Mf = np.zeros((len(runs), H, dv, dk), np.complex128)
    for s, idx in runs:
        sl = idx[-1]
        for h in range(H):
            M = np.zeros((dv, dk), np.complex128) if M0 is None else M0[s, h].copy()
            for c0 in range(sl.start, sl.stop, chunk):
                c1 = min(c0 + chunk, sl.stop)
                rows = (*idx[:-1], slice(c0, c1), h)
                O, M = _chunk(M, K[rows], Q[rows], V[rows], la[rows], be[rows])
                out[rows] = O
            Mf[s, h] = M
    return out, Mf


def backward(K, Q, V, log_lam, beta, M0, dout, dM_final=None, cu_seqlens=None):
    """fp64 gradients of ``forward`` with respect to (K, Q, V, log_lam, beta, M0) for the loss
    gradients dout (dL/d out) and dM_final (dL/d M_final, complex: d/dRe + i d/dIm; None = 0).
    Complex gradients are returned the same way (d/dRe + i d/dIm).

    Through the real form of the recurrence (the module doc: S = [Re M | Im M]^T, head size 2 dk,
    a = lam, b = beta / lam, k = (Re K, Im K) / sqrt(dk), v = lam sqrt(dk) V, q = (Re Q, Im Q) / dk):
    the real backward oracle, then the chain rule of that map --
    dK = dk / sqrt(dk), dQ = dq / dk, dV = lam sqrt(dk) dv, dbeta = db / lam,
    dlog_lam = dlog_a + sum_j dv_j v_j - db b.  Pinned against finite differences of ``forward``."""
    import oracle
    K, Q, M0, dMf = as_complex(K), as_complex(Q), as_complex(M0), as_complex(dM_final)
    V, la, be, dO = _real(V), _real(log_lam), _real(beta), _real(dout)
    dk = K.shape[-1]
    lam = np.exp(la)
    k = np.concatenate([K.real, K.imag], axis=-1) / np.sqrt(dk)
    q = np.concatenate([Q.real, Q.imag], axis=-1) / dk
    v = lam[..., None] * np.sqrt(dk) * V
    b = be / lam

    def to_real_state(M):
        return None if M is None else np.concatenate([M.real, M.imag], axis=-1).swapaxes(-1, -2)
    dq, dkr, dv, dla, db, dS0 = oracle.backward(q, k, v, la, b, to_real_state(M0), dO, to_real_state(dMf),
                                                cu_seqlens=cu_seqlens)
    dK = (dkr[..., :dk] + 1j * dkr[..., dk:]) / np.sqrt(dk)
    dQ = (dq[..., :dk] + 1j * dq[..., dk:]) / dk
    dV = lam[..., None] * np.sqrt(dk) * dv
    dlog_lam = dla + np.sum(dv * v, axis=-1) - db * b
    dS0 = dS0.swapaxes(-1, -2)
    dM0 = dS0[..., :dk] + 1j * dS0[..., dk:]
    return dK, dQ, dV, dlog_lam, db / lam, dM0


def forward_rowdecay(K, Q, V, log_r, beta, M0=None, cu_seqlens=None):
    """The per-row-decay definition, token by token: log_r [..., H, dv] (one decay per value
    channel); otherwise as ``forward``."""
    K, Q, M0 = as_complex(K), as_complex(Q), as_complex(M0)
    V, lr, be = _real(V), _real(log_r), _real(beta)
    dk, dv = K.shape[-1], V.shape[-1]
    H = V.shape[-2]
    out = np.zeros(V.shape)
    if cu_seqlens is None:
        B, T = V.shape[:2]
        runs = [(b, [(b, t) for t in range(T)]) for b in range(B)]
    else:
        runs = [(s, [(t,) for t in range(sl.start, sl.stop)]) for s, sl in _sequences(None, cu_seqlens, None)]
    Mf = np.zeros((len(runs), H, dv, dk), np.complex128)
    for s, toks in runs:
        M = np.zeros((H, dv, dk), np.complex128) if M0 is None else M0[s].copy()
        for idx in toks:
            k, q = K[idx], Q[idx]                                   # [H, dk]
            e = V[idx] - np.einsum("hji,hi->hj", M, np.conj(k)).real / dk
            M = np.exp(lr[idx])[:, :, None] * M + (be[idx][:, None] * e)[:, :, None] * k[:, None, :]
            out[idx] = np.einsum("hji,hi->hj", M, np.conj(q)).real / dk
        Mf[s] = M
    return out, Mf


def _chunk_rowdecay(M0, K, Q, V, lr, be):
    """One chunk of one (sequence, head) with per-channel decays: M0 [dv, dk]; K, Q [C, dk]; V, lr
    [C, dv]; be [C].  With g_t,j the sum of log_r over the chunk's tokens up to t (g_-1 = 0), channel
    j's errors solve its own unit-lower system (I + A_j) e_j = v_j - (1/dk) e^{g_{t-1},j}
    Re(conj(K) M0^T)[:, j], A_j[t, s] = (1/dk) e^{g_{t-1},j - g_s,j} beta_s Re(K_s . conj K_t) for
    s < t: the phasor Gram is shared, the decay weighting is the channel's own."""
    C, dk = K.shape
    dv = V.shape[1]
    g = np.cumsum(lr, axis=0)                                        # [C, dv]
    g_prev = np.concatenate([np.zeros((1, dv)), g[:-1]])
    gram_k = (K @ np.conj(K).T).real                                 # [s, t]
    gram_q = (K @ np.conj(Q).T).real
    read0 = (np.conj(K) @ M0.T).real / dk                            # [C, dv]
    readq = (np.conj(Q) @ M0.T).real / dk
    E = np.zeros((C, dv))
    O = np.zeros((C, dv))
    M_end = np.zeros_like(M0)
    lower = np.tril(np.ones((C, C)), -1) > 0
    incl = np.tril(np.ones((C, C))) > 0
    for j in range(dv):
        A = np.where(lower, np.exp(g_prev[:, j][:, None] - g[:, j][None, :]) * be[None, :] * gram_k.T, 0.0) / dk
        E[:, j] = solve_triangular(np.eye(C) + A, V[:, j] - np.exp(g_prev[:, j]) * read0[:, j], lower=True,
                                   unit_diagonal=True)
        P = np.where(incl, np.exp(g[:, j][:, None] - g[:, j][None, :]) * be[None, :] * gram_q.T, 0.0) / dk
        O[:, j] = np.exp(g[:, j]) * readq[:, j] + P @ E[:, j]
        w = be * np.exp(g[-1, j] - g[:, j])
        M_end[j] = np.exp(g[-1, j]) * M0[j] + (E[:, j] * w) @ K
    return O, M_end


def forward_rowdecay_chunkwise(K, Q, V, log_r, beta, M0=None, chunk=64, cu_seqlens=None):
    """The per-row-decay chunk form: the same results as ``forward_rowdecay`` up to rounding."""
    K, Q, M0 = as_complex(K), as_complex(Q), as_complex(M0)
    V, lr, be = _real(V), _real(log_r), _real(beta)
    dk, dv = K.shape[-1], V.shape[-1]
    H = V.shape[-2]
    out = np.zeros(V.shape)
    if cu_seqlens is None:
        B, T = V.shape[:2]
        runs = [(b, (b, slice(0, T))) for b in range(B)]
    else:
        runs = [(s, (sl,)) for s, sl in _sequences(None, cu_seqlens, None)]
    Mf = np.zeros((len(runs), H, dv, dk), np.complex128)
    for s, idx in runs:
        sl = idx[-1]
        for h in range(H):
            M = np.zeros((dv, dk), np.complex128) if M0 is None else M0[s, h].copy()
            for c0 in range(sl.start, sl.stop, chunk):
                c1 = min(c0 + chunk, sl.stop)
                rows = (*idx[:-1], slice(c0, c1), h)
                O, M = _chunk_rowdecay(M, K[rows], Q[rows], V[rows], lr[rows], be[rows])
                out[rows] = O
            Mf[s, h] = M
    return out, Mf
