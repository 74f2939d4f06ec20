"""Chunkwise WY / UT-transform form of the gated delta rule, numpy fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  This is a second, independently written
computation of the same result as the sequential oracle.  The CPU tests check each against the
other on tiny inputs, so a slip in either fails.  It follows the chunkwise formulation the pages
name -- Sykra README, "Architectural Highlights" (chunkwise parallel training through the WY / unit
triangular transform, a triangular solve per chunk); DeltaPhase README, section 1 ("Fast
Triangular Solve", an exact O(C^2) per-chunk transition solve) -- written out for the real-valued
gated recurrence
    S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T,   o_t = S_t^T q_t.

For one chunk of C tokens (rows r = 0..C-1) entered with state S:
    Gam[r,i] = prod_{j=i+1..r} a_j      (i <= r; decay from token i to token r; Gam[r,r] = 1)
    gam[r]   = prod_{j=0..r}   a_j      (decay from the chunk start to token r, inclusive)
    lam[i]   = Gam[C-1,i]               (decay from token i to the chunk end)
    A  = strictly_lower( diag(b) (Gam o K K^T) )
    T  = (I + A)^{-1}                   unit lower triangular
    W  = T diag(b * gam) K
    Ut = T diag(b) V
    U  = Ut - W S                       row r is u_r = b_r (v_r - a_r S_{r-1}^T k_r)
    O  = diag(gam) Q S + lower_inclusive(Gam o Q K^T) U
    S' = gam[C-1] S + (diag(lam) K)^T U

The decays are formed as plain products of a_j in fp64 (no logarithms, no division), so a gate of
exactly zero (log_alpha = -inf) needs no special case.  The triangular inverse uses the textbook
routine ``scipy.linalg.solve_triangular`` as a single step.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular

from . import _f64


def _decays(a: np.ndarray):
    C = a.shape[0]
    Gam = np.zeros((C, C))
    for r in range(C):
        p = 1.0
        Gam[r, r] = 1.0
        for i in range(r - 1, -1, -1):
            p *= a[i + 1]
            Gam[r, i] = p
    gam = np.cumprod(a)
    lam = Gam[C - 1, :].copy()
    return Gam, gam, lam


def unit_lower_inverse(A: np.ndarray) -> np.ndarray:
    """T = (I + A)^{-1} for strictly lower triangular A (textbook triangular solve)."""
    C = A.shape[0]
    I = np.eye(C)
    return solve_triangular(I + A, I, lower=True, unit_diagonal=True)


def chunk_step(S, Q, K, V, log_alpha, beta):
    """One chunk of the WY / UT form.  Returns (O [C,dv], S' [dk,dv], pieces dict)."""
    a = np.exp(log_alpha)
    b = beta
    C = K.shape[0]
    Gam, gam, lam = _decays(a)
    A = np.tril(b[:, None] * (Gam * (K @ K.T)), k=-1)
    T = unit_lower_inverse(A)
    W = T @ ((b * gam)[:, None] * K)
    Ut = T @ (b[:, None] * V)
    U = Ut - W @ S
    P = np.tril(Gam * (Q @ K.T), k=0)
    O = gam[:, None] * (Q @ S) + P @ U
    S_next = gam[C - 1] * S + (lam[:, None] * K).T @ U
    return O, S_next, dict(A=A, T=T, W=W, Ut=Ut, U=U, P=P, gam=gam, lam=lam, Gam=Gam)


def forward_chunkwise(q, k, v, log_alpha, beta, S0=None, chunk=64, cu_seqlens=None):
    """Chunkwise fp64 forward, same layouts and return values as ``oracle.forward``.

    Each sequence is cut into chunks from its own first token; the last chunk may be shorter
    (a shorter chunk is the same formula with a smaller C).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be = _f64(log_alpha), _f64(beta)
    if cu_seqlens is not None:
        cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                        dtype=np.int64)
        B = cu.shape[0] - 1
        H, dk = q.shape[1], q.shape[2]
        spans = [(int(cu[s]), int(cu[s + 1])) for s in range(B)]
        qf, kf, vf, laf, bef = q, k, v, la, be
    else:
        B, T, H, dk = q.shape
        spans = [(s * T, (s + 1) * T) for s in range(B)]
        qf, kf, vf = q.reshape(B * T, H, dk), k.reshape(B * T, H, dk), v.reshape(B * T, H, -1)
        laf, bef = la.reshape(B * T, H), be.reshape(B * T, H)
    dv = v.shape[-1]
    S0 = _f64(S0)
    out = np.empty_like(vf)
    S_final = np.empty((B, H, dk, dv))
    for s, (t0, t1) in enumerate(spans):
        for h in range(H):
            S = S0[s, h].copy() if S0 is not None else np.zeros((dk, dv))
            for c0 in range(t0, t1, chunk):
                c1 = min(c0 + chunk, t1)
                O, S, _ = chunk_step(S, qf[c0:c1, h], kf[c0:c1, h], vf[c0:c1, h],
                                     laf[c0:c1, h], bef[c0:c1, h])
                out[c0:c1, h] = O
            S_final[s, h] = S
    return out.reshape(v.shape), S_final
